"""Thin Python binding of ``libternary_decoder.so`` (argument marshalling only).

Every function here checks tensor properties, passes raw pointers and the
current CUDA stream to the C entry point of the same name (``tw_`` prefix in
C) and raises ``TernaryError`` on a non-zero status.  All arithmetic runs in
the library's CUDA kernels; there is no fallback: importing this module
fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libternary_decoder.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m ternary_weight_decoder_b200.build` "
        "(or __graft_entry__.build()); there is no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

TW_OK = 0
STATUS = {0: "TW_OK", 1: "TW_ERR_NULL", 2: "TW_ERR_SHAPE", 3: "TW_ERR_ALIGN",
          4: "TW_ERR_BUFSIZE", 5: "TW_ERR_NONFINITE", 6: "TW_ERR_CUDA",
          7: "TW_ERR_TIMEOUT", 8: "TW_ERR_CORRUPT", 9: "TW_ERR_UNSUPPORTED"}


class TernaryError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_i64, _sz, _p, _int = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


tw_packed_bytes = _sig("tw_packed_bytes", _sz, [_i64, _i64])
tw_ternarize_workspace_bytes = _sig("tw_ternarize_workspace_bytes", _sz, [_i64, _i64])
tw_ternarize_pack = _sig("tw_ternarize_pack", _int,
                         [_p, _i64, _i64, _p, _sz, _p, _p, _p, _sz, _p])
tw_ternarize_pack_noalloc = _sig("tw_ternarize_pack_noalloc", _int,
                                 [_p, _i64, _i64, _p, _sz, _p, _p, _p])
NOALLOC_MAX_N = 32768
tw_unpack_codes = _sig("tw_unpack_codes", _int, [_p, _i64, _i64, _p, _p, _p])
tw_quantize_act = _sig("tw_quantize_act", _int, [_p, _i64, _i64, _p, _p, _p, _p])
tw_linear_workspace_bytes = _sig("tw_linear_workspace_bytes", _sz, [_i64, _i64, _i64])
tw_ternary_linear = _sig("tw_ternary_linear", _int,
                         [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p, _sz, _p])
tw_ternary_linear_q = _sig("tw_ternary_linear_q", _int,
                           [_p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p, _sz, _p])
tw_sweep_table_bytes = _sig("tw_sweep_table_bytes", _sz, [_int])
tw_sweep_table_encode = _sig("tw_sweep_table_encode", _int, [_p, _int, _i64, _p, _sz])
tw_sweep_table_encode_gemm = _sig("tw_sweep_table_encode_gemm", _int,
                                  [_p, _int, _i64, _int, _p, _sz])
SWEEP_GEMM = {"auto": 0, "expanded": 1}   # TW_SWEEP_GEMM_AUTO, TW_SWEEP_GEMM_EXPANDED
tw_sweep_workspace_bytes = _sig("tw_sweep_workspace_bytes", _sz, [_p])
tw_decoder_projection_sweep = _sig("tw_decoder_projection_sweep", _int, [_p, _p, _p, _sz, _p])
tw_sweep_launches = _sig("tw_sweep_launches", _int, [_p])
tw_check = _sig("tw_check", _int, [_p])
tw_last_error = _sig("tw_last_error", ctypes.c_char_p, [])
tw_debug_wait_timeout = _sig("tw_debug_wait_timeout", _int, [ctypes.c_uint64, _p])
tw_chain_workspace_bytes = _sig("tw_chain_workspace_bytes", _sz, [_p, _int])
tw_decoder_chain = _sig("tw_decoder_chain", _int, [_p, _int, _p, _p, _sz, _p])
tw_chain_launches = _sig("tw_chain_launches", _int, [_p, _int])
tw_chain_plan_bytes = _sig("tw_chain_plan_bytes", _sz, [_int])
tw_chain_plan_encode = _sig("tw_chain_plan_encode", _int, [_p, _int, _p, _p, _sz])
tw_chain_fused_workspace_bytes = _sig("tw_chain_fused_workspace_bytes", _sz, [_p])
tw_chain_fused_launches = _sig("tw_chain_fused_launches", _int, [_p])
tw_decoder_chain_fused = _sig("tw_decoder_chain_fused", _int, [_p, _p, _p, _sz, _p])
tw_pack_slice = _sig("tw_pack_slice", _int, [_p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _sz, _p])
tw_row_absmax = _sig("tw_row_absmax", _int, [_p, _i64, _i64, _p, _p])
tw_quantize_act_given = _sig("tw_quantize_act_given", _int, [_p, _i64, _i64, _p, _p, _p, _p])
tw_rescale_acc = _sig("tw_rescale_acc", _int, [_p, _i64, _i64, _p, _p, _p, _p])
tw_i8_workspace_bytes = _sig("tw_i8_workspace_bytes", _sz, [_i64, _i64])
tw_i8_quantize_weights = _sig("tw_i8_quantize_weights", _int, [_p, _i64, _i64, _p, _p, _p])
tw_i8_linear_q = _sig("tw_i8_linear_q", _int,
                      [_p, _p, _i64, _i64, _i64, _p, _p, _p, _int, _p, _p, _p])
tw_i8_linear = _sig("tw_i8_linear", _int,
                    [_p, _i64, _i64, _i64, _p, _p, _p, _int, _p, _p, _p, _sz, _p])


class ProjDesc(ctypes.Structure):
    """Mirror of ``tw_proj_desc``."""
    _fields_ = [("x", _p), ("xq", _p), ("amax", _p), ("qsum", _p), ("packed", _p),
                ("wscale", _p), ("y", _p), ("acc_out", _p), ("N", _i64), ("K", _i64)]


def _raise(status: int):
    if status != TW_OK:
        raise TernaryError(status, tw_last_error().decode(errors="replace"))


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, device=True):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def check(stream=None):
    """Synchronise and raise if a kernel recorded an error."""
    _raise(tw_check(_stream(stream)))


def packed_bytes(N: int, K: int) -> int:
    return int(tw_packed_bytes(N, K))


def ternarize_pack(W: torch.Tensor, stream=None):
    """W [N, K] fp32 (CUDA) -> (packed uint8, mean_abs float64[1], wscale float32[1])."""
    _need(W, torch.float32, "W")
    N, K = W.shape
    dev = W.device
    packed = torch.empty(max(packed_bytes(N, K), 16), dtype=torch.uint8, device=dev)
    mean_abs = torch.empty(2, dtype=torch.float64, device=dev)
    wscale = torch.empty(4, dtype=torch.float32, device=dev)
    wsb = int(tw_ternarize_workspace_bytes(N, K))
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    _raise(tw_ternarize_pack(_ptr(W), N, K, _ptr(packed), packed.numel(), _ptr(mean_abs),
                             _ptr(wscale), _ptr(ws), wsb, _stream(stream)))
    return packed, mean_abs[:1], wscale[:1]


def ternarize_pack_noalloc(W: torch.Tensor, packed=None, mean_abs=None, wscale=None,
                           stream=None):
    """Like ternarize_pack, through the entry point that takes no scratch
    (for callers that cannot allocate device memory at the call site).
    Outputs may be passed in pre-allocated; N <= NOALLOC_MAX_N."""
    _need(W, torch.float32, "W")
    N, K = W.shape
    dev = W.device
    if packed is None:
        packed = torch.empty(max(packed_bytes(N, K), 16), dtype=torch.uint8, device=dev)
    if mean_abs is None:
        mean_abs = torch.empty(2, dtype=torch.float64, device=dev)
    if wscale is None:
        wscale = torch.empty(4, dtype=torch.float32, device=dev)
    _raise(tw_ternarize_pack_noalloc(_ptr(W), N, K, _ptr(packed), packed.numel(),
                                     _ptr(mean_abs), _ptr(wscale), _stream(stream)))
    return packed, mean_abs[:1], wscale[:1]


def unpack_codes(packed: torch.Tensor, N: int, K: int, stream=None):
    """-> (codes int8 [N, K], invalid_count int32[1])."""
    _need(packed, torch.uint8, "packed")
    codes = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    invalid = torch.zeros(4, dtype=torch.int32, device=packed.device)
    _raise(tw_unpack_codes(_ptr(packed), N, K, _ptr(codes), _ptr(invalid), _stream(stream)))
    return codes, invalid[:1]


def quantize_act(x: torch.Tensor, stream=None):
    """x [M, K] fp32 -> (xq int8 [M, K], amax fp32 [M], qsum int32 [M])."""
    _need(x, torch.float32, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    amax = torch.empty(M, dtype=torch.float32, device=x.device)
    qsum = torch.empty(M, dtype=torch.int32, device=x.device)
    _raise(tw_quantize_act(_ptr(x), M, K, _ptr(xq), _ptr(amax), _ptr(qsum), _stream(stream)))
    return xq, amax, qsum


def linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(tw_linear_workspace_bytes(M, N, K))


def ternary_linear(x: torch.Tensor, packed: torch.Tensor, wscale: torch.Tensor, N: int,
                   y: torch.Tensor | None = None, acc_out: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None, stream=None):
    """y [M, N] fp32 = the ternary layer on x [M, K] fp32; acc_out optional int32 [M, N]."""
    _need(x, torch.float32, "x")
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    wsb = linear_workspace_bytes(M, N, K)
    if ws is None and wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    _raise(tw_ternary_linear(_ptr(x), M, N, K, _ptr(packed), _ptr(wscale), _ptr(y),
                             _ptr(acc_out), _ptr(ws), ws.numel() if ws is not None else 0,
                             _stream(stream)))
    return y


def ternary_linear_q(xq, amax, qsum, packed, wscale, N: int, y=None, acc_out=None, ws=None,
                     stream=None):
    """y [M, N] fp32 from pre-quantised xq [M, K] int8, amax [M], qsum [M]."""
    _need(xq, torch.int8, "xq")
    M, K = xq.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=xq.device)
    wsb = linear_workspace_bytes(M, N, K)
    if ws is None and wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=xq.device)
    _raise(tw_ternary_linear_q(_ptr(xq), _ptr(amax), _ptr(qsum), M, N, K, _ptr(packed),
                               _ptr(wscale), _ptr(y), _ptr(acc_out), _ptr(ws),
                               ws.numel() if ws is not None else 0, _stream(stream)))
    return y


def _dp(d, key):
    """Device address of d[key]: a tensor, a raw int address, or None."""
    v = d.get(key)
    if v is None:
        return None
    return v if isinstance(v, int) else v.data_ptr()


class SweepTable:
    """An encoded sweep over many projections: the host bytes written by
    ``tw_sweep_table_encode`` and their device copy.  The table holds
    references to the tensors its descriptors name (it stores their
    addresses), so they stay allocated for as long as the table does.
    ``gemm`` picks the GEMM of a sweep of more than 32 tokens: "auto" (by M)
    or "expanded" (the expanded-weights kernel at every M > 32;
    ``tw_sweep_table_encode_gemm``)."""

    def __init__(self, descs: Sequence[dict], M: int, device=None, workspace: bool = True,
                 gemm: str = "auto"):
        n = len(descs)
        arr = (ProjDesc * n)()
        for i, d in enumerate(descs):
            arr[i] = ProjDesc(
                x=_dp(d, "x"), xq=_dp(d, "xq"), amax=_dp(d, "amax"), qsum=_dp(d, "qsum"),
                packed=_dp(d, "packed"), wscale=_dp(d, "wscale"), y=_dp(d, "y"),
                acc_out=_dp(d, "acc_out"), N=int(d["N"]), K=int(d["K"]))
        nbytes = int(tw_sweep_table_bytes(n))
        self.host = torch.empty(nbytes, dtype=torch.uint8).pin_memory() \
            if torch.cuda.is_available() else torch.empty(nbytes, dtype=torch.uint8)
        _raise(tw_sweep_table_encode_gemm(arr, n, M, SWEEP_GEMM[gemm], _ptr(self.host), nbytes))
        self.count, self.M, self.gemm = n, M, gemm
        self.descs = [dict(d) for d in descs]   # owns what the records point at
        self.device = None
        if device is not None:
            self.device = self.host.to(device, non_blocking=False)
        wsb = int(tw_sweep_workspace_bytes(_ptr(self.host)))
        self.launches = int(tw_sweep_launches(_ptr(self.host)))
        # decode scratch: the quantised rows and their scales (rewritten by
        # every call)
        self.ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=device) \
            if device is not None and workspace else None
        self.ws_bytes = wsb


def decoder_projection_sweep(table: SweepTable, stream=None):
    """Run every projection of ``table`` (one persistent launch for decode)."""
    _raise(tw_decoder_projection_sweep(_ptr(table.host), _ptr(table.device), _ptr(table.ws),
                                       table.ws_bytes, _stream(stream)))


def debug_wait_timeout(timeout_ns: int, stream=None):
    _raise(tw_debug_wait_timeout(timeout_ns, _stream(stream)))


# ------------------------------------------------------ decoder-layer chain
class ChainBuffers(ctypes.Structure):
    """Mirror of ``tw_chain_buffers``."""
    _fields_ = [("h", _p), ("v", _p), ("a", _p), ("o", _p), ("h1", _p), ("g", _p), ("u", _p),
                ("act", _p), ("d", _p), ("M", _i64), ("hidden", _i64), ("kv_dim", _i64),
                ("head_dim", _i64), ("inter", _i64)]


class ChainLayer(ctypes.Structure):
    """Mirror of ``tw_chain_layer``."""
    _fields_ = [("qkv_host", _p), ("qkv_dev", _p), ("o_host", _p), ("o_dev", _p),
                ("gu_host", _p), ("gu_dev", _p), ("down_host", _p), ("down_dev", _p)]


CHAIN_PROJECTIONS = ("q", "k", "v", "o", "gate", "up", "down")


class DecoderChain:
    """The activation buffers and the four sweep tables per layer of a
    decoder-layer chain over M tokens.

    ``layers`` is a list with, per layer, a dict mapping each of
    ``CHAIN_PROJECTIONS`` to ``(packed, wscale)`` from ``ternarize_pack``.
    ``acc_out`` optionally maps (layer, name) to an int32 [M, N] tensor that
    receives that projection's integer results.  The buffers are the
    attributes named as in ``tw_chain_buffers`` plus ``q`` and ``k``; ``h``
    is the input of the first layer and, after a run, the output of the
    last."""

    def __init__(self, layers, M: int, hidden: int, kv_dim: int, head_dim: int, inter: int,
                 device, acc_out=None):
        acc_out = dict(acc_out or {})
        # The tables store addresses only: hold the weights and integer
        # outputs here so that they outlive every run of the chain.
        self.layers = [dict(layer) for layer in layers]
        self.acc_out = acc_out
        f32 = dict(dtype=torch.float32, device=device)
        self.M, self.hidden, self.kv_dim, self.head_dim, self.inter = M, hidden, kv_dim, head_dim, inter
        for name, width in (("h", hidden), ("q", hidden), ("k", kv_dim), ("v", kv_dim),
                            ("a", hidden), ("o", hidden), ("h1", hidden), ("g", inter),
                            ("u", inter), ("act", inter), ("d", hidden)):
            setattr(self, name, torch.zeros((M, width), **f32))
        stages = (("qkv", (("q", self.h, self.q, hidden, hidden), ("k", self.h, self.k, kv_dim, hidden),
                           ("v", self.h, self.v, kv_dim, hidden))),
                  ("o", (("o", self.a, self.o, hidden, hidden),)),
                  ("gu", (("gate", self.h1, self.g, inter, hidden), ("up", self.h1, self.u, inter, hidden))),
                  ("down", (("down", self.act, self.d, hidden, inter),)))
        self.tables = []
        c_layers = (ChainLayer * len(layers))()
        for li, layer in enumerate(layers):
            row = {}
            for stage, projs in stages:
                descs = [dict(x=x, packed=layer[name][0], wscale=layer[name][1], y=y,
                              acc_out=acc_out.get((li, name)), N=N, K=K)
                         for name, x, y, N, K in projs]
                row[stage] = SweepTable(descs, M, device=device, workspace=False)
            self.tables.append(row)
            c_layers[li] = ChainLayer(*[_ptr(t) for st in ("qkv", "o", "gu", "down")
                                        for t in (row[st].host, row[st].device)])
        self.c_layers = c_layers
        self.c_buf = ChainBuffers(_ptr(self.h), _ptr(self.v), _ptr(self.a), _ptr(self.o),
                                  _ptr(self.h1), _ptr(self.g), _ptr(self.u), _ptr(self.act),
                                  _ptr(self.d), M, hidden, kv_dim, head_dim, inter)
        self.n_layers = len(layers)
        self.ws_bytes = int(tw_chain_workspace_bytes(c_layers, self.n_layers))
        self.ws = torch.zeros(max(self.ws_bytes, 16), dtype=torch.uint8, device=device)
        self.launches = int(tw_chain_launches(c_layers, self.n_layers))
        # the fused plan (one persistent launch per 8 tokens)
        pb = int(tw_chain_plan_bytes(self.n_layers))
        self.plan_host = torch.empty(pb, dtype=torch.uint8).pin_memory() \
            if torch.cuda.is_available() else torch.empty(pb, dtype=torch.uint8)
        _raise(tw_chain_plan_encode(c_layers, self.n_layers, ctypes.byref(self.c_buf),
                                    _ptr(self.plan_host), pb))
        self.plan_dev = self.plan_host.to(device) if torch.cuda.is_available() else self.plan_host
        self.fused_ws_bytes = int(tw_chain_fused_workspace_bytes(_ptr(self.plan_host)))
        self.fused_ws = torch.zeros(max(self.fused_ws_bytes, 16), dtype=torch.uint8, device=device)
        self.fused_launches = int(tw_chain_fused_launches(_ptr(self.plan_host)))


def decoder_chain_fused(chain: DecoderChain, stream=None):
    """Run every layer of ``chain`` in the fused persistent kernel."""
    _raise(tw_decoder_chain_fused(_ptr(chain.plan_host), _ptr(chain.plan_dev), _ptr(chain.fused_ws),
                                  chain.fused_ws_bytes, _stream(stream)))


def decoder_chain(chain: DecoderChain, first: int = 0, count=None, stream=None):
    """Run layers first .. first+count-1 of ``chain`` (all by default), one
    sweep per stage and the steps between them as their own launches."""
    count = chain.n_layers - first if count is None else count
    if not (0 <= first and count >= 1 and first + count <= chain.n_layers):
        raise ValueError("layer range outside the chain")
    layers = ctypes.cast(ctypes.addressof(chain.c_layers) + first * ctypes.sizeof(ChainLayer),
                         ctypes.POINTER(ChainLayer))
    _raise(tw_decoder_chain(layers, count, ctypes.byref(chain.c_buf), _ptr(chain.ws),
                            chain.ws_bytes, _stream(stream)))


# ------------------------------------------------------ I8_S linear layer
def i8_quantize_weights(W: torch.Tensor, stream=None):
    """W [N, K] fp32 (CUDA) -> (wq int8 [N, K], amax_w fp32[1])."""
    _need(W, torch.float32, "W")
    N, K = W.shape
    wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    amax = torch.empty(4, dtype=torch.float32, device=W.device)
    _raise(tw_i8_quantize_weights(_ptr(W), N, K, _ptr(wq), _ptr(amax), _stream(stream)))
    return wq, amax[:1]


def i8_linear_q(xq, amax_x, wq, amax_w, bias=None, relu: bool = True, y=None, acc_out=None,
                stream=None):
    """y [M, N] fp32 from xq [M, K] int8 + amax_x [M] and wq [N, K] + amax_w."""
    _need(xq, torch.int8, "xq")
    _need(wq, torch.int8, "wq")
    M, K = xq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=xq.device)
    _raise(tw_i8_linear_q(_ptr(xq), _ptr(amax_x), M, N, K, _ptr(wq), _ptr(amax_w), _ptr(bias),
                          int(bool(relu)), _ptr(y), _ptr(acc_out), _stream(stream)))
    return y


def i8_linear(x, wq, amax_w, bias=None, relu: bool = True, y=None, acc_out=None, ws=None,
              stream=None):
    """y [M, N] fp32 = relu?(I8_S layer) from fp32 x [M, K]."""
    _need(x, torch.float32, "x")
    _need(wq, torch.int8, "wq")
    M, K = x.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    wsb = int(tw_i8_workspace_bytes(M, K))
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=x.device)
    _raise(tw_i8_linear(_ptr(x), M, N, K, _ptr(wq), _ptr(amax_w), _ptr(bias), int(bool(relu)),
                        _ptr(y), _ptr(acc_out), _ptr(ws), ws.numel(), _stream(stream)))
    return y


# ------------------------------------------------ tensor-parallel pieces
def pack_slice(packed: torch.Tensor, N: int, K: int, n0: int, rows: int, k0: int, cols: int,
               stream=None):
    """Packed codes of rows [n0, n0+rows) x columns [k0, k0+cols) of a packed [N, K]."""
    _need(packed, torch.uint8, "packed")
    out = torch.empty(max(packed_bytes(rows, cols), 16), dtype=torch.uint8, device=packed.device)
    _raise(tw_pack_slice(_ptr(packed), N, K, n0, rows, k0, cols, _ptr(out), out.numel(),
                         _stream(stream)))
    return out


def row_absmax(x: torch.Tensor, stream=None):
    """amax [M] = max |x| per row of x [M, K] fp32."""
    _need(x, torch.float32, "x")
    M, K = x.shape
    amax = torch.empty(M, dtype=torch.float32, device=x.device)
    _raise(tw_row_absmax(_ptr(x), M, K, _ptr(amax), _stream(stream)))
    return amax


def quantize_act_given(x: torch.Tensor, amax: torch.Tensor, stream=None):
    """(xq int8 [M, K], qsum int32 [M]) of x with the given per-token amax."""
    _need(x, torch.float32, "x")
    _need(amax, torch.float32, "amax")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    qsum = torch.empty(M, dtype=torch.int32, device=x.device)
    _raise(tw_quantize_act_given(_ptr(x), M, K, _ptr(amax), _ptr(xq), _ptr(qsum), _stream(stream)))
    return xq, qsum


def rescale_acc(acc: torch.Tensor, amax: torch.Tensor, wscale: torch.Tensor, y=None, stream=None):
    """y [M, N] fp32 from summed accumulators acc [M, N] int32."""
    _need(acc, torch.int32, "acc")
    M, N = acc.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=acc.device)
    _raise(tw_rescale_acc(_ptr(acc), M, N, _ptr(amax), _ptr(wscale), _ptr(y), _stream(stream)))
    return y
