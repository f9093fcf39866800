"""Python access to the C reference oracle (``ternary_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``; never by the product package.
This module only marshals numpy arrays into the C functions; every step of
the arithmetic lives in ``ternary_oracle.c``.  ``decoder_layer`` composes
them in the order of a decoder layer, rounding each projection output to
float32 as the chain passes it on.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ternary_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O1", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fexcess-precision=standard", "-shared", "-fPIC"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library next to its source."""
    if force or not os.path.exists(_LIB) or (
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.orc_mean_abs.restype = ctypes.c_double
    lib.orc_mean_abs.argtypes = [p, i64, i64]
    lib.orc_ternarize.restype = ctypes.c_int
    lib.orc_ternarize.argtypes = [p, i64, i64, p, p]
    lib.orc_quantize_act.restype = None
    lib.orc_quantize_act.argtypes = [p, i64, i64, p, p]
    lib.orc_ternary_acc.restype = ctypes.c_int
    lib.orc_ternary_acc.argtypes = [p, i64, i64, p, i64, p]
    lib.orc_rescale.restype = None
    lib.orc_rescale.argtypes = [p, i64, i64, p, ctypes.c_double, p]
    lib.orc_gqa_expand.restype = None
    lib.orc_gqa_expand.argtypes = [p, i64, i64, i64, i64, p]
    lib.orc_add_f32.restype = None
    lib.orc_add_f32.argtypes = [p, p, i64, p]
    lib.orc_silu_mul.restype = None
    lib.orc_silu_mul.argtypes = [p, p, i64, p]
    lib.orc_i8_quantize_weights.restype = None
    lib.orc_i8_quantize_weights.argtypes = [p, i64, i64, p, p]
    lib.orc_i8_epilogue.restype = None
    lib.orc_i8_epilogue.argtypes = [p, i64, i64, p, ctypes.c_float, p, ctypes.c_int, p]
    lib.orc_quantize_act_given.restype = None
    lib.orc_quantize_act_given.argtypes = [p, i64, i64, p, p]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def use_library(path):
    """Point this module at another build of the oracle source (the pin
    tests use it to run the pins against deliberately broken copies).
    Returns the previously bound library; pass it back to restore."""
    global _lib
    prev = _load()
    _lib = path if isinstance(path, ctypes.CDLL) else _bind(ctypes.CDLL(path))
    return prev


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile a (modified) copy of the oracle source with the same flags."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *_CFLAGS, "-o", out_path, c_path, "-lm"], check=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def mean_abs(W) -> float:
    W, pw = _c(W, np.float32)
    N, K = W.shape
    return float(_load().orc_mean_abs(pw, N, K))


def ternarize(W):
    """Return (codes int8 [N,K], mean float).  Raises on non-finite W."""
    W, pw = _c(W, np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    mean = ctypes.c_double()
    rc = _load().orc_ternarize(pw, N, K, ctypes.addressof(mean),
                               codes.ctypes.data)
    if rc != 0:
        raise ValueError("non-finite value in W")
    return codes, mean.value


def quantize_act(x):
    """Return (q int8 [M,K], amax float32 [M])."""
    x, px = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    amax = np.empty(M, np.float32)
    _load().orc_quantize_act(px, M, K, q.ctypes.data, amax.ctypes.data)
    return q, amax


def ternary_acc(codes, q):
    """Return acc int32 [M,N] = q @ codes.T (raises on int32 overflow)."""
    codes, pc = _c(codes, np.int8)
    q, pq = _c(q, np.int8)
    N, K = codes.shape
    M, K2 = q.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    if _load().orc_ternary_acc(pc, N, K, pq, M, acc.ctypes.data) != 0:
        raise OverflowError("accumulator does not fit int32")
    return acc


def rescale(acc, amax, mean: float):
    """Return y float64 [M,N] = acc * (amax/127) * mean."""
    acc, pa = _c(acc, np.int32)
    amax, pm = _c(amax, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float64)
    _load().orc_rescale(pa, M, N, pm, float(mean), y.ctypes.data)
    return y


def ternary_linear(x, codes, mean: float):
    """Whole layer on ternary codes: returns dict(q, amax, acc, y)."""
    q, amax = quantize_act(x)
    acc = ternary_acc(codes, q)
    y = rescale(acc, amax, mean)
    return {"q": q, "amax": amax, "acc": acc, "y": y}


# ------------------------------------------------ decoder-layer chain (R13-R16)
def gqa_expand(v, hidden: int, head_dim: int):
    """Identity attention (R13): a [M, hidden] float32 from v [M, kv_dim]."""
    v, pv = _c(v, np.float32)
    M, kv_dim = v.shape
    assert hidden % head_dim == 0 and kv_dim % head_dim == 0
    assert (hidden // head_dim) % (kv_dim // head_dim) == 0
    a = np.empty((M, hidden), np.float32)
    _load().orc_gqa_expand(pv, M, kv_dim, hidden, head_dim, a.ctypes.data)
    return a


def add_f32(x, y):
    """Residual add (R15): float32 x + y, elementwise."""
    x, px = _c(x, np.float32)
    y, py = _c(y, np.float32)
    assert x.shape == y.shape
    out = np.empty(x.shape, np.float32)
    _load().orc_add_f32(px, py, x.size, out.ctypes.data)
    return out


def silu_mul(g, u):
    """SiLU(g) * u in float64 (R16)."""
    g, pg = _c(g, np.float32)
    u, pu = _c(u, np.float32)
    assert g.shape == u.shape
    out = np.empty(g.shape, np.float64)
    _load().orc_silu_mul(pg, pu, g.size, out.ctypes.data)
    return out


def decoder_layer(h, layer, head_dim: int = 128):
    """One layer of the chain in the oracle's own precision, from float32 h
    [M, hidden] and ``layer`` = dict(q, k, v, o, gate, up, down), each a
    (codes, mean) pair.  Every projection output is rounded to float32
    before it is used (the chain passes float32 activations).  Returns a
    dict of every intermediate; ``h_next`` is the layer's output."""
    def proj(x, name):
        codes, mean = layer[name]
        return ternary_linear(x, codes, mean)["y"].astype(np.float32)
    hidden = h.shape[1]
    q, k, v = proj(h, "q"), proj(h, "k"), proj(h, "v")
    a = gqa_expand(v, hidden, head_dim)
    o = proj(a, "o")
    h1 = add_f32(h, o)
    g, u = proj(h1, "gate"), proj(h1, "up")
    act = silu_mul(g, u).astype(np.float32)
    d = proj(act, "down")
    return {"q": q, "k": k, "v": v, "a": a, "o": o, "h1": h1, "g": g, "u": u,
            "act": act, "d": d, "h_next": add_f32(h1, d)}


# ------------------------------------------------ I8_S linear (R17-R19)
def i8_quantize_weights(W):
    """R17: (wq int8 [N,K], amax_w float32) -- one absmax scale per tensor."""
    W, pw = _c(W, np.float32)
    N, K = W.shape
    wq = np.empty((N, K), np.int8)
    amax = np.empty(1, np.float32)
    _load().orc_i8_quantize_weights(pw, N, K, wq.ctypes.data, amax.ctypes.data)
    return wq, np.float32(amax[0])


def i8_epilogue(acc, amax_x, amax_w, bias=None, relu=True):
    """R19: y float64 [M,N] = relu?(acc * amax_x/127 * amax_w/127 + bias)."""
    acc, pa = _c(acc, np.int32)
    amax_x, px = _c(amax_x, np.float32)
    M, N = acc.shape
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
        assert bias.shape == (N,)
    y = np.empty((M, N), np.float64)
    _load().orc_i8_epilogue(pa, M, N, px, float(amax_w), pb, int(bool(relu)), y.ctypes.data)
    return y


def i8_linear(x, wq, amax_w, bias=None, relu=True):
    """The I8_S layer on quantised weights: quantise x per token (R18),
    int8 dot products (exact), rescale + bias + ReLU.  dict(q, amax, acc, y)."""
    q, amax = quantize_act(x)
    acc = ternary_acc(wq, q)       # an exact int8 dot product for any int8 weights
    y = i8_epilogue(acc, amax, amax_w, bias, relu)
    return {"q": q, "amax": amax, "acc": acc, "y": y}


# ------------------------------------------------ tensor-parallel split (R20)
def quantize_act_given(x, amax):
    """R20: q int8 [M,K] of x [M,K] with the given per-token amax [M]."""
    x, px = _c(x, np.float32)
    amax, pa = _c(amax, np.float32)
    M, K = x.shape
    assert amax.shape == (M,)
    q = np.empty((M, K), np.int8)
    _load().orc_quantize_act_given(px, M, K, pa, q.ctypes.data)
    return q
