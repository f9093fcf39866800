"""CPU-side checks of the C ABI: the library builds, loads and exports every
symbol ``include/ternary_decoder.h`` declares; the host-only entry points
(size queries, sweep-table encoding) behave as documented.  No kernel runs."""
import ctypes
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT
from tests import layout_spec

HEADER = os.path.join(ROOT, "include", "ternary_decoder.h")


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_decoder_b200 import build
    return ctypes.CDLL(build.build())


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TW_API\s+[\w\s\*]+?\b(tw_\w+)\s*\(", text)))


def test_header_declares_the_path():
    syms = declared_symbols()
    for name in ("tw_ternarize_pack", "tw_quantize_act", "tw_ternary_linear",
                 "tw_decoder_projection_sweep", "tw_unpack_codes", "tw_check"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_size_queries(lib):
    from ternary_weight_decoder_b200 import api
    assert api.packed_bytes(1536, 1536) == 589_824
    assert api.packed_bytes(256, 1536) == 98_304
    assert api.packed_bytes(8960, 1536) == 3_440_640
    assert api.packed_bytes(1536, 8960) == 3_440_640
    assert api.packed_bytes(17, 128) == 32 * 128 // 4   # padded to 2 row blocks
    assert api.packed_bytes(0, 128) == 0
    assert api.tw_ternarize_workspace_bytes(1536, 1536) % 256 == 0
    assert api.tw_ternarize_workspace_bytes(1536, 1536) >= 256 + 8 * 1536
    assert api.linear_workspace_bytes(32, 1536, 1536) == 32 * 1536 + 256
    assert api.linear_workspace_bytes(1, 8960, 8960) == 8960 + 256
    assert api.linear_workspace_bytes(256, 1536, 1536) >= 256 * 1536 + 2 * 256 * 4


def _descs(shapes, base=0x10000):
    from ternary_weight_decoder_b200 import api
    arr = (api.ProjDesc * len(shapes))()
    for i, (N, K) in enumerate(shapes):
        a = base + i * 0x100000
        arr[i] = api.ProjDesc(x=a, xq=None, amax=None, qsum=None, packed=a + 0x1000,
                              wscale=a + 0x2000, y=a + 0x3000, acc_out=None, N=N, K=K)
    return arr


REC = np.dtype([("x", "<u8"), ("xq", "<u8"), ("amax", "<u8"), ("qsum", "<u8"),
                ("packed", "<u8"), ("wscale", "<u8"), ("y", "<u8"), ("acc_out", "<u8"),
                ("N", "<i8"), ("K", "<i8"), ("rb_begin", "<i8"), ("tile_begin", "<i8"),
                ("ptile_begin", "<i8"), ("ws_xq_off", "<i8"), ("cost_begin", "<i8"),
                ("tmap_ok", "<i8"),
                ("tmap", "u1", 128), ("tmap_codes", "u1", 128)])
HDR = np.dtype([("magic", "<u4"), ("count", "<i4"), ("M", "<i8"), ("total_rb", "<i8"),
                ("total_units", "<i8"), ("total_ptiles", "<i8"), ("max_K", "<i4"),
                ("gemm", "<i4"), ("total_cost", "<i8"), ("ws_bytes", "<i8")])


def test_table_encode_prefix_sums(lib):
    from ternary_weight_decoder_b200 import api
    shapes = [(1536, 1536), (256, 1536), (17, 256), (1536, 8960)]
    arr = _descs(shapes)
    n = api.tw_sweep_table_bytes(len(shapes))
    assert n == 64 + (384 + 16) * len(shapes)   # header, records, unit order
    buf = np.zeros(n, np.uint8)
    rc = api.tw_sweep_table_encode(arr, len(shapes), 1, buf.ctypes.data, n)
    assert rc == 0, api.tw_last_error()
    hdr = buf[:64].view(HDR)[0]
    recs = buf[64:64 + 384 * len(shapes)].view(REC)
    order = buf[64 + 384 * len(shapes):].view(np.dtype([("d", "<i4"), ("units", "<i4"),
                                                          ("unit_begin", "<i8")]))
    assert hdr["magic"] == 0x54574431 and hdr["count"] == 4 and hdr["M"] == 1
    nrb = [-(-N // 16) for N, K in shapes]
    ntiles = [r * (K // 128) for r, (N, K) in zip(nrb, shapes)]
    assert recs["rb_begin"].tolist() == np.concatenate([[0], np.cumsum(nrb)[:-1]]).tolist()
    assert recs["tile_begin"].tolist() == np.concatenate([[0], np.cumsum(ntiles)[:-1]]).tolist()
    assert hdr["total_rb"] == sum(nrb)
    # tensor-core units: 128 rows each, projections of larger K first (stable)
    assert order["d"].tolist() == [3, 0, 1, 2]
    units = [-(-shapes[d][0] // 128) for d in order["d"]]
    assert order["units"].tolist() == units
    assert order["unit_begin"].tolist() == np.concatenate([[0], np.cumsum(units)[:-1]]).tolist()
    assert hdr["total_units"] == sum(units)
    assert hdr["max_K"] == 8960
    # static split by cost: 16 units per 128-column tile + 45 per row block
    cost = [r * (16 * (K // 128) + 45) for r, (N, K) in zip(nrb, shapes)]
    assert recs["cost_begin"].tolist() == np.concatenate([[0], np.cumsum(cost)[:-1]]).tolist()
    assert hdr["total_cost"] == sum(cost)
    assert recs["N"].tolist() == [s[0] for s in shapes]
    # scratch: 256 bytes of counters, then per projection room for 8 token
    # rows (the tensor-core blocks of M <= 8), then the scales
    xq = [8 * K for N, K in shapes]
    head = 256
    assert recs["ws_xq_off"].tolist() == (head + np.concatenate([[0], np.cumsum(xq)[:-1]])).tolist()
    assert hdr["ws_bytes"] == head + sum(xq) + 256 * len(shapes)
    assert api.tw_sweep_workspace_bytes(buf.ctypes.data) == hdr["ws_bytes"]
    assert api.tw_sweep_launches(buf.ctypes.data) == 2   # quantise + decode


@pytest.mark.parametrize("bad,status", [
    ({"K": 100}, 2), ({"K": 0}, 2), ({"N": 0}, 2), ({"packed": None}, 1),
    ({"y": None}, 1), ({"x": None}, 1), ({"x": 0x10008}, 3), ({"K": 70000}, 2)])
def test_table_encode_rejects(lib, bad, status):
    from ternary_weight_decoder_b200 import api
    arr = _descs([(64, 256), (32, 128)])
    for k, v in bad.items():
        setattr(arr[1], k, v)
    n = api.tw_sweep_table_bytes(2)
    buf = np.zeros(n, np.uint8)
    assert api.tw_sweep_table_encode(arr, 2, 4, buf.ctypes.data, n) == status
    assert api.tw_last_error()


def test_table_encode_gemm_choice(lib):
    """The GEMM choice: only TW_SWEEP_GEMM_AUTO (0) and _EXPANDED (1) are
    accepted, before any descriptor is read; a decode table ignores it and
    encodes the same bytes as tw_sweep_table_encode."""
    from ternary_weight_decoder_b200 import api
    shapes = [(1536, 1536), (17, 256)]
    arr = _descs(shapes)
    n = api.tw_sweep_table_bytes(len(shapes))
    for bad in (-1, 2, 7):
        buf = np.zeros(n, np.uint8)
        assert api.tw_sweep_table_encode_gemm(arr, 2, 1, bad, buf.ctypes.data, n) == 2
        assert b"gemm" in api.tw_last_error()
        assert not buf.any()
    ref = np.zeros(n, np.uint8)
    assert api.tw_sweep_table_encode(arr, 2, 4, ref.ctypes.data, n) == 0
    for gemm in (0, 1):
        buf = np.zeros(n, np.uint8)
        assert api.tw_sweep_table_encode_gemm(arr, 2, 4, gemm, buf.ctypes.data, n) == 0
        assert (buf == ref).all()
        assert buf[:64].view(HDR)[0]["gemm"] == 0
    assert api.SWEEP_GEMM == {"auto": 0, "expanded": 1}


def test_table_encode_rejects_small_buffer_and_count(lib):
    from ternary_weight_decoder_b200 import api
    arr = _descs([(64, 256)])
    buf = np.zeros(1024, np.uint8)
    assert api.tw_sweep_table_encode(arr, 1, 1, buf.ctypes.data, 100) == 4
    assert api.tw_sweep_table_encode(arr, 0, 1, buf.ctypes.data, 1024) == 2
    assert api.tw_sweep_table_encode(arr, 1, 0, buf.ctypes.data, 1024) == 2


def test_layout_spec_round_trip():
    rng = np.random.default_rng(0)
    for N, K in [(16, 128), (37, 256), (5, 384)]:
        c = rng.integers(-1, 2, (N, K)).astype(np.int8)
        p = layout_spec.pack(c)
        assert p.size == -(-N // 16) * 16 * K // 4
        assert (layout_spec.unpack(p, N, K) == c).all()
        # every 32-bit word holds 16 consecutive k of one row
        w = p.view(np.uint32).astype(np.int64)
        dec = [int((w[0] >> (8 * b + 2 * s)) & 3) - 1 for s in range(4) for b in range(4)]
        assert dec == c[0, :16].tolist()


def test_layout_spec_fast_pack_matches_the_statement():
    """pack_fast (used at full size) writes the same bytes as pack."""
    rng = np.random.default_rng(1)
    for N, K in [(16, 128), (37, 256), (5, 384), (1, 128), (48, 1152)]:
        c = rng.integers(-1, 2, (N, K)).astype(np.int8)
        assert (layout_spec.pack_fast(c) == layout_spec.pack(c)).all(), (N, K)


QWEN_LAYER = [(1536, 1536), (256, 1536), (256, 1536), (1536, 1536),
              (8960, 1536), (8960, 1536), (1536, 8960)]


@pytest.mark.parametrize("M", list(range(1, 33)))
def test_sweep_launch_count_196(lib, M):
    """Launches per step of the 196-projection sweep, as the host plans them
    for 148 SMs: one or two quantisation launches (two once a row gets at
    most 2 warps: the 28 K = 8960 rows split off), then one decode launch.
    Up to 16 tokens that is one register-kernel launch (every token group
    fits: 15 consumer warps with 2 KB chunks beside 16 rows of K = 8960),
    above that the tensor-core kernel."""
    from ternary_weight_decoder_b200 import api
    shapes = QWEN_LAYER * 28
    arr = _descs(shapes)
    n = api.tw_sweep_table_bytes(len(shapes))
    buf = np.zeros(n, np.uint8)
    assert api.tw_sweep_table_encode(arr, len(shapes), M, buf.ctypes.data, n) == 0, \
        api.tw_last_error()
    # warps per row: the largest of 8, 4, 2, 1 with 196*M*w <= 148*24, i.e.
    # 8 for M <= 2, 4 for M = 3..4, 2 or 1 from M = 5 on
    quant = 1 if M <= 4 else 2
    assert api.tw_sweep_launches(buf.ctypes.data) == quant + 1


# ------------------------------------------------------ decoder-layer chain
CHAIN_BUFS = ("h", "v", "a", "o", "h1", "g", "u", "act", "d")


CHAIN_ADDR = {n: 0x7f0000000000 + 0x100000 * i for i, n in enumerate(CHAIN_BUFS + ("q", "k"))}


def _fake_chain(M=1, hidden=256, kv=128, hd=128, inter=512, n_layers=2, tweak=None):
    """Encoded tables of a chain over placeholder device addresses (nothing
    is launched): per layer qkv, o, gate/up and down, as the chain wants
    them unless `tweak(layer, stage, descs)` changes the descriptors."""
    from ternary_weight_decoder_b200 import api
    addr = CHAIN_ADDR
    stages = {"qkv": [("h", "q", hidden, hidden), ("h", "k", kv, hidden), ("h", "v", kv, hidden)],
              "o": [("a", "o", hidden, hidden)],
              "gu": [("h1", "g", inter, hidden), ("h1", "u", inter, hidden)],
              "down": [("act", "d", hidden, inter)]}
    keep, layers = [], (api.ChainLayer * n_layers)()
    for li in range(n_layers):
        ptrs = []
        for st in ("qkv", "o", "gu", "down"):
            descs = stages[st]
            arr = (api.ProjDesc * len(descs))()
            for i, (x, y, N, K) in enumerate(descs):
                w = 0x7d0000000000 + 0x1000000 * (8 * li + i)
                arr[i] = api.ProjDesc(x=addr[x], xq=None, amax=None, qsum=None, packed=w,
                                      wscale=w + 0x800000, y=addr[y], acc_out=None, N=N, K=K)
            if tweak:
                tweak(li, st, arr)
            n = api.tw_sweep_table_bytes(len(descs))
            buf = np.zeros(n, np.uint8)
            assert api.tw_sweep_table_encode(arr, len(descs), M, buf.ctypes.data, n) == 0, \
                api.tw_last_error()
            keep.append(buf)
            ptrs += [buf.ctypes.data, 0x7e0000000000 + 0x10000 * len(keep)]
        layers[li] = api.ChainLayer(*ptrs)
    cbuf = api.ChainBuffers(*[addr[n] for n in CHAIN_BUFS], M, hidden, kv, hd, inter)
    return layers, cbuf, keep


def test_chain_launch_count_and_workspace(lib):
    """Per layer four sweeps of one quantisation and one decode launch each
    (at M = 1) and four element-wise launches; the workspace is the largest
    table's."""
    from ternary_weight_decoder_b200 import api
    layers, cbuf, keep = _fake_chain(n_layers=3)
    assert api.tw_chain_launches(layers, 3) == 3 * (4 * 2 + 4)
    per_table = [api.tw_sweep_workspace_bytes(b.ctypes.data) for b in keep]
    assert api.tw_chain_workspace_bytes(layers, 3) == max(per_table)
    assert api.tw_chain_launches(layers, 0) == 0
    assert api.tw_chain_workspace_bytes(None, 1) == 0


def test_chain_checks_every_table_before_launching(lib):
    """A well-formed chain passes every host check and stops only at the
    missing workspace (nothing launched)."""
    from ternary_weight_decoder_b200 import api
    import ctypes
    layers, cbuf, keep = _fake_chain()
    assert api.tw_decoder_chain(layers, 2, ctypes.byref(cbuf), None, 0, None) == 4
    assert b"workspace" in api.tw_last_error()


def _tw(arr, i, **kw):
    for k, v in kw.items():
        setattr(arr[i], k, v)


@pytest.mark.parametrize("case,status", [
    ("o_reads_wrong_buffer", 2), ("v_writes_wrong_buffer", 2), ("down_wrong_K", 2),
    ("gate_wrong_N", 2), ("qkv_two_projections", 2), ("table_other_M", 2),
    ("q_writes_into_h", 2), ("k_writes_into_a", 2), ("acc_out_in_h1", 2),
    ("acc_out_in_act", 2)])
def test_chain_rejects_mismatched_tables(lib, case, status):
    from ternary_weight_decoder_b200 import api
    import ctypes
    M = 1
    tweaks = {
        "o_reads_wrong_buffer": lambda l, st, a: st == "o" and l == 1 and _tw(a, 0, x=a[0].x + 0x100000),
        "v_writes_wrong_buffer": lambda l, st, a: st == "qkv" and _tw(a, 2, y=a[2].y + 0x100000),
        "down_wrong_K": lambda l, st, a: st == "down" and _tw(a, 0, K=256),
        "gate_wrong_N": lambda l, st, a: st == "gu" and _tw(a, 0, N=384),
        # q's output inside h: the sweep would overwrite h while k and v read it
        "q_writes_into_h": lambda l, st, a: st == "qkv" and _tw(a, 0, y=CHAIN_ADDR["h"] + 256),
        "k_writes_into_a": lambda l, st, a: st == "qkv" and _tw(a, 1, y=CHAIN_ADDR["a"]),
        "acc_out_in_h1": lambda l, st, a: st == "o" and _tw(a, 0, acc_out=CHAIN_ADDR["h1"]),
        "acc_out_in_act": lambda l, st, a: st == "gu" and l == 1 and _tw(a, 1, acc_out=CHAIN_ADDR["act"] + 512),
    }
    if case in tweaks:
        layers, cbuf, keep = _fake_chain(tweak=tweaks[case])
    elif case == "qkv_two_projections":
        layers, cbuf, keep = _fake_chain()
        other, _, keep2 = _fake_chain(tweak=None)
        keep += keep2
        # a two-projection table (gate/up of another chain) where qkv belongs
        layers[0].qkv_host, layers[0].qkv_dev = other[0].gu_host, other[0].gu_dev
    else:
        layers, cbuf, keep = _fake_chain(M=2)
        cbuf.M = M
    assert api.tw_decoder_chain(layers, 2, ctypes.byref(cbuf), 0x7c0000000000, 1 << 30, None) == status
    assert api.tw_last_error()


@pytest.mark.parametrize("field,value,status", [
    ("h", None, 1), ("act", 0x7f0000000008, 3), ("M", 33, 2), ("M", 0, 2),
    ("hidden", 200, 2), ("head_dim", 96, 2), ("kv_dim", 384, 2),
    ("h1", CHAIN_ADDR["h"] + 512, 2), ("d", CHAIN_ADDR["act"], 2)])
def test_chain_rejects_bad_buffers(lib, field, value, status):
    from ternary_weight_decoder_b200 import api
    import ctypes
    layers, cbuf, keep = _fake_chain()
    setattr(cbuf, field, value)
    assert api.tw_decoder_chain(layers, 2, ctypes.byref(cbuf), 0x7c0000000000, 1 << 30, None) == status
    assert api.tw_last_error()


def test_chain_binding_owns_the_tensors_it_points_at(lib):
    """The tables hold raw addresses; the binding must keep the weights and
    integer outputs alive after the caller drops them (a freed weight scale
    reused by a later allocation would silently change the outputs)."""
    import gc
    import weakref
    import torch
    from ternary_weight_decoder_b200 import api
    hidden, kv, hd, inter = 256, 128, 128, 512
    shapes = {"q": (hidden, hidden), "k": (kv, hidden), "v": (kv, hidden), "o": (hidden, hidden),
              "gate": (inter, hidden), "up": (inter, hidden), "down": (hidden, inter)}
    layers = [{n: (torch.zeros(api.packed_bytes(N, K), dtype=torch.uint8), torch.ones(4))
               for n, (N, K) in shapes.items()} for _ in range(2)]
    acc = {(1, "k"): torch.zeros((1, kv), dtype=torch.int32)}
    refs = [weakref.ref(t) for layer in layers for pair in layer.values() for t in pair]
    refs.append(weakref.ref(acc[(1, "k")]))
    chain = api.DecoderChain(layers, 1, hidden, kv, hd, inter, torch.device("cpu"), acc_out=acc)
    del layers, acc
    gc.collect()
    assert all(r() is not None for r in refs)
    assert chain.launches == 2 * (4 * 2 + 4)
    # the binding's tables pass every host check of the chain; with no
    # workspace the call stops there, before any launch
    import ctypes
    assert api.tw_decoder_chain(chain.c_layers, 2, ctypes.byref(chain.c_buf), None, 0, None) == 4
    assert b"workspace" in api.tw_last_error()
    # a sweep table alone owns its descriptors' tensors too
    x = torch.zeros((1, 128))
    t = api.SweepTable([dict(x=x, packed=torch.zeros(api.packed_bytes(16, 128), dtype=torch.uint8),
                             wscale=torch.ones(4), y=torch.zeros((1, 16)), N=16, K=128)], 1)
    r = weakref.ref(x)
    del x
    gc.collect()
    assert r() is not None and t.count == 1


def test_chain_fused_plan_host_checks(lib):
    """The fused chain's plan passes the same table checks, sizes its
    scratch from the widest stage and launches once per 8 tokens."""
    from ternary_weight_decoder_b200 import api
    import ctypes
    for M, launches in ((1, 1), (8, 1), (9, 2), (20, 3)):
        layers, cbuf, keep = _fake_chain(M=M, n_layers=2)
        nb = api.tw_chain_plan_bytes(2)
        assert nb >= 4 * 2 * 256
        plan = np.zeros(nb, np.uint8)
        assert api.tw_chain_plan_encode(layers, 2, ctypes.byref(cbuf), plan.ctypes.data, nb) == 0, \
            api.tw_last_error()
        assert api.tw_chain_fused_launches(plan.ctypes.data) == launches
        # counters + three sum buffers of 8 rows of the widest stage (gate/up: 2 x 512)
        assert api.tw_chain_fused_workspace_bytes(plan.ctypes.data) == 256 + 4 * 8 * 1024 * 4
        assert api.tw_chain_plan_encode(layers, 2, ctypes.byref(cbuf), plan.ctypes.data, nb - 1) == 4
    # a table that does not match the buffers is refused here too
    layers, cbuf, keep = _fake_chain(tweak=lambda l, st, a: st == "o" and _tw(a, 0, x=a[0].x + 0x100000))
    plan = np.zeros(api.tw_chain_plan_bytes(2), np.uint8)
    assert api.tw_chain_plan_encode(layers, 2, ctypes.byref(cbuf), plan.ctypes.data, plan.size) == 2
    # a plan that was not encoded is refused before any launch
    assert api.tw_decoder_chain_fused(np.zeros(512, np.uint8).ctypes.data, 0x7e0000000000,
                                      0x7c0000000000, 1 << 20, None) == 8
    assert api.tw_chain_fused_workspace_bytes(np.zeros(512, np.uint8).ctypes.data) == 0
