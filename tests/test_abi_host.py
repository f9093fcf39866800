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
                ("total_units", "<i8"), ("total_ptiles", "<i8"), ("max_K", "<i8"),
                ("total_cost", "<i8"), ("ws_bytes", "<i8")])


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
