"""Parity at the workload's full sizes, in the launch configuration bench.py
times: the 196-projection decode sweep (M = 1 and M = 4, 8, 16, 32) and the
196-projection prefill sweep (M = 256, 1024, 4096), checked on sampled
outputs against the oracle.

Every projection is ternarised on the GPU; its packed bytes (the whole
matrix, all 196 of them), mean|W| and scale are compared bit for bit with
the oracle's codes laid out by the layout statement in tests/layout_spec.py.
Then for a seeded sample of 64 weight rows per projection (and, for prefill,
16 token rows including the first and last 128-token tile) the oracle
recomputes the activations and accumulators one by one: accumulators
bit-exact, outputs within 1e-6 relative.  Every output of every projection
is poisoned before the call and checked to have been written.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from tests import layout_spec
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu

ROWS_PER_PROJ = 64
TOKENS_PER_PREFILL = 16


@pytest.fixture(scope="module")
def model():
    """All 196 projections ternarised on the GPU, each compared whole with
    the oracle (packed bytes, mean, scale), with oracle codes kept for a
    seeded sample of rows of each."""
    dev = G.torch_dev()
    api = G.api()
    shapes = synth.sweep_shapes()
    rng = np.random.default_rng(20261202)
    pool = cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4))
    futs = {}
    projs = []
    for i, (l, p, name, N, K) in enumerate(shapes):
        for j in range(i, min(i + 12, len(shapes))):
            if j not in futs:
                lj, pj, _, Nj, Kj = shapes[j]
                futs[j] = pool.submit(synth.weights, lj, pj, Nj, Kj)
        W = futs.pop(i).result()
        packed, mean_abs, wscale = api.ternarize_pack(G.to_dev(W, dev))
        codes, mean = orc.ternarize(W)
        want = layout_spec.pack_fast(codes)
        got = packed.cpu().numpy()
        assert got.size >= want.size and (got[:want.size] == want).all(), \
            f"packed codes of L{l}.{name} ({N}x{K}) differ from the oracle's"
        del want, got
        rows = np.sort(rng.choice(N, size=min(ROWS_PER_PROJ, N), replace=False))
        projs.append(dict(l=l, p=p, name=name, N=N, K=K, packed=packed, mean_abs=mean_abs,
                          wscale=wscale, mean=mean, rows=rows, codes=codes[rows].copy()))
    api.check()
    pool.shutdown()
    for d in projs:
        assert float(d["mean_abs"].cpu()[0]) == d["mean"], (d["l"], d["name"])
        assert float(d["wscale"].cpu()[0]) == np.float32(d["mean"])
    return dev, api, projs


def _check_rows(d, x_rows, y_rows, acc_rows, tag):
    """Oracle on the sampled weight rows for the given token rows."""
    ref = orc.ternary_linear(x_rows, d["codes"], d["mean"])
    assert (acc_rows == ref["acc"]).all(), f"{tag}: accumulators differ"
    G.assert_y_close(y_rows, ref["y"], tag)


@pytest.mark.parametrize("M", [1, 4, 8, 16, 32])
def test_decode_sweep_full_size(model, M):
    import torch
    dev, api, projs = model
    descs = []
    for d in projs:
        x = synth.activations(d["l"], d["p"], M, d["K"])
        descs.append(dict(x=G.to_dev(x, dev), packed=d["packed"], wscale=d["wscale"],
                          y=torch.full((M, d["N"]), float("nan"), device=dev),
                          acc_out=torch.full((M, d["N"]), -2**31, dtype=torch.int32,
                                             device=dev),
                          N=d["N"], K=d["K"], xh=x))
    table = api.SweepTable(descs, M, device=dev)
    api.decoder_projection_sweep(table)
    api.check()
    for d, s in zip(projs, descs):
        y = s["y"].cpu().numpy()
        assert np.isfinite(y).all(), f"unwritten outputs in L{d['l']}.{d['name']}"
        _check_rows(d, s["xh"], y[:, d["rows"]], s["acc_out"].cpu().numpy()[:, d["rows"]],
                    f"M={M} L{d['l']}.{d['name']}")


@pytest.mark.parametrize("M", [256, 1024, 4096])
def test_prefill_sweep_full_size(model, M):
    import torch
    dev, api, projs = model
    rng = np.random.default_rng(M)
    descs, keep = [], []
    for d in projs:
        x = synth.activations(d["l"], d["p"], M, d["K"])
        xd = G.to_dev(x, dev)
        xq, amax, qsum = api.quantize_act(xd)
        del xd
        # the first and last token of the first and last 128-token tile, the
        # rest seeded
        fixed = {0, 1, M - 1, M - 2, (M - 1) // 128 * 128}
        rest = [t for t in rng.permutation(M) if t not in fixed]
        toks = np.sort(np.array(sorted(fixed) + rest[:TOKENS_PER_PREFILL - len(fixed)]))
        keep.append((toks, x[toks].copy()))
        descs.append(dict(xq=xq, amax=amax, qsum=qsum, packed=d["packed"],
                          wscale=d["wscale"],
                          y=torch.full((M, d["N"]), float("nan"), device=dev),
                          acc_out=torch.full((M, d["N"]), -2**31, dtype=torch.int32,
                                             device=dev),
                          N=d["N"], K=d["K"]))
        del x
    table = api.SweepTable(descs, M, device=dev)
    api.decoder_projection_sweep(table)
    api.check()
    for d, s, (toks, xr) in zip(projs, descs, keep):
        y = s["y"]
        assert not torch.isnan(y).any().item(), f"unwritten outputs in L{d['l']}.{d['name']}"
        rows = torch.as_tensor(d["rows"], device=dev)
        tk = torch.as_tensor(toks, device=dev)
        ys = y[tk][:, rows].cpu().numpy()
        accs = s["acc_out"][tk][:, rows].cpu().numpy()
        _check_rows(d, xr, ys, accs, f"M={M} L{d['l']}.{d['name']}")
