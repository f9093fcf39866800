"""Parity at the workload's full sizes, in the launch configuration bench.py
times: the 196-projection decode sweep (M = 1 and M = 4, 8, 16, 32) and the
196-projection prefill sweep (M = 256, 1024, 4096), checked on sampled
outputs against the oracle.

Every projection is ternarised on the GPU and its mean|W| and scale checked
bit-exact against the oracle over the whole matrix; then for a seeded sample
of weight rows (and, for prefill, of token rows) the oracle recomputes the
codes, activations and accumulators one by one: accumulators bit-exact,
outputs within 1e-6 relative.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu

ROWS_PER_PROJ = 8


@pytest.fixture(scope="module")
def model():
    """All 196 projections ternarised on the GPU, with oracle references for
    a seeded sample of rows of each."""
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
        toks = np.sort(rng.choice(M, size=6, replace=False))
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
