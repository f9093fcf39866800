"""Parity of the CUDA path (through the C ABI) with the reference oracle.

Codes, packed bytes, int8 activations, amax, sum(q) and int32 accumulators
must be bit-exact; fp32 outputs within 1e-6 relative of the fp64 oracle.
Sizes span several tiles plus ragged tails; every output buffer is poisoned
before the call so an unwritten element shows up (the NaN fingerprint of a
missing remainder-row path, "The Paper Says ARM Support" post, round three).
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from tests.conftest import ROOT
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu

POISON_I32 = np.int32(-2**31)


@pytest.fixture(scope="module")
def dev():
    return G.torch_dev()


@pytest.fixture(scope="module")
def api():
    return G.api()


def _weights(N, K, seed, sigma=0.02):
    return synth.weights(seed, 17, N, K, sigma)


def _acts(M, K, seed, outliers=True):
    return synth.activations(seed, 23, M, K, outliers)


# ------------------------------------------------------------ ternarise
@pytest.mark.parametrize("N,K", [(16, 128), (37, 256), (256, 1536), (1536, 1536),
                                 (100, 8960), (1, 128)])
def test_ternarize_pack_bit_exact(dev, api, N, K):
    W = _weights(N, K, N + K)
    packed, mean_abs, wscale = G.ternarize_gpu(W, dev)
    codes, _ = G.check_packed_against_oracle(W, packed, mean_abs, wscale, N, K)
    got, invalid = api.unpack_codes(packed, N, K)
    api.check()
    assert (got.cpu().numpy() == codes).all()
    assert int(invalid.cpu()[0]) == 0


def test_ternarize_hand_case(dev, api, golden_dir):
    g = json.load(open(os.path.join(golden_dir, "hand_4x8.json")))
    W = np.tile(np.array(g["W"], np.float32), (1, 16))          # K = 128, mean unchanged
    packed, mean_abs, wscale = G.ternarize_gpu(W, dev)
    assert float(mean_abs.cpu()[0]) == g["mean_abs"]
    codes, _ = api.unpack_codes(packed, 4, 128)
    assert (codes.cpu().numpy() == np.tile(np.array(g["codes"], np.int8), (1, 16))).all()
    x = np.tile(np.array(g["x"], np.float32), (1, 16))
    acc = G.to_dev(np.full((1, 4), POISON_I32), dev)
    y = api.ternary_linear(G.to_dev(x, dev), packed, wscale, 4, acc_out=acc)
    api.check()
    assert acc.cpu().numpy().tolist() == [[16 * v for v in g["acc"][0]]]
    assert y.cpu().numpy().tolist() == [[16.0 * v for v in g["y"][0]]]


def test_ternarize_zero_weights(dev, api):
    W = np.zeros((20, 256), np.float32)
    packed, mean_abs, wscale = G.ternarize_gpu(W, dev)
    assert float(mean_abs.cpu()[0]) == 1e-5
    codes, _ = api.unpack_codes(packed, 20, 256)
    assert not codes.cpu().numpy().any()
    y = api.ternary_linear(G.to_dev(_acts(3, 256, 1), dev), packed, wscale, 20)
    api.check()
    assert not y.cpu().numpy().any()


def test_ternarize_nonfinite_reported(dev, api):
    W = _weights(16, 128, 5)
    W[3, 7] = np.inf
    api.ternarize_pack(G.to_dev(W, dev))
    with pytest.raises(api.TernaryError) as e:
        api.check()
    assert e.value.status == 5
    api.check()  # the error word was cleared


# ------------------------------------------------------------ act quant
@pytest.mark.parametrize("M,K", [(1, 1536), (5, 8960), (33, 128), (300, 256)])
def test_quantize_act_bit_exact(dev, api, M, K):
    x = _acts(M, K, M * 7 + K)
    x[min(2, M - 1)] = 0.0  # an all-zero token
    xq, amax, qsum = api.quantize_act(G.to_dev(x, dev))
    api.check()
    q, a = orc.quantize_act(x)
    assert (xq.cpu().numpy() == q).all()
    assert (amax.cpu().numpy() == a).all()
    assert (qsum.cpu().numpy() == q.astype(np.int64).sum(axis=1)).all()


# ------------------------------------------------------------ decode linear
def _run_linear(api, dev, W, x, N):
    import torch
    packed, mean_abs, wscale = G.ternarize_gpu(W, dev)
    M = x.shape[0]
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
    api.ternary_linear(G.to_dev(x, dev), packed, wscale, N, y=y, acc_out=acc)
    api.check()
    return y.cpu().numpy(), acc.cpu().numpy()


@pytest.mark.parametrize("M", list(range(1, 34)))
def test_linear_m_tails(dev, api, M):
    """M = 1..32 run the decode kernel, M = 33 the tensor-core prefill."""
    N, K = 80, 640   # 5 row blocks, 5 k tiles (one partial ring chunk)
    W = _weights(N, K, 100 + M)
    x = _acts(M, K, 200 + M)
    y, acc = _run_linear(api, dev, W, x, N)
    codes, mean = orc.ternarize(W)
    ref = orc.ternary_linear(x, codes, mean)
    assert (acc == ref["acc"]).all()
    G.assert_y_close(y, ref["y"], f"M={M}")


@pytest.mark.parametrize("M,N,K", [(1, 1536, 1536), (1, 256, 1536), (1, 1536, 8960),
                                   (4, 8960, 1536), (8, 37, 1152), (16, 1536, 8960),
                                   (32, 1536, 8960), (32, 300, 1536), (3, 1, 128)])
def test_decode_linear_shapes(dev, api, M, N, K):
    W = _weights(N, K, M + N + K)
    x = _acts(M, K, M * 3 + K)
    y, acc = _run_linear(api, dev, W, x, N)
    codes, mean = orc.ternarize(W)
    ref = orc.ternary_linear(x, codes, mean)
    assert (acc == ref["acc"]).all()
    G.assert_y_close(y, ref["y"], f"{M}x{N}x{K}")


def test_decode_zero_token_row(dev, api):
    N, K = 64, 256
    W = _weights(N, K, 9)
    x = _acts(3, K, 9)
    x[1] = 0.0
    y, acc = _run_linear(api, dev, W, x, N)
    assert not acc[1].any() and not y[1].any()


def test_decode_k_permutation_detector(dev, api):
    """A joint permutation of K leaves acc unchanged; swapping the two
    64-halves of every 128-block of W alone changes it (a 64-vs-128 block
    mis-read, "The Paper Says ARM Support" post, postscript two)."""
    N, K, M = 48, 512, 4
    W = _weights(N, K, 31)
    x = _acts(M, K, 32)
    _, acc = _run_linear(api, dev, W, x, N)
    perm = np.random.default_rng(0).permutation(K)
    _, acc_p = _run_linear(api, dev, np.ascontiguousarray(W[:, perm]),
                           np.ascontiguousarray(x[:, perm]), N)
    assert (acc_p == acc).all()
    blk = np.arange(K).reshape(-1, 2, 64)[:, ::-1, :].ravel()
    _, acc_s = _run_linear(api, dev, np.ascontiguousarray(W[:, blk]), x, N)
    assert (acc_s != acc).any()


# ------------------------------------------------------------ prefill linear
@pytest.mark.parametrize("M,N,K", [(33, 80, 640), (128, 256, 128), (129, 257, 256),
                                   (255, 1536, 1536), (256, 1536, 1536), (257, 300, 1152),
                                   (1024, 256, 1536), (300, 8960, 1536), (64, 1536, 8960),
                                   (40, 1, 128), (200, 30, 384), (1023, 1536, 1536),
                                   (4095, 300, 1536)])
def test_prefill_linear_shapes(dev, api, M, N, K):
    W = _weights(N, K, 7 * M + N + K)
    x = _acts(M, K, 11 * M + K)
    y, acc = _run_linear(api, dev, W, x, N)
    codes, mean = orc.ternarize(W)
    ref = orc.ternary_linear(x, codes, mean)
    assert (acc == ref["acc"]).all(), f"{M}x{N}x{K}: {(acc != ref['acc']).sum()} accumulators off"
    G.assert_y_close(y, ref["y"], f"{M}x{N}x{K}")


def test_prefill_linear_q_and_zero_rows(dev, api):
    """Pre-quantised entry point; an all-zero token row gives zeros."""
    import torch
    M, N, K = 150, 512, 1024
    W = _weights(N, K, 77)
    x = _acts(M, K, 78)
    x[5] = 0.0
    packed, _, wscale = G.ternarize_gpu(W, dev)
    xq, amax, qsum = api.quantize_act(G.to_dev(x, dev))
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
    api.ternary_linear_q(xq, amax, qsum, packed, wscale, N, y=y, acc_out=acc)
    api.check()
    codes, mean = orc.ternarize(W)
    ref = orc.ternary_linear(x, codes, mean)
    assert (acc.cpu().numpy() == ref["acc"]).all()
    G.assert_y_close(y.cpu().numpy(), ref["y"])
    assert not y.cpu().numpy()[5].any()


# ------------------------------------------------------------ sweep
def _sweep_case(api, dev, layers, M, seed_base=0):
    import torch
    descs, keep, refs = [], [], []
    for (l, p, name, N, K) in synth.sweep_shapes(layers):
        W = synth.weights(l + seed_base, p, N, K)
        x = synth.activations(l + seed_base, p, M, K)
        packed, mean_abs, wscale = G.ternarize_gpu(W, dev)
        xd = G.to_dev(x, dev)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        d = dict(x=xd, packed=packed, wscale=wscale, y=y, acc_out=acc, N=N, K=K)
        if M > 32:   # prefill sweeps take pre-quantised activations
            d["xq"], d["amax"], d["qsum"] = api.quantize_act(xd)
        descs.append(d)
        keep.append((W, x))
    table = api.SweepTable(descs, M, device=dev)
    api.decoder_projection_sweep(table)
    api.check()
    return descs, keep


@pytest.mark.parametrize("M", [1, 4, 8, 16, 32, 33, 256])
def test_sweep_one_layer(dev, api, M):
    descs, keep = _sweep_case(api, dev, 1, M, seed_base=M)
    for d, (W, x) in zip(descs, keep):
        codes, mean = orc.ternarize(W)
        ref = orc.ternary_linear(x, codes, mean)
        assert (d["acc_out"].cpu().numpy() == ref["acc"]).all(), (M, d["N"], d["K"])
        G.assert_y_close(d["y"].cpu().numpy(), ref["y"], f"M={M} N={d['N']} K={d['K']}")


def test_sweep_two_layers_m1(dev, api):
    descs, keep = _sweep_case(api, dev, 2, 1, seed_base=50)
    for d, (W, x) in zip(descs, keep):
        codes, mean = orc.ternarize(W)
        ref = orc.ternary_linear(x, codes, mean)
        assert (d["acc_out"].cpu().numpy() == ref["acc"]).all()
        G.assert_y_close(d["y"].cpu().numpy(), ref["y"])


def test_sweep_ragged_small_projections(dev, api):
    """Many tiny projections (fewer row blocks than CTAs, ragged N)."""
    import torch
    M = 3
    rng = np.random.default_rng(5)
    shapes = [(int(rng.integers(1, 70)), 128 * int(rng.integers(1, 6))) for _ in range(40)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 1000 + i)
        x = _acts(M, K, 2000 + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        descs.append(dict(x=G.to_dev(x, dev), packed=packed, wscale=wscale, y=y, acc_out=acc,
                          N=N, K=K))
        keep.append((W, x))
    table = api.SweepTable(descs, M, device=dev)
    api.decoder_projection_sweep(table)
    api.check()
    for d, (W, x) in zip(descs, keep):
        codes, mean = orc.ternarize(W)
        ref = orc.ternary_linear(x, codes, mean)
        assert (d["acc_out"].cpu().numpy() == ref["acc"]).all()
        G.assert_y_close(d["y"].cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M", [1, 3, 5, 8, 13, 16])
def test_sweep_chunk_tails(dev, api, M):
    """K = 128 .. 1792 (1 to 14 k tiles) in one sweep: every length of the
    last ring chunk of a row block (1..6 tiles for 7-tile chunks up to 4
    tokens, 1..5 for 6-tile chunks above) and whole chunks, with ragged N."""
    import torch
    shapes = [(16 * kt + 8 * (kt % 3) + kt % 5, 128 * kt) for kt in range(1, 15)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 3000 + 50 * M + i)
        x = _acts(M, K, 4000 + 50 * M + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        descs.append(dict(x=G.to_dev(x, dev), packed=packed, wscale=wscale, y=y, acc_out=acc,
                          N=N, K=K))
        keep.append((W, x))
    table = api.SweepTable(descs, M, device=dev)
    api.decoder_projection_sweep(table)
    api.check()
    for (N, K), d, (W, x) in zip(shapes, descs, keep):
        codes, mean = orc.ternarize(W)
        ref = orc.ternary_linear(x, codes, mean)
        assert (d["acc_out"].cpu().numpy() == ref["acc"]).all(), f"M={M} N={N} K={K}"
        G.assert_y_close(d["y"].cpu().numpy(), ref["y"], f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [9, 12, 16, 17, 20, 24, 31, 32])
def test_sweep_tensor_core_decode_ragged(dev, api, M):
    """The tensor-core decode kernel (9..32 tokens): every token-block width
    (16 with four slot accumulators, 32 with one),
    projections whose N is not a multiple of 128 (the last 128-row unit
    partial, row blocks past N read as zero), several K, and the unit order
    (larger K first) different from the record order."""
    import torch
    shapes = [(200, 256), (128, 1536), (17, 384), (385, 640), (256, 2048), (1, 128)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 3000 + 10 * M + i)
        x = _acts(M, K, 4000 + 10 * M + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        descs.append(dict(x=G.to_dev(x, dev), packed=packed, wscale=wscale, y=y, acc_out=acc,
                          N=N, K=K))
        keep.append((W, x))
    table = api.SweepTable(descs, M, device=dev)
    for _ in range(2):   # twice: the work counters are left zero for the next call
        api.decoder_projection_sweep(table)
        api.check()
        for d, (W, x) in zip(descs, keep):
            codes, mean = orc.ternarize(W)
            ref = orc.ternary_linear(x, codes, mean)
            assert (d["acc_out"].cpu().numpy() == ref["acc"]).all(), (M, d["N"], d["K"])
            G.assert_y_close(d["y"].cpu().numpy(), ref["y"])
        for d in descs:
            d["y"].fill_(float("nan"))
            d["acc_out"].fill_(int(POISON_I32))


@pytest.mark.parametrize("M", [33, 200, 300])
def test_sweep_more_tokens_from_fp32_x(dev, api, M):
    """Sweeps of more than 32 tokens given fp32 x (weights-in-tensor-memory
    kernel at 33 and 200 tokens, expanded-weights kernel at 300): the sweep
    quantises x into each descriptor's xq, amax and qsum (bit-exact against
    the oracle's R2-R4) before the product; a descriptor given xq without x
    in the same table is used as given (and left as it was)."""
    import torch
    shapes = [(200, 256), (128, 1536), (17, 384), (385, 640), (256, 2048), (1, 128)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 7000 + 10 * M + i)
        x = _acts(M, K, 7500 + 10 * M + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        from_x = i % 3 != 2
        if from_x:
            xq = torch.full((M, K), -77, dtype=torch.int8, device=dev)
            amax = torch.full((M,), float("nan"), dtype=torch.float32, device=dev)
            qsum = torch.full((M,), int(POISON_I32), dtype=torch.int32, device=dev)
            xd = G.to_dev(x, dev)
        else:
            xq, amax, qsum = api.quantize_act(G.to_dev(x, dev))
            xd = None
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        d = dict(xq=xq, amax=amax, qsum=qsum, packed=packed, wscale=wscale, y=y, acc_out=acc,
                 N=N, K=K)
        if xd is not None:
            d["x"] = xd
        descs.append(d)
        keep.append((W, x, from_x))
    table = api.SweepTable(descs, M, device=dev)
    assert table.launches == 2
    for _ in range(2):
        api.decoder_projection_sweep(table)
        api.check()
        for d, (W, x, from_x) in zip(descs, keep):
            q_ref, amax_ref = orc.quantize_act(x)
            assert np.array_equal(d["xq"].cpu().numpy(), q_ref), (M, d["N"], d["K"], from_x)
            assert np.array_equal(d["amax"].cpu().numpy(), amax_ref), (M, d["K"], from_x)
            assert np.array_equal(d["qsum"].cpu().numpy(),
                                  q_ref.astype(np.int64).sum(axis=1).astype(np.int32))
            codes, mean = orc.ternarize(W)
            ref = orc.ternary_linear(x, codes, mean)
            assert (d["acc_out"].cpu().numpy() == ref["acc"]).all(), (M, d["N"], d["K"])
            G.assert_y_close(d["y"].cpu().numpy(), ref["y"], f"M={M} N={d['N']} K={d['K']}")
        for d, (_, _, from_x) in zip(descs, keep):
            d["y"].fill_(float("nan"))
            d["acc_out"].fill_(int(POISON_I32))
            if from_x:
                d["xq"].fill_(-77)


# ------------------------------------------------------------ errors
def test_wait_timeout_is_reported(dev, api):
    api.debug_wait_timeout(2_000_000)   # 2 ms; nothing ever arrives
    with pytest.raises(api.TernaryError) as e:
        api.check()
    assert e.value.status == 7
    api.check()


def test_argument_errors(dev, api):
    import torch
    x = torch.zeros((2, 128), dtype=torch.float32, device=dev)
    packed, _, wscale = G.ternarize_gpu(_weights(16, 128, 1), dev)
    with pytest.raises(api.TernaryError) as e:
        api.ternary_linear(torch.zeros((2, 100), dtype=torch.float32, device=dev), packed,
                           wscale, 16)
    assert e.value.status == 2
    flat = torch.zeros(2 * 128 + 1, dtype=torch.float32, device=dev)
    with pytest.raises(api.TernaryError) as e:
        api.ternary_linear(flat[1:].view(2, 128), packed, wscale, 16)
    assert e.value.status == 3
    y = api.ternary_linear(x, packed, wscale, 16)
    api.check()
    assert not y.cpu().numpy().any()


@pytest.mark.parametrize("M", [33, 64, 65, 96, 97, 127, 128, 129, 191, 192, 193, 255, 300])
def test_sweep_mid_m(dev, api, M):
    """More than 32 tokens (the weights-in-tensor-memory kernel up to 192,
    with units of 64, 96, 128 or 192 tokens by M and both sides of each
    width switch; the expanded-weights kernel from 193): every token-tile
    tail, projections whose N is not a multiple of 128 (the last 128-row
    unit partial), several K, twice in a row (the unit counters are left
    zero for the next call)."""
    import torch
    shapes = [(200, 256), (128, 1536), (17, 384), (385, 640), (256, 2048), (1, 128)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 5000 + 10 * M + i)
        x = _acts(M, K, 6000 + 10 * M + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        xq, amax, qsum = api.quantize_act(G.to_dev(x, dev))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        acc = torch.full((M, N), int(POISON_I32), dtype=torch.int32, device=dev)
        descs.append(dict(xq=xq, amax=amax, qsum=qsum, packed=packed, wscale=wscale, y=y,
                          acc_out=acc, N=N, K=K))
        keep.append((W, x))
    table = api.SweepTable(descs, M, device=dev)
    for _ in range(2):
        api.decoder_projection_sweep(table)
        api.check()
        for d, (W, x) in zip(descs, keep):
            codes, mean = orc.ternarize(W)
            ref = orc.ternary_linear(x, codes, mean)
            assert (d["acc_out"].cpu().numpy() == ref["acc"]).all(), (M, d["N"], d["K"])
            G.assert_y_close(d["y"].cpu().numpy(), ref["y"], f"M={M} N={d['N']} K={d['K']}")
        for d in descs:
            d["y"].fill_(float("nan"))
            d["acc_out"].fill_(int(POISON_I32))


@pytest.mark.parametrize("M", [33, 100, 192])
def test_sweep_gemm_choice(dev, api, M):
    """A table encoded for the expanded-weights GEMM (TW_SWEEP_GEMM_EXPANDED)
    at token counts where the default runs the weights-in-TMEM GEMM: the
    oracle's sums and outputs, and the same bytes as the default table."""
    import torch
    shapes = [(200, 256), (128, 1536), (17, 384), (385, 640)]
    descs, keep = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(N, K, 7100 + 10 * M + i)
        x = _acts(M, K, 7200 + 10 * M + i)
        packed, _, wscale = G.ternarize_gpu(W, dev)
        xq, amax, qsum = api.quantize_act(G.to_dev(x, dev))
        descs.append(dict(xq=xq, amax=amax, qsum=qsum, packed=packed, wscale=wscale, N=N, K=K))
        keep.append((W, x))
    outs = {}
    for gemm in ("expanded", "auto"):
        ds = [dict(d, y=torch.full((M, d["N"]), float("nan"), dtype=torch.float32, device=dev),
                   acc_out=torch.full((M, d["N"]), int(POISON_I32), dtype=torch.int32,
                                      device=dev)) for d in descs]
        table = api.SweepTable(ds, M, device=dev, gemm=gemm)
        api.decoder_projection_sweep(table)
        api.check()
        outs[gemm] = [(d["y"].cpu().numpy(), d["acc_out"].cpu().numpy()) for d in ds]
    for (ye, ae), (ya, aa), (W, x), (N, K) in zip(outs["expanded"], outs["auto"], keep, shapes):
        codes, mean = orc.ternarize(W)
        ref = orc.ternary_linear(x, codes, mean)
        assert (ae == ref["acc"]).all(), (M, N, K)
        G.assert_y_close(ye, ref["y"], f"expanded M={M} N={N} K={K}")
        assert (ae == aa).all() and (ye.view(np.uint32) == ya.view(np.uint32)).all(), (M, N, K)
