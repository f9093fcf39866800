"""Parity of the I8_S linear layer (int8 weights and activations, bias and
ReLU fused) with the oracle, through the C ABI.

Weights quantised on the GPU (wq, amax_w) and int32 accumulators must be
bit-exact.  The fp32 outputs are compared with the oracle's fp64 value
within 1e-6 of |acc * amax_x/127 * amax_w/127| + |bias| (the GPU rounds
four products and one sum in fp32, < 5 * 2^-24 of those magnitudes; the
bound is taken on the magnitudes because a bias may cancel the product).
Every output is poisoned before the call.
"""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-6


@pytest.fixture(scope="module")
def dev():
    return G.torch_dev()


@pytest.fixture(scope="module")
def api():
    return G.api()


def _w(N, K, seed):
    return synth.weights(seed, 41, N, K, 0.05)


def _x(M, K, seed):
    return synth.activations(seed, 43, M, K, outliers=True)


def _bias(N, seed):
    return (np.random.default_rng(seed).standard_normal(N) * 2.0).astype(np.float32)


def check_y(y_gpu, ref, amax_w, bias, ctx):
    prod = ref["acc"].astype(np.float64) * (ref["amax"].astype(np.float64)[:, None] / 127.0) * \
        (float(amax_w) / 127.0)
    mag = np.abs(prod) + (0.0 if bias is None else np.abs(bias.astype(np.float64))[None, :])
    err = np.abs(np.asarray(y_gpu, np.float64) - ref["y"])
    bad = ~(err <= TOL * mag)
    assert not bad.any(), f"{ctx}: {int(bad.sum())} outputs off, worst {float(err[bad].max()):.3e}"


@pytest.mark.parametrize("N,K", [(1024, 256), (37, 48), (300, 1040), (1, 16), (2048, 512)])
def test_i8_weight_quant_bit_exact(dev, api, N, K):
    W = _w(N, K, N + K)
    wq, amax = api.i8_quantize_weights(G.to_dev(W, dev))
    api.check()
    want_q, want_a = orc.i8_quantize_weights(W)
    assert float(amax.cpu()[0]) == float(want_a)
    assert (wq.cpu().numpy() == want_q).all()


def test_i8_weight_quant_zero_and_nonfinite(dev, api):
    wq, amax = api.i8_quantize_weights(G.to_dev(np.zeros((8, 32), np.float32), dev))
    api.check()
    assert float(amax.cpu()[0]) == 0.0 and not wq.cpu().numpy().any()
    W = _w(8, 32, 1)
    W[2, 5] = np.nan
    api.i8_quantize_weights(G.to_dev(W, dev))
    with pytest.raises(api.TernaryError) as e:
        api.check()
    assert e.value.status == 5


def _run(api, dev, M, N, K, seed, relu=True, with_bias=True):
    import torch
    W = _w(N, K, seed)
    x = _x(M, K, seed + 1)
    bias = _bias(N, seed + 2) if with_bias else None
    wq, amax_w = api.i8_quantize_weights(G.to_dev(W, dev))
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    acc = torch.full((M, N), -2**31, dtype=torch.int32, device=dev)
    api.i8_linear(G.to_dev(x, dev), wq, amax_w, None if bias is None else G.to_dev(bias, dev),
                  relu=relu, y=y, acc_out=acc)
    api.check()
    want_q, want_a = orc.i8_quantize_weights(W)
    ref = orc.i8_linear(x, want_q, want_a, bias, relu=relu)
    return y.cpu().numpy(), acc.cpu().numpy(), ref, want_a, bias


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (128, 128, 128), (129, 257, 272), (300, 1024, 256),
                                   (64, 4096, 1024), (1000, 384, 528), (33, 6, 1040),
                                   (200, 130, 128), (257, 1, 32)])
def test_i8_linear_shapes(dev, api, M, N, K):
    """Several tiles and ragged M, N and K tails; N not a multiple of 4 (6,
    130, 1) takes the row-store epilogue."""
    y, acc, ref, aw, bias = _run(api, dev, M, N, K, 7 * M + N + K)
    assert (acc == ref["acc"]).all(), f"{(acc != ref['acc']).sum()} accumulators off"
    check_y(y, ref, aw, bias, f"{M}x{N}x{K}")


@pytest.mark.parametrize("relu,with_bias", [(False, True), (True, False), (False, False)])
def test_i8_linear_modes(dev, api, relu, with_bias):
    M, N, K = 150, 200, 384
    y, acc, ref, aw, bias = _run(api, dev, M, N, K, 99, relu=relu, with_bias=with_bias)
    assert (acc == ref["acc"]).all()
    check_y(y, ref, aw, bias, f"relu={relu} bias={with_bias}")
    if relu:
        assert (y >= 0).all()
    else:
        assert (y < 0).any()


def test_i8_zero_weights_give_relu_bias(dev, api):
    import torch
    M, N, K = 40, 64, 128
    bias = _bias(N, 5)
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    amax_w = torch.full((4,), 0.5, dtype=torch.float32, device=dev)[:1]
    y = api.i8_linear(G.to_dev(_x(M, K, 6), dev), wq, amax_w, G.to_dev(bias, dev), relu=True)
    api.check()
    assert (y.cpu().numpy() == np.maximum(bias, 0)[None, :]).all()


def test_i8_linear_q_matches_and_k_permutation(dev, api):
    """The pre-quantised entry gives the same bytes; a joint permutation of
    K leaves the accumulators unchanged."""
    import torch
    M, N, K = 96, 160, 256
    W, x = _w(N, K, 11), _x(M, K, 12)
    Wd, xd = G.to_dev(W, dev), G.to_dev(x, dev)
    wq, aw = api.i8_quantize_weights(Wd)
    acc1 = torch.empty((M, N), dtype=torch.int32, device=dev)
    y1 = api.i8_linear(xd, wq, aw, None, relu=False, acc_out=acc1)
    xq, amax, _ = api.quantize_act(xd)
    acc2 = torch.empty((M, N), dtype=torch.int32, device=dev)
    y2 = api.i8_linear_q(xq, amax, wq, aw, None, relu=False, acc_out=acc2)
    perm = torch.as_tensor(np.random.default_rng(0).permutation(K), device=dev)
    acc3 = torch.empty((M, N), dtype=torch.int32, device=dev)
    api.i8_linear(xd[:, perm].contiguous(), wq[:, perm].contiguous(), aw, None, relu=False,
                  acc_out=acc3)
    api.check()
    assert torch.equal(y1, y2) and torch.equal(acc1, acc2) and torch.equal(acc1, acc3)


def test_i8_encoder_shape_full(dev, api):
    """The synthetic encoder shape at full size (16384 tokens, 256 -> 1024
    channels: activations 16 : 1 over weights), every output checked."""
    M, N, K = 16384, 1024, 256
    y, acc, ref, aw, bias = _run(api, dev, M, N, K, 2024)
    assert (acc == ref["acc"]).all()
    check_y(y, ref, aw, bias, "16384x1024x256")


def test_i8_argument_errors(dev, api):
    import torch
    wq = torch.zeros((16, 24), dtype=torch.int8, device=dev)   # K = 24 is not a multiple of 16
    aw = torch.ones(4, device=dev)[:1]
    with pytest.raises(api.TernaryError) as e:
        api.i8_linear(torch.zeros((4, 24), device=dev), wq, aw)
    assert e.value.status == 2
    wq = torch.zeros((16, 32), dtype=torch.int8, device=dev)
    flat = torch.zeros(4 * 32 + 1, device=dev)
    with pytest.raises(api.TernaryError) as e:
        api.i8_linear(flat[1:].view(4, 32), wq, aw)
    assert e.value.status == 3
