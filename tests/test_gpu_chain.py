"""Parity of the decoder-layer chain (through the C ABI) with the oracle.

Each layer runs on its own; every stage is then checked against the oracle
on the GPU's own input of that stage, since later stages quantise values
that an fp64 oracle would round differently: the projections' int32
accumulators bit-exact and their fp32 outputs within 1e-6 relative, the
identity attention and the two single-precision residual adds bit-exact,
SiLU(gate) * up within 1e-6 relative (expf is within 2 ulp).  A run of all
layers in one call must then reproduce the layer-by-layer results exactly.
Intermediate buffers are poisoned before every call.
"""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu

POISON_I32 = np.int32(-2**31)
ACT_RTOL = 1e-6
PROJ = ("q", "k", "v", "o", "gate", "up", "down")


@pytest.fixture(scope="module")
def dev():
    return G.torch_dev()


@pytest.fixture(scope="module")
def api():
    return G.api()


def _shapes(hidden, kv, inter):
    return {"q": (hidden, hidden), "k": (kv, hidden), "v": (kv, hidden), "o": (hidden, hidden),
            "gate": (inter, hidden), "up": (inter, hidden), "down": (hidden, inter)}


def _build(api, dev, M, dims, n_layers, seed):
    import torch
    hidden, kv, hd, inter = dims
    shapes = _shapes(hidden, kv, inter)
    gpu_layers, orc_layers, acc = [], [], {}
    for li in range(n_layers):
        g, o = {}, {}
        for pi, name in enumerate(PROJ):
            N, K = shapes[name]
            W = synth.weights(seed + li, 40 + pi, N, K)
            packed, _, wscale = G.ternarize_gpu(W, dev)
            g[name] = (packed, wscale)
            o[name] = orc.ternarize(W)
            acc[(li, name)] = torch.empty((M, N), dtype=torch.int32, device=dev)
        gpu_layers.append(g)
        orc_layers.append(o)
    chain = api.DecoderChain(gpu_layers, M, hidden, kv, hd, inter, dev, acc_out=acc)
    return chain, orc_layers, acc


def _poison(chain, acc):
    for name in ("q", "k", "v", "a", "o", "h1", "g", "u", "act", "d"):
        getattr(chain, name).fill_(float("nan"))
    for t in acc.values():
        t.fill_(int(POISON_I32))


def _np(t):
    return t.cpu().numpy()


def _check_proj(x_in, codes_mean, y_gpu, acc_gpu, ctx):
    codes, mean = codes_mean
    ref = orc.ternary_linear(x_in, codes, mean)
    assert (acc_gpu == ref["acc"]).all(), f"{ctx}: accumulators differ"
    G.assert_y_close(y_gpu, ref["y"], ctx)


def _check_layer(chain, orc_layer, acc, li, h_in):
    hidden, hd = chain.hidden, chain.head_dim
    got = {n: _np(getattr(chain, n)) for n in ("q", "k", "v", "a", "o", "h1", "g", "u", "act",
                                                "d", "h")}
    a_cc = {n: _np(acc[(li, n)]) for n in PROJ}
    for n in ("q", "k", "v"):
        _check_proj(h_in, orc_layer[n], got[n], a_cc[n], f"layer {li} {n}")
    assert np.array_equal(got["a"], orc.gqa_expand(got["v"], hidden, hd)), f"layer {li} attention"
    _check_proj(got["a"], orc_layer["o"], got["o"], a_cc["o"], f"layer {li} o")
    assert np.array_equal(got["h1"], orc.add_f32(h_in, got["o"])), f"layer {li} h + o"
    _check_proj(got["h1"], orc_layer["gate"], got["g"], a_cc["gate"], f"layer {li} gate")
    _check_proj(got["h1"], orc_layer["up"], got["u"], a_cc["up"], f"layer {li} up")
    ref = orc.silu_mul(got["g"], got["u"])
    err = np.abs(got["act"].astype(np.float64) - ref)
    assert np.isfinite(got["act"]).all() and (err <= ACT_RTOL * np.abs(ref) + 1e-30).all(), \
        f"layer {li} SiLU * up: worst {float(err.max()):.3e}"
    _check_proj(got["act"], orc_layer["down"], got["d"], a_cc["down"], f"layer {li} down")
    assert np.array_equal(got["h"], orc.add_f32(got["h1"], got["d"])), f"layer {li} h1 + d"
    return got["h"]


SMALL = (256, 128, 128, 512)          # 2 query heads over 1 KV head
SMALL_G1 = (256, 256, 128, 384)       # one query head per KV head
QWEN = (1536, 256, 128, 8960)         # 12 query heads over 2 KV heads


@pytest.mark.parametrize("M,dims", [(1, SMALL), (5, SMALL), (16, SMALL), (3, SMALL_G1),
                                    (1, QWEN), (20, QWEN)])
def test_chain_stagewise(dev, api, M, dims):
    n_layers = 2
    chain, orc_layers, acc = _build(api, dev, M, dims, n_layers, seed=300 + M)
    h0 = synth.activations(310 + M, 0, M, dims[0])
    chain.h.copy_(G.to_dev(h0, dev))
    h_in = h0
    for li in range(n_layers):
        _poison(chain, acc)
        api.decoder_chain(chain, first=li, count=1)
        api.check()
        h_in = _check_layer(chain, orc_layers[li], acc, li, h_in)
    # all layers in one call: the same bytes as layer by layer
    chain.h.copy_(G.to_dev(h0, dev))
    _poison(chain, acc)
    api.decoder_chain(chain)
    api.check()
    assert np.array_equal(_np(chain.h), h_in)


def test_chain_zero_weights_return_input(dev, api):
    """All projections zero: the chain returns its input unchanged (the
    residual adds add +0), on the GPU as in the oracle's closed form."""
    import torch
    hidden, kv, hd, inter = SMALL
    shapes = _shapes(hidden, kv, inter)
    layers = []
    for _ in range(3):
        layer = {}
        for name in PROJ:
            N, K = shapes[name]
            packed, _, wscale = G.ternarize_gpu(np.zeros((N, K), np.float32), dev)
            layer[name] = (packed, wscale)
        layers.append(layer)
    chain = api.DecoderChain(layers, 4, hidden, kv, hd, inter, dev)
    h0 = synth.activations(7, 0, 4, hidden)
    chain.h.copy_(G.to_dev(h0, dev))
    api.decoder_chain(chain)
    api.check()
    assert np.array_equal(_np(chain.h), h0)
    assert not torch.any(chain.act) and not torch.any(chain.d)


def _snapshot(chain, acc):
    names = ("h", "q", "k", "v", "a", "o", "h1", "g", "u", "act", "d")
    return ({n: getattr(chain, n).clone() for n in names},
            {k: t.clone() for k, t in acc.items()})


@pytest.mark.parametrize("M,dims", [(1, SMALL), (5, SMALL), (16, SMALL), (3, SMALL_G1),
                                    (1, QWEN), (9, QWEN), (20, QWEN)])
def test_chain_fused_matches_unfused(dev, api, M, dims):
    """The fused persistent chain gives the bytes of the unfused chain (which
    the stagewise test pins to the oracle): every buffer and every
    projection's integer outputs of the last layer, twice in a row (the
    barrier counters and sum buffers are reset by each call)."""
    import torch
    n_layers = 3
    chain, _, acc = _build(api, dev, M, dims, n_layers, seed=500 + M)
    h0 = G.to_dev(synth.activations(510 + M, 0, M, dims[0]), dev)
    chain.h.copy_(h0)
    _poison(chain, acc)
    api.decoder_chain(chain)
    api.check()
    want, want_acc = _snapshot(chain, acc)
    for _ in range(2):
        chain.h.copy_(h0)
        _poison(chain, acc)
        api.decoder_chain_fused(chain)
        api.check()
        got, got_acc = _snapshot(chain, acc)
        for n in want:
            assert torch.equal(got[n], want[n]), f"fused chain M={M}: buffer {n} differs"
        for k in want_acc:
            if k[0] == n_layers - 1:
                assert torch.equal(got_acc[k], want_acc[k]), f"fused chain M={M}: acc {k} differs"


def test_chain_fused_zero_weights_return_input(dev, api):
    hidden, kv, hd, inter = SMALL
    shapes = _shapes(hidden, kv, inter)
    layers = []
    for _ in range(2):
        layer = {}
        for name in PROJ:
            N, K = shapes[name]
            packed, _, wscale = G.ternarize_gpu(np.zeros((N, K), np.float32), dev)
            layer[name] = (packed, wscale)
        layers.append(layer)
    chain = api.DecoderChain(layers, 2, hidden, kv, hd, inter, dev)
    h0 = synth.activations(8, 0, 2, hidden)
    chain.h.copy_(G.to_dev(h0, dev))
    api.decoder_chain_fused(chain)
    api.check()
    assert np.array_equal(_np(chain.h), h0)
