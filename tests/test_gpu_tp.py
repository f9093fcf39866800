"""The tensor-parallel pieces on one GPU: ranks emulated one after another
(their kernels never wait on one another), the all-reduces done as a
maximum and an int32 sum of the ranks' tensors.  Code slices must unpack to
the oracle's code slices; row-parallel partial sums must add up to the
unsplit accumulators and the rescaled outputs match the unsplit GPU outputs
bit for bit (and the oracle); column shards give the unsplit columns."""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import gpu_util as G
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return G.torch_dev()


@pytest.fixture(scope="module")
def api():
    return G.api()


@pytest.mark.parametrize("N,K,n0,rows,k0,cols", [(1536, 1536, 0, 768, 0, 1536),
                                                 (1000, 640, 992, 8, 128, 384),
                                                 (256, 8960, 16, 240, 4480, 4480),
                                                 (37, 256, 32, 5, 0, 128)])
def test_pack_slice_matches_oracle_codes(dev, api, N, K, n0, rows, k0, cols):
    W = synth.weights(N, K % 977, N, K)
    packed, _, _ = G.ternarize_gpu(W, dev)
    sl = api.pack_slice(packed, N, K, n0, rows, k0, cols)
    got, invalid = api.unpack_codes(sl, rows, cols)
    api.check()
    codes, _ = orc.ternarize(W)
    assert (got.cpu().numpy() == codes[n0:n0 + rows, k0:k0 + cols]).all()
    assert int(invalid.cpu()[0]) == 0


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("M,N,K", [(1, 1536, 8960), (5, 1536, 1536), (300, 256, 1536)])
def test_row_parallel_sums_to_single_device(dev, api, world, M, N, K):
    import torch
    from ternary_weight_decoder_b200 import tp
    W = synth.weights(M + world, 5, N, K)
    x = synth.activations(M + world, 5, M, K)
    packed, _, wscale = G.ternarize_gpu(W, dev)
    xd = G.to_dev(x, dev)
    acc_full = torch.empty((M, N), dtype=torch.int32, device=dev)
    y_full = api.ternary_linear(xd, packed, wscale, N, acc_out=acc_full)
    ops = tp.CudaOps()
    shards = []
    for r in range(world):
        pl, k0, cols = tp.row_shard(packed, N, K, world, r)
        xl = xd[:, k0:k0 + cols].contiguous()
        shards.append((pl, xl))
    amax = torch.stack([ops.row_absmax(xl) for _, xl in shards]).max(dim=0).values   # max all-reduce
    acc = torch.zeros((M, N), dtype=torch.int32, device=dev)
    for pl, xl in shards:
        xq, qsum = ops.quantize_given(xl, amax)
        acc += ops.partial_acc(xq, amax, qsum, pl, wscale, N)                         # sum all-reduce
    y = ops.rescale(acc, amax, wscale)
    api.check()
    assert torch.equal(acc, acc_full)
    assert torch.equal(y, y_full)
    codes, mean = orc.ternarize(W)
    ref = orc.ternary_linear(x, codes, mean)
    assert (acc.cpu().numpy() == ref["acc"]).all()
    G.assert_y_close(y.cpu().numpy(), ref["y"], f"tp{world} {M}x{N}x{K}")


@pytest.mark.parametrize("world", [2, 3])
def test_column_parallel_gives_the_columns(dev, api, world):
    import torch
    from ternary_weight_decoder_b200 import tp
    M, N, K = 4, 1000, 1536
    W, x = synth.weights(9, 9, N, K), synth.activations(9, 9, M, K)
    packed, _, wscale = G.ternarize_gpu(W, dev)
    xd = G.to_dev(x, dev)
    y_full = api.ternary_linear(xd, packed, wscale, N)
    parts = []
    for r in range(world):
        pl, n0, rows = tp.column_shard(packed, N, K, world, r)
        parts.append(tp.column_parallel(xd, pl, wscale, rows))
    api.check()
    assert torch.equal(torch.cat(parts, dim=1), y_full)


def test_quantize_given_and_rescale_match_oracle(dev, api):
    M, K, N = 6, 1024, 64
    x = synth.activations(3, 3, M, K)
    amax = (np.abs(x).max(axis=1) * np.float32(1.5)).astype(np.float32)
    amax[2] = 0.0
    xq, qsum = api.quantize_act_given(G.to_dev(x, dev), G.to_dev(amax, dev))
    api.check()
    want = orc.quantize_act_given(x, amax)
    assert (xq.cpu().numpy() == want).all()
    assert (qsum.cpu().numpy() == want.astype(np.int64).sum(axis=1)).all()
    acc = np.random.default_rng(0).integers(-10**6, 10**6, (M, N)).astype(np.int32)
    y = api.rescale_acc(G.to_dev(acc, dev), G.to_dev(amax, dev),
                        G.to_dev(np.array([0.0173], np.float32), dev))
    api.check()
    G.assert_y_close(y.cpu().numpy(), orc.rescale(acc, amax, float(np.float32(0.0173))), "rescale")
