"""The tensor-parallel split's host structure (ternary_weight_decoder_b200.tp)
as two and three gloo ranks on the CPU: the row-parallel projection's max
all-reduce of the token absmax, the slices quantised with it, the int32 sum
all-reduce of the partial accumulators and the rescale give the unsplit
oracle's accumulators and outputs exactly; the column shards cover every
weight row once.  The four arithmetic steps run in the oracle here (no
GPU); the GPU tests run them in the library's kernels."""
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    """The steps of a row-parallel projection in the oracle, on CPU tensors."""

    def row_absmax(self, x):
        import torch
        return torch.from_numpy(np.abs(x.numpy()).max(axis=1).astype(np.float32))

    def quantize_given(self, x, amax):
        import torch
        from oracle import oracle as orc
        q = orc.quantize_act_given(x.numpy(), amax.numpy())
        return torch.from_numpy(q), torch.from_numpy(q.astype(np.int32).sum(axis=1).astype(np.int32))

    def partial_acc(self, xq, amax, qsum, codes_local, mean, N):
        import torch
        from oracle import oracle as orc
        return torch.from_numpy(orc.ternary_acc(codes_local, xq.numpy()))

    def rescale(self, acc, amax, mean):
        from oracle import oracle as orc
        return orc.rescale(acc.numpy(), amax.numpy(), mean)


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth, tp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, N, K = 3, 40, 896          # 7 tiles of 128 columns: unequal shares
        W = synth.weights(5, 6, N, K)
        x = synth.activations(5, 6, M, K)
        codes, mean = orc.ternarize(W)                 # the whole matrix's scale
        k0, k1 = tp.shard_bounds(K, 128, world, rank)
        y, acc = tp.row_parallel(torch.from_numpy(np.ascontiguousarray(x[:, k0:k1])),
                                 np.ascontiguousarray(codes[:, k0:k1]), mean, N, ops=OracleOps())
        n0, n1 = tp.shard_bounds(N, 16, world, rank)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), y=y, acc=acc.numpy(),
                 k=np.array([k0, k1]), n=np.array([n0, n1]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_parallel_equals_single_device(tmp_path, world):
    import torch.multiprocessing as mp
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    M, N, K = 3, 40, 896
    W, x = synth.weights(5, 6, N, K), synth.activations(5, 6, M, K)
    codes, mean = orc.ternarize(W)
    full = orc.ternary_linear(x, codes, mean)
    ks, ns = [], []
    for rank in range(world):
        r = np.load(tmp_path / f"r{rank}.npz")
        assert (r["acc"] == full["acc"]).all(), rank     # every rank: the whole sum
        assert (r["y"] == full["y"]).all(), rank
        ks.append(tuple(r["k"]))
        ns.append(tuple(r["n"]))
    # the shards tile K and N exactly, on 128-column and 16-row boundaries
    assert ks[0][0] == 0 and ks[-1][1] == K and all(a[1] == b[0] for a, b in zip(ks, ks[1:]))
    assert all(k0 % 128 == 0 for k0, _ in ks)
    assert ns[0][0] == 0 and ns[-1][1] == N and all(a[1] == b[0] for a, b in zip(ns, ns[1:]))
    assert all(n0 % 16 == 0 for n0, _ in ns)
