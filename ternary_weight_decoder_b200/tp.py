"""Tensor-parallel split of the ternary projections across ranks (one GPU
each), Megatron-style, on top of the library's entry points.

column-parallel (q, k, v, gate, up): a rank holds weight rows [n0, n0+rows)
    and the whole input; its output is its slice of y; nothing is exchanged.
row-parallel (o, down): a rank holds input columns [k0, k0+cols) and the
    matching columns of every weight row.  The ranks agree on each token's
    absmax (a max all-reduce of M floats), quantise their slices with it,
    add their partial int32 sums (a sum all-reduce of M x N) and rescale.
    Integer addition is exact, so every rank ends with the single-device
    bytes.

The slices of a matrix keep the scale of the whole matrix (ternarised
before the split).  Shard boundaries fall on 16-row blocks (column-parallel)
and 128-column tiles (row-parallel) and need not be equal.  The collectives
are torch.distributed all-reduces (NCCL between GPUs).  The arithmetic runs
in the library's kernels; `ops` only lets the host-side structure be
exercised with other implementations of the same four steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_bounds(total: int, unit: int, world: int, rank: int):
    """[start, stop) of rank's share of `total` in whole `unit`s (the last
    unit may be partial), as even as the units allow."""
    units = -(-total // unit)
    a, b = units * rank // world, units * (rank + 1) // world
    return min(a * unit, total), min(b * unit, total)


def column_shard(packed, N: int, K: int, world: int, rank: int):
    """(packed rows of this rank, n0, rows): 16-row blocks split evenly."""
    from ternary_weight_decoder_b200 import api
    n0, n1 = shard_bounds(N, 16, world, rank)
    return api.pack_slice(packed, N, K, n0, n1 - n0, 0, K), n0, n1 - n0


def row_shard(packed, N: int, K: int, world: int, rank: int):
    """(packed columns of this rank, k0, cols): 128-column tiles split evenly."""
    from ternary_weight_decoder_b200 import api
    k0, k1 = shard_bounds(K, 128, world, rank)
    return api.pack_slice(packed, N, K, 0, N, k0, k1 - k0), k0, k1 - k0


class CudaOps:
    """The four steps of a row-parallel projection, in the library's kernels."""

    def row_absmax(self, x):
        from ternary_weight_decoder_b200 import api
        return api.row_absmax(x)

    def quantize_given(self, x, amax):
        from ternary_weight_decoder_b200 import api
        return api.quantize_act_given(x, amax)

    def partial_acc(self, xq, amax, qsum, packed, wscale, N):
        from ternary_weight_decoder_b200 import api
        M = xq.shape[0]
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
        y = torch.empty((M, N), dtype=torch.float32, device=xq.device)
        api.ternary_linear_q(xq, amax, qsum, packed, wscale, N, y=y, acc_out=acc)
        return acc

    def rescale(self, acc, amax, wscale):
        from ternary_weight_decoder_b200 import api
        return api.rescale_acc(acc, amax, wscale)


def row_parallel(x_local, packed_local, wscale, N: int, group=None, ops=None):
    """y [M, N] (every rank) of a row-parallel projection from this rank's
    input slice x_local [M, cols] and its code columns packed_local."""
    ops = ops or CudaOps()
    amax = ops.row_absmax(x_local)
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    xq, qsum = ops.quantize_given(x_local, amax)
    acc = ops.partial_acc(xq, amax, qsum, packed_local, wscale, N)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return ops.rescale(acc, amax, wscale), acc


def column_parallel(x, packed_local, wscale, rows: int):
    """This rank's output columns of a column-parallel projection."""
    from ternary_weight_decoder_b200 import api
    return api.ternary_linear(x, packed_local, wscale, rows)
