"""The multi-GPU path of bench.py (data-parallel replicas, no collective on
the data path) as two gloo ranks on the CPU: the timing is the maximum over
ranks on every rank, the whole-job value counts every rank's tokens over
that time, each rank decodes its own token stream, and the reference arm
runs on rank 0 only."""
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


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    import bench
    from ternary_weight_decoder_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        ms = 10.0 * (rank + 1)                       # rank 1 is the slow one
        max_ms = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        value = bench.job_value(M=4, world=world, steps=100, max_ms=max_ms)
        x = synth.activations(bench.rank_layer_seed(3, rank), 1, 2, 256)
        gathered = [None] * world
        dist.all_gather_object(gathered, x.tobytes())
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.array([max_ms, value, float(gathered[0] != gathered[1])]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_is_max_and_value_counts_all_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for rank in (0, 1):
        max_ms, value, differ = np.load(tmp_path / f"r{rank}.npy")
        assert max_ms == 20.0                        # the slowest rank, on both ranks
        assert value == pytest.approx(4 * 2 * 100 / 0.020)
        assert differ == 1.0                         # ranks decode different tokens


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    # rank 1 returns at once, without touching the oracle or printing

    class A:
        m, layers, steps, warmup, gpus = 1, 28, 3, 3, 2
    assert bench.run_reference(A()) is None
    assert capsys.readouterr().out == ""
