"""The N > 1 host logic of bench.py on CPU: two gloo ranks, each with its own
(fake) step time; the job time is the slowest rank's and the whole-job value
counts every rank's bytes (weak scaling: each rank codes its own tensors, so
there is no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 is slower in the first, faster in the second
        mx = bench.reduce_max(times, "cpu")
        val = bench.weak_scaling_value(2e9, world, mx[0])
        out[rank] = (mx, val)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        mx, val = out[r]
        assert mx == [15.0, 3.0]
        assert val == pytest.approx(world * 2e9 / (15.0 * 1e6))


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.weak_scaling_value(1e9, 1, 1.0) == pytest.approx(1000.0)
