"""Multi-process host logic of bench.py's replica runs (world size 2, gloo on
the CPU): the step time is the slowest rank's and the value is the whole job's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        ms = bench.max_over_ranks(times[rank], world, "cpu")
        out[rank] = ms
        out[world + rank] = bench.replica_value(world, 465_041_408, 200, ms)
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_slowest_rank():
    world = 2
    times = [221.5, 230.25]  # ms for 200 steps on each rank
    out = torch.zeros(2 * world, dtype=torch.float64).share_memory_()
    mp.start_processes(_worker, args=(world, _free_port(), times, out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0].item() == pytest.approx(max(times))
    assert out[1].item() == pytest.approx(max(times))
    expect = world * 465_041_408 * 200 / (max(times) * 1e-3) / 1e9
    assert out[2].item() == pytest.approx(expect)
    assert out[3].item() == pytest.approx(expect)


def test_single_rank_is_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.replica_value(1, 1e9, 1, 1000.0) == pytest.approx(1.0)
