"""Host logic of the multi-GPU bench run (replicas with max-over-ranks timing), exercised
with two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank                   # rank 1 is the slower one
        mx = bench.max_over_ranks(local_ms, world)
        rate = bench.job_throughput(1000.0, mx, world)
        bench.barrier(world)
        out[rank] = (mx, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_the_slowest_and_units_add_up():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        mx, rate = out[r]
        assert mx == pytest.approx(15.0)
        # 1000 units on each of 2 ranks in the slowest rank's 15 ms
        assert rate == pytest.approx(2000.0 / 15e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.job_throughput(10.0, 2.0, 1) == pytest.approx(5000.0)
