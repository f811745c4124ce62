"""The N > 1 bench path on CPU: two gloo ranks agree on the slowest rank's time and the whole-job
throughput counts every rank's units over that time."""

import os
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(times[rank])
        value = bench.job_throughput(8, world, 10, slowest)
        out[rank] = (slowest, value)
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_units():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + (os.getpid() % 1000)
    times = [12.5, 20.0]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 20.0
    # 8 queries*layers per rank-step, 2 ranks, 10 steps in 20 ms
    assert out[0][1] == pytest.approx(8 * 2 * 10 / 0.020)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(4, 1, 5, 10.0) == pytest.approx(4 * 5 / 0.010)
