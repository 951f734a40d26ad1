"""The multi-GPU plumbing of bench.py on CPU: two ranks over gloo (127.0.0.1).

bench.py runs one independent copy of the workload per rank (no data-path collective:
the problems are independent), times it between a barrier and a synchronize, takes the
slowest rank's time with an all-reduce(MAX) and reports units processed by all ranks
divided by that time.  These tests exercise exactly that plumbing with gloo ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, times, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    d = bench.Dist()
    d.init("gloo")
    try:
        d.barrier()
        slowest = d.max(times[rank])
        value = bench.whole_job_value(1000.0, d.world, slowest)
        d.barrier()
        results[rank] = (d.rank, d.world, slowest, value)
    finally:
        d.close()


@pytest.mark.parametrize("world", [2])
def test_two_ranks_max_time_and_whole_job_value(world):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    times = [3.0, 5.0]  # per-rank ms; the slowest rank sets the job's time
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert sorted(results.keys()) == [0, 1]
    for r in range(world):
        rank, w, slowest, value = results[r]
        assert rank == r and w == world
        assert slowest == 5.0                      # max over ranks
        # units of all ranks over the slowest rank's time: 2 * 1000 / 5 ms = 400000 / s
        assert value == pytest.approx(2 * 1000.0 / 5e-3)


def test_single_process_defaults():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    d = bench.Dist()
    d.init("gloo")  # world 1: no process group
    assert d.world == 1 and d.rank == 0 and d.pg is None
    assert d.max(7.5) == 7.5
    d.barrier()
    d.close()
    assert bench.whole_job_value(10.0, 1, 2.0) == pytest.approx(5000.0)
