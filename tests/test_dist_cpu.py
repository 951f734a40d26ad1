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


# ---------------------------------------------------------------- row-sharded quantization
def _shard_main(rank: int, world: int, port: int, x, splits, results):
    """Each rank: the oracle's amax of its rows, the library's reduce_amax_ over gloo,
    then the oracle's quantization of its rows with the reduced tensor's g."""
    import numpy as np
    import oracle
    import torch
    import torch.distributed as dist

    from block_scaled_fp4_04_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = splits[rank], splits[rank + 1]
        local = np.ascontiguousarray(x[lo:hi])
        amax = torch.tensor([oracle.amax(local)], dtype=torch.float32)
        sharded.reduce_amax_(amax)
        g = oracle.global_scale(float(amax.item()))
        q = oracle.quantize(local, oracle.NVFP4, 16, g_in=g)
        results[rank] = (float(amax.item()), q["codes"].tobytes(), q["scales"].tobytes(), float(g))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("splits", [[0, 40, 96], [0, 95, 96]])
def test_row_shards_with_one_max_all_reduce_equal_the_whole_tensor(splits):
    """Two gloo ranks hold row shards of one tensor (the largest element on one of them);
    after the all-reduce (MAX) of their local maxima, each rank's quantization equals the
    whole tensor's rows bit for bit, and both ranks hold the same g."""
    import numpy as np
    import oracle
    world = len(splits) - 1
    rng = np.random.default_rng(3)
    x = rng.standard_normal((splits[-1], 256)).astype(np.float32)
    x[splits[1], 7] = 60.0              # the tensor amax sits on rank 1
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_shard_main, args=(r, world, port, x, splits, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    whole = oracle.quantize(x, oracle.NVFP4, 16)
    for r in range(world):
        amax, codes, scales, g = results[r]
        lo, hi = splits[r], splits[r + 1]
        assert amax == 60.0
        assert np.float32(g) == whole["g"]
        assert codes == whole["codes"][lo:hi].tobytes()
        assert scales == whole["scales"][lo:hi].tobytes()
    # without the exchange rank 0 would pick its own, smaller g and different scales
    local0 = oracle.quantize(np.ascontiguousarray(x[:splits[1]]), oracle.NVFP4, 16)
    assert local0["g"] != whole["g"]


def test_reduce_amax_is_a_no_op_without_a_process_group():
    import torch
    from block_scaled_fp4_04_b200 import sharded
    t = torch.tensor([2.5])
    assert sharded.reduce_amax_(t).item() == 2.5


def test_bench_refuses_a_gpu_count_without_matching_ranks():
    """`bench.py --gpus 2` outside torchrun would silently measure one GPU: it stops with
    a message naming the launch command instead (before touching a GPU)."""
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"), "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode != 0
    assert "--nproc-per-node 2" in r.stderr
