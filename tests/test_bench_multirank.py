"""Host logic of the multi-GPU bench path (N independent replicas), run as
two gloo ranks on the CPU: ranks meet at the barrier, device times are
reported as the max over ranks, and the job rate counts every rank's units
over the slowest rank's time."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank                  # rank 1 is the slowest
        bench.barrier(world)
        mx = bench.max_over_ranks(my_ms, world)
        rate = bench.job_throughput(8192 * 20, world, mx)
        bench.barrier(world)
        results[rank] = (mx, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_job_rate():
    world = 2
    port = 29500 + os.getpid() % 1000
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = dict(results)
    assert got[0] == got[1]
    mx, rate = got[0]
    assert mx == 15.0
    assert rate == pytest.approx(2 * 8192 * 20 / 15e-3)


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(100, 1, 2.0) == pytest.approx(5e4)
