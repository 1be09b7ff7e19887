"""The benchmark's multi-GPU host logic on CPU: two gloo ranks, each timing
its own replica; the job time is the max over ranks and the throughput
counts every rank's tokens (weak scaling, no data-path collective)."""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms)
        rate = bench.weak_scaling_rate(1000.0, 4, world, total)
        q.put((rank, total, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_and_rate_counts_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, total, rate in res:
        assert total == pytest.approx(15.0)
        assert rate == pytest.approx(2 * 1000.0 * 4 / 0.015)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_rate(100.0, 2, 1, 1.0) == pytest.approx(200000.0)
