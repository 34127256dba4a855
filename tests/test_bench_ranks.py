"""Host logic of bench.py's multi-process path on CPU: two gloo ranks agree
on the max-over-ranks time and the whole-job value of N replicas."""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [2.0, 3.5][rank]
        ms = bench.max_over_ranks(dist, ms_local, "cpu")
        q.put((rank, ms, bench.whole_job_value(world, 3.2e12, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == 3.5
        assert value == pytest.approx(2 * 3.2e12 / 3.5e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 1.25, "cpu") == 1.25
    assert bench.whole_job_value(1, 1e12, 1.0) == pytest.approx(1000.0)
