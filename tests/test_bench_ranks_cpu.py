"""The multi-rank host logic of bench.py on CPU: two gloo ranks (replicas)
agree on the job's step time (the max over ranks) and the whole-job
throughput (every replica's bytes over that time).  No GPU."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], world, dist, "cpu")
        q.put((rank, ms, bench.job_gbs(2 ** 31, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 2000
    times = [0.36, 0.41]  # ms per step on each replica
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in got] == [0, 1]
    for _, ms, gbs in got:
        assert ms == pytest.approx(0.41)
        assert gbs == pytest.approx(2 * 2 ** 31 / 0.41e-3 / 1e9)


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1, None, "cpu") == 0.5
    assert bench.job_gbs(10 ** 9, 1, 1.0) == pytest.approx(1000.0)
