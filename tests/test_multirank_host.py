"""The N > 1 host path of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job rate (each rank runs its own copy of the step: weak scaling, no data-path exchange)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [1.25, 3.5][rank]  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(local_ms, dist, device="cpu")
        rate = bench.whole_job_rate(world, 4 * 4096 * 1024, ms_max)
        dist.barrier()
        q.put((rank, ms_max, rate))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get() for _ in range(2))
    for rank, ms_max, rate in got:
        assert ms_max == 3.5
        # 2 ranks x 16 MiB of weights each, over the slowest rank's 3.5 ms
        assert rate == pytest.approx(2 * 4 * 4096 * 1024 / 3.5e-3 / 1e9)


def test_one_rank_keeps_its_own_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.0, None, device="cpu") == 2.0
    assert bench.whole_job_rate(1, 1e9, 1.0) == pytest.approx(1000.0)
