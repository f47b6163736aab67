"""The replica (multi-GPU) bookkeeping of bench.py, on the CPU with two gloo
ranks: times reduce to the slowest rank's, and the whole-job rate counts
every rank's work over that time.  The path has no data exchange; these are
the only cross-rank operations."""

import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        vals = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 3.0])
        rate = bench.whole_job_rate(1e9, 2, world, vals[0])
        q.put((rank, vals, rate))
    finally:
        dist.destroy_process_group()


def test_times_are_the_slowest_ranks_and_rates_count_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(2):
            rank, vals, rate = q.get(timeout=120)
            out[rank] = (vals, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert sorted(out) == [0, 1]
    for vals, rate in out.values():
        assert vals == [2.0, 5.0, 3.0]
        # 2 ranks x 2 steps x 1 GB in the slowest rank's 2 ms
        assert rate == pytest.approx(2 * 2 * 1e9 / 2e-3 / 1e9)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([4.0, 1.5]) == [4.0, 1.5]
    assert bench.whole_job_rate(3e9, 5, 1, 1000.0) == pytest.approx(15.0)
