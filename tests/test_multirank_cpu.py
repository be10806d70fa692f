"""Host logic of bench.py's multi-rank mode on CPU: two gloo ranks, each timing its own
independent batch, agree on the slowest rank's time and report the whole-job rate."""

import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_by_rank, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(ms_by_rank[rank], dist, torch.device("cpu"))
        rate = bench.whole_job_rate(1000, world, slowest)
        queue.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ms_by_rank", [(2.0, 3.0), (5.0, 1.0)])
def test_two_ranks_report_the_slowest_time(ms_by_rank):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ms_by_rank, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(queue.get(timeout=10) for _ in range(2))
    want = max(ms_by_rank)
    for rank, slowest, rate in got:
        assert slowest == want
        assert rate == pytest.approx(1000 * 2 / (want * 1e-3))


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.5, None, torch.device("cpu")) == 4.5
    assert bench.whole_job_rate(10, 1, 2.0) == pytest.approx(5000.0)
