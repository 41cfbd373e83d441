"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks (no GPU).

The library itself has no collective (the product is replicas only, one
independent call stream per GPU); what multi-GPU runs share is the timing
contract: every rank's device time is reduced with a max over ranks, and the
job's value counts the calls of all ranks.
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        local_ms = [3.0, 5.0][rank]               # rank 1 is the slow one
        ms = bench.aggregate_max(local_ms)
        value = bench.job_us_per_call(ms, steps=10, calls_per_step=6, world=world)
        q.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_all_calls():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [g[0] for g in got] == [0, 1]
    for _, ms, value in got:
        assert ms == pytest.approx(5.0)                          # max over ranks, on every rank
        assert value == pytest.approx(5.0 * 1000.0 / (10 * 6 * 2))  # all ranks' calls in the slowest time
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_value_is_plain_time_per_call():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.job_us_per_call(12.0, steps=100, calls_per_step=6, world=1) == pytest.approx(20.0)
