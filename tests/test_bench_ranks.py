"""bench.py's multi-rank bookkeeping on CPU: two gloo ranks with different
timings agree on the slowest one, and the job throughput counts every rank's
units over that time (weak scaling: each rank proves its own statement)."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import datetime

    import torch.distributed as td

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is slower
        slowest = bench.max_over_ranks(mine, td, "cpu")
        q.put((rank, slowest, bench.job_throughput(1000.0, world, 4, slowest)))
        td.barrier()
    finally:
        td.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [15.0, 15.0]
    # 2 ranks x 1000 units x 4 steps in 15 ms
    assert got[0][2] == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(10.0, 1, 2, 1000.0) == pytest.approx(20.0)
