"""The bench's multi-rank path on CPU: world size 2 over gloo (127.0.0.1).

Each rank runs its own replica of the step, so the only cross-rank steps are a
barrier and the maximum of the device timings; this checks that both ranks get
the slowest rank's time and that the whole-job rate counts every rank's bytes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        mine = [10.0 + rank, 20.0 - rank]            # rank 1 slower on the first figure
        got = bench.max_over_ranks(mine, dist)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [11.0, 20.0]


def test_whole_job_rate_counts_every_rank():
    import bench
    assert bench.whole_job_rate(2_000_000_000, 1, 1.0) == pytest.approx(2000.0)
    assert bench.whole_job_rate(2_000_000_000, 4, 2.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
