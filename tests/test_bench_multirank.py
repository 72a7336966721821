"""The bench's multi-rank aggregation on 2 gloo ranks (CPU, no GPU).

With N > 1 every rank runs an independent replica; the job's time is the max over
ranks and its throughput counts every rank's tokens over that time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = [3.0, 5.0][rank]                 # rank 1 is the slow one
        m = bench.max_over_ranks(elapsed, "cpu")
        dist.barrier()
        q.put((rank, m))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 5.0, 1: 5.0}


def test_single_rank_is_identity():
    assert bench.max_over_ranks(2.5, "cpu") == 2.5


def test_job_throughput_counts_every_rank():
    # 38,400 tokens per step, 10 steps, 2 ranks, slowest rank 4 ms
    assert bench.job_throughput(38400, 10, 2, 4.0) == pytest.approx(192.0)
