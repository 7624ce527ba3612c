"""Multi-process host logic of the replica benchmark, on CPU with gloo
(world size 2): each rank times its own replica, the job's time is the
slowest rank's, and the value counts the units of every rank."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        q.put((r, w, local, ms, bench.whole_job_value(6400.0, 10, w, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_time_is_max_over_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 for g in got)
    assert all(g[3] == 15.0 for g in got)                     # slowest rank
    assert all(g[4] == pytest.approx(6400 * 10 * 2 / 0.015) for g in got)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    assert bench.whole_job_value(100.0, 4, 1, 2.0) == pytest.approx(200000.0)
