"""Rank logic of bench.py with world size 2 over gloo on CPU.

Every rank runs a full replica of the workload; the reported time is the
slowest rank's, and the job value counts the work of all ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local = [10.0, 12.5][rank]
    ms = bench.max_over_ranks(local, world, "cpu")
    dist.barrier()
    q.put((rank, ms, bench.job_value(world, 4 * 10**12, ms)))
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 12.5                              # the slowest rank's time
        assert abs(value - 2 * 4 * 10**12 / 12.5e-3 / 1e12) < 1e-9


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert abs(bench.job_value(1, 10**12, 1000.0) - 1.0) < 1e-12
