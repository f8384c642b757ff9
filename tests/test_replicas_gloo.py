"""The multi-GPU bench path (independent replicas) on CPU with gloo, world size 2.

Every rank times its own replica; the job's step time is the max over ranks and
the job's rate counts every rank's work.  This exercises bench.py's reduction
and rate helpers across two real processes.
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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]     # per-rank (step, e2e) timings
        dist.barrier()
        got = bench.max_over_ranks(mine, "cpu")
        rate = bench.replica_rate(world, 2.0e12, got[0])
        out[rank] = (got[0], got[1], rate)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        step, e2e, rate = out[r]
        assert step == 15.0 and e2e == 20.0
        assert rate == pytest.approx(world * 2.0e12 / 15e-3 / 1e12)

