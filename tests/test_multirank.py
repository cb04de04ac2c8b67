"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Each rank runs its own copy of the workload (weak scaling); the reported
time is the max over ranks and the work the sum over ranks.  The ranks here
only exercise that reduction; no GPU is involved.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, rank, world)
        elapsed = 1.0 + rank          # rank 1 is the slow one
        units = 16 * (rank + 1)
        t, u = bench.aggregate(elapsed, units)
        bench.barrier()
        q.put((rank, t, u))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_total_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, u in got:
        assert t == 2.0            # the slowest rank's time
        assert u == 16 + 32        # every rank's tokens


def test_single_process_passthrough():
    import bench
    assert bench.aggregate(1.5, 16) == (1.5, 16)
