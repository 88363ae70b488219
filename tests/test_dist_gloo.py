"""The multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each rank quantizes its own weight set (weak scaling, no data-path
collective); the job's throughput is the units of all ranks divided by the
slowest rank's time.  Here each rank reports made-up units and times and the
reduction is checked.
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
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    try:
        bench.init_dist(world, "gloo")
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        units = 1000.0 * (rank + 1)          # rank 0: 1000, rank 1: 2000
        secs = 0.5 + rank                    # rank 0: 0.5 s, rank 1: 1.5 s
        thr, t = bench.job_throughput(units, secs, world)
        bench.barrier(world)
        q.put((rank, thr, t))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_job_throughput_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, thr, t in res:
        assert t == pytest.approx(1.5)              # slowest rank
        assert thr == pytest.approx(3000.0 / 1.5)   # all units / slowest time


def test_single_rank_is_identity():
    import bench
    thr, t = bench.job_throughput(100.0, 2.0, 1)
    assert (thr, t) == (50.0, 2.0)
