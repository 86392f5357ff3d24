"""Multi-process host logic of bench.py's replica mode, on the CPU with gloo (world size 2).

Each rank runs an independent replica; the job is timed by the slowest rank and its throughput is
the units of all ranks over that time.  No data-path collective is involved.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [0.5, 2.0][rank]                        # rank 1 is the slow one
        t = bench.max_over_ranks(dist, local, torch.device("cpu"))
        thr = bench.replica_throughput(100.0, world, t)
        dist.barrier()
        q.put((rank, t, thr))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, thr in got:
        assert t == 2.0                                 # max over ranks, seen by every rank
        assert thr == 100.0 * 2 / 2.0                   # units of both replicas over the slow time
