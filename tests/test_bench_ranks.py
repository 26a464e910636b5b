"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The benchmark runs one independent graph per rank (weak scaling, no data-path
collective); the reported time is the max over ranks and the processed edges are
summed over ranks.  This checks that reduction with real processes and the gloo
backend, and that a single process needs no process group.
"""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench._dist() == (world, rank, rank)
        ms, edges = bench.reduce_over_ranks(10.0 + 5.0 * rank, 1000 * (rank + 1))
        q.put((rank, ms, edges))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, edges in res:
        assert ms == 15.0          # max over ranks
        assert edges == 3000.0     # sum over ranks


def test_reduce_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(7.5, 42) == (7.5, 42.0)
