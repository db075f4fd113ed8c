"""The multi-rank bench path on the CPU: two gloo ranks, each with its own
device time; the reported time is the max over ranks and the value counts the
tokens of every rank (replicas, weak scaling)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_info() == (world, rank, rank)
        my_ms = [40.0, 55.0][rank]
        ms, value = bench.aggregate(my_ms, tokens_per_rank=1000, steps=10, world=world)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_aggregate_max_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == 55.0
        assert value == pytest.approx(2 * 1000 * 10 / 0.055)


def test_aggregate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.aggregate(20.0, tokens_per_rank=500, steps=4, world=1)
    assert ms == 20.0 and value == pytest.approx(500 * 4 / 0.02)
