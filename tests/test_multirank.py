"""The N > 1 bench path on CPU: two gloo ranks, each timing its own replica.

The path has no exchange step, so the only cross-rank operation is the
max-over-ranks reduction of the per-step time; every rank must see the max.
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_env()
        ms = 1.5 + rank  # rank 1 is the slow one
        got = bench.reduce_max(ms, dist, "cpu")
        q.put((rank, w, r, lr, got))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks():
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
    assert [r[:4] for r in res] == [(0, 2, 0, 0), (1, 2, 1, 1)]
    assert all(r[4] == pytest.approx(2.5) for r in res)


def test_single_rank_identity():
    import bench

    assert bench.reduce_max(3.25) == 3.25
