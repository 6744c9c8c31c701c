"""The token-sharded training step on CPU process groups (gloo, world size 2).

Each rank runs the local forward and backward of its own contiguous token shard
(here the fp64 oracle stands in for the CUDA library, which this host cannot
run); the step sums the weight gradients over the ranks. The result must equal
the gradients of the whole batch computed in one process: Y and dX row for row
(rows are independent), the weight gradients up to the order of the fp64 sums.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from activation_sparse_ffn_gemm_b200.sharded import GRAD_KEYS, ShardedTwellFFN, shard_bounds

LAM = 1e-3


def test_shard_bounds_cover_the_batch():
    for M in (0, 1, 7, 96, 97, 4096):
        for world in (1, 2, 3, 8):
            spans = [shard_bounds(M, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)


def _inputs():
    from synthetic import Workload, make_inputs

    w = Workload("dp", 97, 64, 256, 128, 8, 0.08, row_scale="lognormal", training=True, seed=5)
    return make_inputs(w)


def _oracle_step(inp, lo, hi):
    """Local step of rows [lo, hi) with the oracle: Y, dX of those rows and the
    weight gradients of those rows alone, as float64 torch tensors."""
    from oracle import oracle as O

    rows = np.arange(lo, hi, dtype=np.int32)
    Y = O.ffn_fwd(inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], rows=rows)
    g = O.ffn_bwd(inp["X"][lo:hi], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], inp["dY"][lo:hi], LAM)
    out = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in g.items()}
    out["Y"] = torch.from_numpy(Y)
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _inputs()
        lo, hi = shard_bounds(inp["X"].shape[0], world, rank)
        step = ShardedTwellFFN(local_step=lambda *a: _oracle_step(inp, lo, hi))
        out, handles = step.step(None, None, None, None, None, None, LAM, wait=False)
        assert len(handles) == len(GRAD_KEYS)
        for h in handles:
            h.wait()
        q.put((rank, lo, hi, {k: v.numpy() for k, v in out.items()}))
    finally:
        dist.destroy_process_group()


def test_two_rank_step_equals_the_whole_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    inp = _inputs()
    M = inp["X"].shape[0]
    whole = {k: v.numpy() for k, v in _oracle_step(inp, 0, M).items()}
    assert [(r[1], r[2]) for r in res] == [(0, 49), (49, 97)]  # uneven shards
    for rank, lo, hi, out in res:
        # rows are independent: this rank's Y and dX are those rows of the whole batch, exactly
        assert np.array_equal(out["Y"], whole["Y"][lo:hi])
        assert np.array_equal(out["dX"], whole["dX"][lo:hi])
        # the summed weight gradients are the whole batch's, up to the order of the fp64 sums
        for k in GRAD_KEYS:
            scale = np.abs(whole[k]).max()
            assert scale > 0
            np.testing.assert_allclose(out[k], whole[k], rtol=0, atol=1e-12 * scale)
    # both ranks hold the same reduced gradients
    for k in GRAD_KEYS:
        assert np.array_equal(res[0][3][k], res[1][3][k])


def test_single_process_step_needs_no_group():
    inp = _inputs()
    step = ShardedTwellFFN(local_step=lambda *a: _oracle_step(inp, 0, 10))
    out, handles = step.step(None, None, None, None, None, None, LAM)
    assert handles == [] and out["dX"].shape == (10, 64)
