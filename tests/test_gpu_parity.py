"""GPU parity of the sm_100a path against the fp64 CPU oracle, through the C ABI.

Small cases compare every output element; the full-size workloads compare the
pack on every row, the gate output element by element, and Y on every row (the
uniform inference workload) or on a seeded sample of rows plus every overflow
row (the heavy-tailed ones); the training workloads' gradients on full tensors.
Tolerances are stated in tests/twell_testlib.py: the plain bounds on the
uniform cases, the per-row reading on the lognormal ones.
"""

import json
import os

import numpy as np
import pytest

from synthetic import WORKLOADS, Workload, make_inputs, sweep_workload
from twell_testlib import (assert_active_set, assert_gate_close, assert_matches_oracle, assert_pack_equal,
                           assert_plan_valid, bits_of, f32_of_bits, gate_error_bound, gpu_gmat, gpu_gmat_cols,
                           gpu_gmat_rows, state_to_numpy, to_dev)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import activation_sparse_ffn_gemm_b200 as tw

    tw.lib()
    return tw


def _dev(inp):
    return {k: to_dev(v) for k, v in inp.items() if k != "meta"}


def _run_fwd(tw, inp, w, cap=None, save=True, dense_min=0):
    D = _dev(inp)
    Y, st, z = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], T_n=w.T_n, K=w.K, ovf_cap=cap,
                          save_for_backward=save, z_debug=True, dense_min=dense_min)
    torch.cuda.synchronize()
    return D, Y, st, z


def _check_fwd(orc, inp, w, Y, st, z, rows=None, cap=None):
    """Pack bit-exact (all rows); gate z element by element, active set and Y
    (all rows or the given sample)."""
    M, f = inp["X"].shape[0], inp["W_g"].shape[0]
    zg = z.cpu().numpy()
    p_gpu = state_to_numpy(st)
    p_ref = orc.pack(zg.astype(np.float64), w.T_n, w.K, cap=cap, dense_min=st.dense_min)
    assert_pack_equal(p_gpu, p_ref)
    expect = 8 if p_ref["n_ovf_total"] > p_ref["n_ovf"] else 0  # TWELL_STATUS_OVERFLOW_CAP
    assert st.read_status() == expect
    if rows is None:
        rows = np.arange(M, dtype=np.int32)
    z64 = orc.gate(inp["X"], inp["W_g"], inp["b_g"], rows=rows)
    assert_gate_close(zg[rows], z64, gate_error_bound(inp["X"], inp["W_g"], inp["b_g"], rows=rows))
    flips = assert_active_set(zg[rows], z64, float(np.sqrt(np.mean(z64 ** 2))))
    args = (inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"])
    G = gpu_gmat(p_gpu, M, f, w.T_n, w.K)
    y_stored = orc.ffn_fwd(*args, rows=rows, gmat=G[rows])
    y_plain = orc.ffn_fwd(*args, rows=rows)
    yg = f32_of_bits(bits_of(Y))[rows]
    stats = assert_matches_oracle(yg, y_stored, y_plain, "Y", bf16_out=True, per_row=w.row_scale == "lognormal")
    return p_gpu, flips, stats


def _check_bwd(orc, inp, g, G, lam, name, per_row, skip_rows=None):
    """Every gradient on its full tensor (dX without the rows in skip_rows)."""
    args = (inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], inp["dY"], lam)
    ref_s = orc.ffn_bwd(*args, gmat=G)
    ref_p = orc.ffn_bwd(*args, mask=(G != 0).astype(np.uint8))
    keep = None
    if skip_rows is not None and len(skip_rows):
        keep = np.setdiff1d(np.arange(inp["X"].shape[0]), skip_rows)
    for k in ("dX", "dW_g", "dW_u", "dW_d", "db_g"):
        a, rs, rp = g[k].cpu().numpy(), ref_s[k], ref_p[k]
        if k == "dX" and keep is not None:
            a, rs, rp = a[keep], rs[keep], rp[keep]
        assert_matches_oracle(a, rs, rp, f"{name} {k} lambda={lam}", per_row=per_row)


CASES = {
    # name: (M, d, f, K, activity, row_scale, seed)
    "tiny": (64, 256, 1024, 16, 0.03, "none", 0),
    "ragged": (300, 192, 384, 8, 0.05, "lognormal", 1),
    "ragged_k16": (389, 320, 640, 16, 0.06, "lognormal", 2),
    "k32": (257, 512, 1024, 32, 0.1, "lognormal", 3),
    "k64": (130, 256, 2048, 64, 0.2, "lognormal", 4),
    "one_row": (1, 128, 256, 8, 0.3, "none", 5),
    "multi_tile": (700, 1024, 2048, 8, 0.01, "lognormal", 6),
    # rows of ~400 kept entries (the long-row pass) with two warps per token
    "long_rows_w2": (96, 4096, 4096, 32, 0.1, "none", 7),
    # four and eight warps per token (d_model / 8 chunks of 16 bytes > 512)
    "wide_d_w4": (40, 8192, 1024, 16, 0.05, "none", 8),
    "widest_d_w8": (24, 16384, 512, 8, 0.03, "none", 10),
    # overflow rows dense enough that their weight gradients run as GEMMs
    # (190 and 183 overflow rows: the contraction's zeroed tail rows matter)
    "dense_wgrad": (300, 256, 512, 8, 0.12, "lognormal", 17),
    "dense_wgrad_ragged": (260, 192, 384, 8, 0.15, "lognormal", 19),
    # 170 overflow rows of a heavy-tailed batch: split-K dense backup GEMMs,
    # overflow pairs kept in the pair list
    "heavy_small": (1024, 1024, 4096, 8, 0.02, "lognormal", 23),
    # the supported extremes: d_ff = 16384 (128 tiles), d_model = 64
    "max_d_ff": (40, 256, 16384, 8, 0.02, "none", 31),
    "min_d_model": (50, 64, 256, 8, 0.05, "lognormal", 32),
    # 8 and 9 overflow rows: split-K dense backup GEMMs of a few rows
    "ovf_rows_8": (384, 512, 2048, 8, 0.02, "none", 30),
    "ovf_rows_9": (384, 512, 2048, 8, 0.02, "none", 41),
}


# cases whose plan splits some rows into several pieces (the ordered
# accumulation across pieces is exercised)
SPLIT_CASES = ("k64", "long_rows_w2", "multi_tile")
# cases whose overflow rows pass the cost model of the dense weight gradients;
# the others keep their overflow rows in the pair list
DENSE_WGRAD_CASES = ("dense_wgrad", "dense_wgrad_ragged")


@pytest.mark.parametrize("name", sorted(CASES))
def test_fwd_bwd_small(tw, orc, name):
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w)
    p, flips, _ = _check_fwd(orc, inp, w, Y, st, z)
    if name.startswith("ovf_rows_"):
        assert p["n_ovf"] == int(name.rsplit("_", 1)[1])
    plan = assert_plan_valid(st)
    if name in SPLIT_CASES:
        assert plan["split_rows"] > 0, "this case should split rows into several pieces"
    assert plan["dense_wgrad"] == (name in DENSE_WGRAD_CASES)
    for lam in (0.0, 1e-3):
        g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=lam)
        torch.cuda.synchronize()
        _check_bwd(orc, inp, g, gpu_gmat(p, M, f, 128, K), lam, name, per_row=rs == "lognormal")
        assert_plan_valid(st)


def test_degenerate_all_inactive(tw, orc):
    w = Workload("off", 200, 256, 512, 128, 8, 0.01, training=True)
    inp = make_inputs(w)
    inp["b_g"][:] = 0xC6C0  # bf16 -24576: no unit can be active
    D, Y, st, z = _run_fwd(tw, inp, w)
    assert not st.count.any().item() and st.n_overflow() == (0, 0)
    assert not Y.float().abs().sum().item()
    g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=0.5)
    for k, v in g.items():
        assert not v.abs().sum().item(), k


def test_degenerate_all_active_dense_path(tw, orc):
    """b >> 0: every unit active, every row overflows K < T_n, everything runs dense."""
    w = Workload("on", 150, 256, 384, 128, 8, 0.01, training=True, seed=9)
    inp = make_inputs(w)
    inp["b_g"][:] = 0x4120  # bf16 10.0
    D, Y, st, z = _run_fwd(tw, inp, w)
    p, _, _ = _check_fwd(orc, inp, w, Y, st, z)
    assert p["n_ovf"] == 150 and p["row_ovf"].all()
    assert assert_plan_valid(st)["dense_wgrad"]
    g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
    _check_bwd(orc, inp, g, gpu_gmat(p, 150, 384, 128, 8), 1e-3, "all-active", per_row=False)


def test_overflow_capacity_exceeded(tw, orc):
    w = Workload("cap", 256, 256, 512, 128, 8, 0.15, row_scale="lognormal", seed=3)
    inp = make_inputs(w)
    Z = orc.gate(inp["X"], inp["W_g"], inp["b_g"])
    n_flag = orc.pack(Z, 128, 8)["n_ovf_total"]
    assert n_flag >= 4
    cap = n_flag // 2
    D = _dev(inp)
    st, z = tw.pack(D["X"], D["W_g"], D["b_g"], T_n=128, K=8, ovf_cap=cap, z_debug=True)
    torch.cuda.synchronize()
    p_ref = orc.pack(z.cpu().numpy().astype(np.float64), 128, 8, cap=cap)
    assert_pack_equal(state_to_numpy(st), p_ref)
    assert st.n_overflow() == (cap, p_ref["n_ovf_total"])
    assert st.read_status(clear=True) == tw.STATUS_OVERFLOW_CAP
    assert st.read_status() == 0


def test_empty_batch(tw):
    d, f = 256, 512
    X = torch.empty((0, d), dtype=torch.bfloat16, device="cuda")
    W = torch.randn((f, d), device="cuda").bfloat16()
    Wd = torch.randn((d, f), device="cuda").bfloat16()
    b = torch.zeros(f, device="cuda").bfloat16()
    Y, st = tw.ffn_fwd(X, W, b, W, Wd, K=8)
    g = tw.ffn_bwd(X, W, W, Wd, st, X, lam=0.1)
    torch.cuda.synchronize()
    assert Y.shape == (0, d)
    for k in ("dW_g", "dW_u", "dW_d", "db_g"):
        assert not g[k].abs().sum().item()


def test_deterministic(tw):
    w = Workload("det", 300, 512, 1024, 128, 8, 0.05, row_scale="lognormal", training=True, seed=11)
    D = _dev(make_inputs(w))
    outs = []
    for _ in range(2):
        Y, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=8)
        g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
        torch.cuda.synchronize()
        outs.append([Y.clone()] + [g[k].clone() for k in sorted(g)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


SCHEDULE_CASES = ("ragged", "k64", "long_rows_w2", "wide_d_w4", "widest_d_w8", "heavy_small", "multi_tile",
                  "min_d_model", "max_d_ff", "dense_wgrad")


@pytest.mark.parametrize("name", SCHEDULE_CASES)
def test_schedules_agree_bit_for_bit(tw, name):
    """The fused sparse kernels and the multi-pass schedule (one pass per
    gathered weight matrix), the latter also with a 64 KiB L2 budget that cuts
    the up and dH passes into many hidden-tile chunks and the down and dX passes
    into column chunks: Y, the saved u and every gradient are identical, for a
    training forward and for an inference forward (u in the workspace)."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    D = _dev(make_inputs(w))
    outs = {}
    try:
        for label, mode, budget in (("fused", tw.SCHED_FUSED, 0), ("passes", tw.SCHED_PASSES, 0),
                                    ("chunked", tw.SCHED_PASSES, 64 << 10)):
            tw.set_sparse_schedule(mode, budget)
            Y, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
            g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
            Yi, sti = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K, save_for_backward=False)
            torch.cuda.synchronize()
            assert st.read_status() == 0 and sti.read_status() == 0, label
            cnt = (st.count.to(torch.int32) & 0xFFFF).clamp(max=K)
            kept = (torch.arange(K, device=cnt.device) < cnt[..., None]) & (st.row_ovf[:M] == 0)[:, None, None]
            outs[label] = [Y, st.u_ell[kept], Yi] + [g[k] for k in sorted(g)]
    finally:
        tw.set_sparse_schedule(tw.SCHED_AUTO, 0)
    for label in ("passes", "chunked"):
        for a, b in zip(outs["fused"], outs[label]):
            assert torch.equal(a, b), label


def test_overlap_agrees_and_captures(tw):
    """The dense-backup chain on the library's side stream (twell_set_overlap)
    gives the same Y and gradients as everything on the caller's stream, bit
    for bit, on a batch whose dense backup runs split-K (170 overflow rows) and
    on one whose dense rows' weight gradients run as GEMMs; and a forward +
    backward with the side stream captured into a CUDA graph and replayed
    reproduces them too (the fork and join are capturable)."""
    for name in ("heavy_small", "dense_wgrad"):
        M, d, f, K, act, rs, seed = CASES[name]
        w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
        D = _dev(make_inputs(w))
        outs = {}
        try:
            for on in (False, True):
                tw.set_overlap(on)
                Y, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
                g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
                torch.cuda.synchronize()
                assert st.read_status() == 0
                outs[on] = [Y] + [g[k] for k in sorted(g)]
            for a, b in zip(outs[False], outs[True]):
                assert torch.equal(a, b), name
            # graph capture with the overlap on: preallocated state, workspaces and outputs
            tw.set_overlap(True)
            dev = D["X"].device
            st = tw.HybridState(M, f, 128, K, M, dev, with_u=True)
            wsf = tw.workspace(tw.OP_FWD, M, d, f, 128, K, M, dev)
            wsb = tw.workspace(tw.OP_BWD, M, d, f, 128, K, M, dev)
            Wdt = tw.transpose_wd(D["W_d"])
            Y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
            out = dict(dX=torch.empty((M, d), device=dev), dW_g=torch.empty((f, d), device=dev),
                       dW_u=torch.empty((f, d), device=dev), dW_d=torch.empty((d, f), device=dev),
                       db_g=torch.empty((f,), device=dev))

            def run():
                tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K, W_dt=Wdt, state=st, ws=wsf, Y=Y)
                tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3, W_dt=Wdt, ws=wsb, out=out)

            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                run()
            torch.cuda.current_stream().wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                run()
            for k in out:
                out[k].zero_()
            Y.zero_()
            graph.replay()
            torch.cuda.synchronize()
            assert st.read_status() == 0
            for a, b in zip([Y] + [out[k] for k in sorted(out)], outs[True]):
                assert torch.equal(a, b), name + " (graph replay)"
            del graph
        finally:
            tw.set_overlap(tw.OVERLAP_AUTO)


def test_prepared_wdt_matches(tw):
    w = Workload("wdt", 256, 512, 1024, 128, 8, 0.03, training=True, seed=12)
    D = _dev(make_inputs(w))
    Wdt = tw.transpose_wd(D["W_d"])
    assert torch.equal(Wdt, D["W_d"].t().contiguous())
    Y1, st1 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=8)
    Y2, st2 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=8, W_dt=Wdt)
    g1 = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st1, D["dY"], lam=0.0)
    g2 = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st2, D["dY"], lam=0.0, W_dt=Wdt)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


# ------------------------------------------------------------ full-size workloads


def _sample_rows(M, n, seed, extra=()):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist()) | set(int(r) for r in extra)
    return np.array(sorted(rows), dtype=np.int32)


def test_uniform_full_size(tw, orc):
    """Inference forward, uniform 1% activity, M=4096 d=2048 d_ff=8192 K=8 (no overflow rows):
    the gate output and Y on every row."""
    w = WORKLOADS["uniform"]
    with open(os.path.join(GOLDEN, "uniform_seed.json")) as fh:
        seed = json.load(fh)["seed"]
    inp = make_inputs(w, seed=seed)
    D, Y, st, z = _run_fwd(tw, inp, w, save=False)
    p, flips, stats = _check_fwd(orc, inp, w, Y, st, z)
    assert p["n_ovf_total"] == 0
    assert assert_plan_valid(st)["split_rows"] == 0  # 1% i.i.d. rows are short: one piece each


def test_heavy_tail_full_size(tw, orc):
    """Inference forward, lognormal row scale, M=16384 d=4096 d_ff=14336 K=8: exercises the dense backup."""
    w = WORKLOADS["heavy"]
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w, save=False)
    p = state_to_numpy(st)
    assert p["n_ovf"] > 0
    cnt = p["count"].astype(np.float64)
    assert cnt.max() / cnt.mean() >= 10
    rng = np.random.default_rng(1)
    ovf_sample = rng.choice(p["ovf_rows"], size=min(64, p["n_ovf"]), replace=False)
    plan = assert_plan_valid(st)
    assert plan["split_rows"] > 0  # the heavy ELL rows are split into pieces
    pieces = st.row_plan.cpu().numpy()[4 + 2 * w.M:4 + 2 * w.M + 2 * plan["pieces"]].reshape(-1, 2)
    split = np.unique(pieces[pieces[:, 1] == 1, 0])
    split_sample = rng.choice(split, size=min(32, split.size), replace=False)
    rows = _sample_rows(w.M, 128, 1, extra=np.concatenate([ovf_sample, split_sample]))
    _check_fwd(orc, inp, w, Y, st, z, rows=rows)


def test_train_full_size(tw, orc):
    """Training step, M=8192 d=2048 d_ff=8192 K=8, lambda in {0, 1e-3}; gradients on full tensors."""
    w = WORKLOADS["train"]
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w)
    rows = _sample_rows(w.M, 256, 2)
    p, _, _ = _check_fwd(orc, inp, w, Y, st, z, rows=rows)
    G = gpu_gmat(p, w.M, w.d_ff, w.T_n, w.K)
    for lam in (0.0, 1e-3):
        g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=lam)
        torch.cuda.synchronize()
        _check_bwd(orc, inp, g, G, lam, "train", per_row=False)


@pytest.mark.parametrize("name", ["tiny", "ragged", "heavy_small", "one_row", "k64"])
def test_count_stats(tw, orc, name):
    """twell_count_stats bit-exact against the oracle's statistics of its own pack
    of the GPU's z; the rows above K are the routed overflow rows, the actives
    of the other rows are the plan's kept total; the K choice runs on them."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w)
    gs = {k: v.cpu().numpy() for k, v in tw.count_stats(st).items()}
    p_ref = orc.pack(z.cpu().numpy().astype(np.float64), 128, K)
    ref = orc.count_stats(p_ref["count"], 128)
    for k in ref:
        assert np.array_equal(gs[k], ref[k]), k
    assert gs["rows_by_max"][K + 1:].sum() == st.n_overflow()[1]
    assert gs["act_by_max"][:K + 1].sum() == int(st.row_plan[2].item())
    best, times = tw.suggest_k(gs, d, f)
    assert best in times and len(times) == 4
    # with a row threshold, rows of at least dense_min actives move to the last bin
    dm = max(1, int(np.median(p_ref["count"].astype(np.int64).sum(1))))
    st.c.dense_min = dm
    gs = {k: v.cpu().numpy() for k, v in tw.count_stats(st).items()}
    ref = orc.count_stats(p_ref["count"], 128, dense_min=dm)
    for k in ref:
        assert np.array_equal(gs[k], ref[k]), k


@pytest.mark.parametrize("name,frac", [("heavy_small", 0.5), ("ragged", 0.3), ("k64", 0.6)])
def test_dense_min_routing(tw, orc, name, frac):
    """Rows with at least dense_min active units go to the dense backup as well
    (threshold at a quantile of the row totals): pack bit-exact against the
    oracle's pack with the same rule, Y and every gradient against the oracle."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D0, Y0, st0, z0 = _run_fwd(tw, inp, w)
    totals = st0.count.cpu().numpy().view(np.uint16).astype(np.int64).sum(1)
    dm = max(1, int(np.quantile(totals, 1.0 - frac)))
    D, Y, st, z = _run_fwd(tw, inp, w, dense_min=dm)
    n_plain, n_thr = st0.n_overflow()[1], st.n_overflow()[1]
    assert n_thr == int(((st0.count.cpu().numpy().view(np.uint16) > K).any(1) | (totals >= dm)).sum())
    assert n_thr > n_plain
    p, _, _ = _check_fwd(orc, inp, w, Y, st, z)
    assert_plan_valid(st)
    for lam in (0.0, 1e-3):
        g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=lam)
        torch.cuda.synchronize()
        _check_bwd(orc, inp, g, gpu_gmat(p, M, f, 128, K), lam, f"{name} dense_min={dm}", per_row=rs == "lognormal")
    assert st.read_status() == 0


def test_autograd_function(tw, orc):
    """twell_ffn under autograd: the same Y as twell_ffn_fwd and the same
    gradients as twell_ffn_bwd (rounded to the inputs' bf16), for a 3-D input,
    with the L1 term and a row threshold; and Y against the oracle."""
    M, d, f, K, act, rs, seed = CASES["ragged"]
    w = Workload("ragged", M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D = _dev(inp)
    dm = 20
    Y_ref, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K, dense_min=dm)
    g_ref = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
    leaves = {k: D[k].clone().requires_grad_() for k in ("X", "W_g", "b_g", "W_u", "W_d")}
    X3 = leaves["X"].view(2, M // 2, d)
    Y = tw.twell_ffn(X3, leaves["W_g"], leaves["b_g"], leaves["W_u"], leaves["W_d"], K=K, lam=1e-3, dense_min=dm)
    assert Y.shape == (2, M // 2, d) and torch.equal(Y.reshape(M, d), Y_ref)
    (Y.float() * D["dY"].view(2, M // 2, d).float()).sum().backward()
    torch.cuda.synchronize()
    for k, gk in (("X", "dX"), ("W_g", "dW_g"), ("b_g", "db_g"), ("W_u", "dW_u"), ("W_d", "dW_d")):
        assert leaves[k].grad.dtype == torch.bfloat16
        assert torch.equal(leaves[k].grad, g_ref[gk].to(torch.bfloat16)), k
    args = (inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"])
    G = gpu_gmat(state_to_numpy(st), M, f, 128, K)
    assert_matches_oracle(f32_of_bits(bits_of(Y_ref)), orc.ffn_fwd(*args, gmat=G), orc.ffn_fwd(*args),
                          "autograd Y", bf16_out=True, per_row=rs == "lognormal")


def test_count_stats_empty_batch(tw):
    st = tw.HybridState(0, 256, 128, 8, 0, "cuda")
    out = tw.count_stats(st)
    torch.cuda.synchronize()
    assert all(v.shape == (130,) and int(v.abs().sum().item()) == 0 for v in out.values())


@pytest.mark.parametrize("M,activity,bwd", [(2048, 0.1, False), (512, 0.001, False), (64, 0.1, True),
                                              (96, 0.05, True)])
def test_sweep_points(tw, orc, M, activity, bwd):
    """Points of the d_model=4096, d_ff=14336 lognormal sweep (K = 64, 8, 64, 32):
    pack on all rows and Y on a sample plus every overflow row; for the small-M
    points also the backward, every gradient on its full tensor."""
    w = sweep_workload(M, activity)
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w, save=bwd)
    p = state_to_numpy(st)
    extra = p["ovf_rows"][:p["n_ovf"]][:16]
    rows = np.arange(M, dtype=np.int32) if bwd else _sample_rows(M, 64, 3, extra=extra)
    p, _, _ = _check_fwd(orc, inp, w, Y, st, z, rows=rows)
    assert_plan_valid(st)
    if bwd:
        G = gpu_gmat(p, M, w.d_ff, w.T_n, w.K)
        g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
        torch.cuda.synchronize()
        assert st.read_status() == 0
        _check_bwd(orc, inp, g, G, 1e-3, w.name, per_row=True)


@pytest.mark.parametrize("name", ["k32", "multi_tile", "ragged_k16", "tiny"])
def test_tile_routing_forward(tw, orc, name):
    """Per-(row, tile) overflow routing: every active unit runs sparsely (tiles
    over K read from their spilled slice); Y matches the oracle with the GPU's
    stored g = bf16(ReLU(z)) for every unit, no row is dense, and the state is
    refused by the backward."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D = _dev(inp)
    Y, st, z = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], T_n=128, K=K, z_debug=True,
                          tile_routing=True)
    torch.cuda.synchronize()
    zg = z.cpu().numpy()
    p_gpu = state_to_numpy(st)
    p_ref = orc.pack(zg.astype(np.float64), 128, K)
    for k in ("count", "val", "col"):
        assert np.array_equal(p_gpu[k], p_ref[k]), k
    assert not p_gpu["row_ovf"].any() and st.n_overflow() == (0, 0)
    assert st.read_status() == 0
    plan = st.row_plan.cpu().numpy()
    assert plan[3] == -1
    counts = p_gpu["count"].astype(np.int64)
    assert plan[2] == counts.sum()  # every active unit is listed
    G = orc.bf16_round(np.maximum(zg.astype(np.float64), 0.0))
    args = (inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"])
    y_stored = orc.ffn_fwd(*args, gmat=G)
    y_plain = orc.ffn_fwd(*args)
    assert_matches_oracle(f32_of_bits(bits_of(Y)), y_stored, y_plain, f"{name} tile-routed Y", bf16_out=True,
                          per_row=rs == "lognormal")
    # the inference-only state is refused by the backward, which writes nothing
    tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=0.0)
    assert st.read_status(clear=True) == tw.STATUS_BAD_STATE


def test_turnstile_wait_gives_up(tw, orc):
    """Failure detection without a GPU fault: a piece whose predecessor never
    runs waits on its row's turnstile word, which nothing sets; the bounded
    wait (2 s of %globaltimer) gives up, the kernel records
    TWELL_STATUS_TIMEOUT and returns, and the context stays usable."""
    w = Workload("turn", 64, 256, 1024, 128, 16, 0.05, training=True, seed=21)
    inp = make_inputs(w)
    D = _dev(inp)
    Y, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=16)
    torch.cuda.synchronize()
    assert st.read_status() == 0
    kept0 = int(np.minimum(st.count[0].cpu().numpy().view(np.uint16), 16).sum())
    assert kept0 >= 2
    # plan: one piece, (row 0, q = 1) of a row cut into pieces of one entry;
    # piece q = 0 is never handed out, so turn word 0 never reaches 1
    M = st.M
    plan = st.row_plan
    plan[0] = 1
    plan[1] = 1
    plan[3] = 0
    plan[4:4 + M] = 0
    plan[4 + 2 * M:4 + 2 * M + 2] = torch.tensor([0, 1], dtype=torch.int32, device=plan.device)
    torch.cuda.synchronize()
    tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=0.0)
    assert st.read_status(clear=True) & tw.STATUS_TIMEOUT
    # the context is still usable: a fresh forward and backward run clean
    Y2, st2 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=16)
    g2 = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st2, D["dY"], lam=0.0)
    torch.cuda.synchronize()
    assert st2.read_status() == 0
    assert torch.equal(Y2, Y)


@pytest.mark.parametrize("activity", [0.01, 0.1])
def test_sweep_scale_training(tw, orc, activity):
    """A sweep point at full width: d_model=4096, d_ff=14336, M=8192 tokens with
    lognormal row scaling, at 99% (K=8) and 90% (K=64) sparsity. The pack on every
    row; the gate output and Y on a seeded sample of 256 rows plus every overflow
    row; every gradient on its full tensor (lambda = 1e-3). Hundreds of rows
    overflow, so the dense backup runs without split-K and the overflow rows'
    weight gradients take the tensor-core path."""
    w = sweep_workload(8192, activity)
    inp = make_inputs(w)
    D, Y, st, z = _run_fwd(tw, inp, w)
    p = state_to_numpy(st)
    assert p["n_ovf"] >= 64
    plan = assert_plan_valid(st)
    assert plan["dense_wgrad"]
    rows = _sample_rows(w.M, 256, 5, extra=p["ovf_rows"][:p["n_ovf"]])
    p, _, _ = _check_fwd(orc, inp, w, Y, st, z, rows=rows)
    G = gpu_gmat(p, w.M, w.d_ff, w.T_n, w.K)
    g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
    torch.cuda.synchronize()
    assert st.read_status() == 0
    _check_bwd(orc, inp, g, G, 1e-3, w.name, per_row=True)


def test_headline_full_size(tw, orc):
    """The benchmark's headline workload at full size, in its launch configuration:
    d_model=4096, d_ff=14336, M=65536 tokens, 99% sparsity, lognormal rows, K=8,
    dense-backup capacity M/4, the default (multi-pass) schedule, a training step
    with lambda = 1e-3. On a seeded sample of 192 rows plus 64 overflow rows: the
    pack bit-exact against the oracle's pack of the GPU's z, z element by element,
    Y and dX against the oracle given the GPU's stored g. The weight gradients of
    16 units (12 seeded, 4 active in overflow rows) against the oracle's
    per-unit gradients over all 65536 rows."""
    w = WORKLOADS["large"]
    inp = make_inputs(w)
    M, d, f, K, T_n = w.M, w.d_model, w.d_ff, w.K, w.T_n
    D = _dev(inp)
    Y, st, z = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], T_n=T_n, K=K, ovf_cap=M // 4,
                          save_for_backward=True, z_debug=True)
    g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3)
    torch.cuda.synchronize()
    assert st.read_status() == 0
    p = state_to_numpy(st)
    n = p["n_ovf"]
    assert n > 1000 and p["n_ovf_total"] == n
    plan = assert_plan_valid(st)
    assert plan["dense_wgrad"] and plan["split_rows"] > 0
    rows = _sample_rows(M, 192, 11, extra=p["ovf_rows"][:n][:: max(1, n // 64)][:64])
    zr = z[torch.from_numpy(rows.astype(np.int64)).to(z.device)].cpu().numpy()
    del z
    # pack of the sampled rows (row-local) against the oracle's pack of the GPU's z
    ref = orc.pack(zr.astype(np.float64), T_n, K)
    for k in ("count", "val", "col", "row_ovf"):
        assert np.array_equal(p[k][rows], ref[k]), k
    is_ovf = p["row_ovf"][rows] != 0
    slots = np.searchsorted(p["ovf_rows"][:n], rows[is_ovf])
    assert np.array_equal(p["g_ovf"][slots], ref["g_ovf"][:ref["n_ovf"]])
    # gate output on the sampled rows
    z64 = orc.gate(inp["X"], inp["W_g"], inp["b_g"], rows=rows)
    assert_gate_close(zr, z64, gate_error_bound(inp["X"], inp["W_g"], inp["b_g"], rows=rows))
    assert_active_set(zr, z64, float(np.sqrt(np.mean(z64 ** 2))))
    # Y and dX on the sampled rows (both row-local), given the GPU's stored g
    Gr = gpu_gmat_rows(p, rows, f, T_n, K)
    assert np.array_equal(Gr, orc.unpack(ref, f, T_n, K))
    args = (inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"])
    yg = f32_of_bits(bits_of(Y))[rows]
    assert_matches_oracle(yg, orc.ffn_fwd(*args, rows=rows, gmat=Gr), orc.ffn_fwd(*args, rows=rows), "headline Y",
                          bf16_out=True, per_row=True)
    Xs, dYs = inp["X"][rows], inp["dY"][rows]
    sub = (Xs, inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], dYs, 1e-3)
    assert_matches_oracle(g["dX"].cpu().numpy()[rows], orc.ffn_bwd(*sub, gmat=Gr)["dX"],
                          orc.ffn_bwd(*sub, mask=(Gr != 0).astype(np.uint8))["dX"], "headline dX", per_row=True)
    # the weight gradients of sampled units over every row
    rng = np.random.default_rng(12)
    busy = np.nonzero(p["g_ovf"][:n].any(axis=0))[0]
    units = np.unique(np.concatenate([rng.choice(f, 12, replace=False), rng.choice(busy, 4, replace=False)]))
    ru = orc.ffn_bwd_units(inp["X"], inp["W_u"], inp["W_d"], inp["dY"], 1e-3, units,
                           gpu_gmat_cols(p, units, M, T_n, K))
    ut = torch.from_numpy(units).to(g["dW_u"].device)
    for k, a in (("dW_g", g["dW_g"][ut]), ("dW_u", g["dW_u"][ut]), ("dW_d", g["dW_d"][:, ut].t())):
        o = ru[k] if k != "dW_d" else ru[k].T
        assert_matches_oracle(a.cpu().numpy(), o, o, f"headline {k} (sampled units)", per_row=True)
    assert_matches_oracle(g["db_g"][ut].cpu().numpy(), ru["db_g"], ru["db_g"], "headline db_g (sampled units)")


def test_split_epilogue_barrier_gives_up(tw):
    """Failure detection without a GPU fault: the split-K dense-backup GEMM of a
    forward with 8 overflow rows runs with one epilogue warp that never reaches
    the bounded barrier before the tile's partial sums are counted (the
    library's test switch). The wait runs out after 2 s, the kernel sets
    TWELL_STATUS_TIMEOUT and unwinds; the context stays usable, and the next
    forward gives the clean result again."""
    M, d, f, K, act, rs, seed = CASES["ovf_rows_8"]
    w = Workload("ovf_rows_8", M, d, f, 128, K, act, row_scale=rs, seed=seed)
    D = _dev(make_inputs(w))
    Y0, st0 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
    torch.cuda.synchronize()
    assert st0.read_status() == 0 and st0.n_overflow() == (8, 8)
    try:
        tw.test_withhold_epilogue_arrival(2)  # the forward's two dense-backup GEMMs; the second splits
        Y1, st1 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
        torch.cuda.synchronize()
    finally:
        tw.test_withhold_epilogue_arrival(0)
    assert st1.read_status(clear=True) & tw.STATUS_TIMEOUT
    Y2, st2 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
    torch.cuda.synchronize()
    assert st2.read_status() == 0
    assert torch.equal(Y2, Y0)


def test_backward_over_capacity(tw, orc):
    """A forward that flagged more overflow rows than ovf_cap: the backward sets
    TWELL_STATUS_OVERFLOW_CAP again, leaves the dX rows of the rows it could not
    store untouched and their pairs out of the weight gradients; every other
    gradient entry matches the oracle evaluated on the g the GPU stored (in which
    those rows hold no active unit)."""
    w = Workload("cap", 256, 256, 512, 128, 8, 0.15, row_scale="lognormal", training=True, seed=3)
    inp = make_inputs(w)
    n_flag = orc.pack(orc.gate(inp["X"], inp["W_g"], inp["b_g"]), 128, 8)["n_ovf_total"]
    assert n_flag >= 4
    cap = n_flag // 2
    D = _dev(inp)
    Y, st = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=8, ovf_cap=cap)
    torch.cuda.synchronize()
    assert st.read_status(clear=True) == tw.STATUS_OVERFLOW_CAP
    assert st.n_overflow() == (cap, n_flag)
    M, d, f = w.M, w.d_model, w.d_ff
    out = dict(dX=torch.full((M, d), 7.0, device="cuda"), dW_g=torch.empty((f, d), device="cuda"),
               dW_u=torch.empty((f, d), device="cuda"), dW_d=torch.empty((d, f), device="cuda"),
               db_g=torch.empty(f, device="cuda"))
    g = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3, out=out)
    torch.cuda.synchronize()
    assert st.read_status() == tw.STATUS_OVERFLOW_CAP
    p = state_to_numpy(st)
    unstored = np.setdiff1d(np.nonzero(p["row_ovf"])[0], p["ovf_rows"][:p["n_ovf"]])
    assert unstored.size == n_flag - cap
    assert bool((g["dX"][torch.from_numpy(unstored).cuda()] == 7.0).all())
    G = gpu_gmat(p, M, f, 128, 8)
    assert not G[unstored].any()
    _check_bwd(orc, inp, g, G, 1e-3, "over capacity", per_row=True, skip_rows=unstored)
