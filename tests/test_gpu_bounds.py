"""The bounds-checked build (libtwell_bounds.so) on guarded buffers: the
sanitizer substitute of this library (compute-sanitizer is not available).

Every caller-owned array of a forward and backward (state, workspaces, W_dt, Y
and the gradients) is carved from the middle of a larger allocation whose guard
regions before and after hold a known byte pattern. After the calls the guards
must be intact (no kernel wrote outside its arrays), the status word must not
carry TWELL_STATUS_BOUNDS (no index the kernels read was out of range), and the
results must be those of the regular library. A state whose column index was
corrupted on purpose (on the host side of the test, to a value that stays inside
every array even if it were used) must raise the bounds bit instead.
"""

import numpy as np
import pytest

from synthetic import Workload, make_inputs
from twell_testlib import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 1 << 16
PATTERN = 0xA5


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import activation_sparse_ffn_gemm_b200 as tw

    tw.lib()
    with tw.bounds_checked():
        tw.lib()
    return tw


class Guarded:
    """Arrays carved from allocations with GUARD pattern bytes before and after."""

    def __init__(self):
        self.parts = []

    def empty(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.empty(GUARD + n + GUARD, dtype=torch.uint8, device="cuda")
        raw[:GUARD].fill_(PATTERN)
        raw[GUARD + n:].fill_(PATTERN)
        self.parts.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        return all(bool((raw[:GUARD] == PATTERN).all()) and bool((raw[GUARD + n:] == PATTERN).all())
                   for raw, n in self.parts)


CASES = {
    # name: (M, d, f, K, activity, row_scale, seed)
    "ragged": (300, 192, 384, 8, 0.05, "lognormal", 1),
    "k64_split_rows": (130, 256, 2048, 64, 0.2, "lognormal", 4),
    "dense_wgrad": (300, 256, 512, 8, 0.12, "lognormal", 17),
    "heavy_small": (1024, 1024, 4096, 8, 0.02, "lognormal", 23),
    "ovf_rows_8": (384, 512, 2048, 8, 0.02, "none", 30),
}


def _run(tw, D, w, G, K):
    M, d, f = w.M, w.d_model, w.d_ff
    st = tw.HybridState(M, f, 128, K, None, "cuda", alloc=G.empty)
    wsf = tw.workspace(tw.OP_FWD, M, d, f, 128, K, M, alloc=G.empty)
    wsb = tw.workspace(tw.OP_BWD, M, d, f, 128, K, M, alloc=G.empty)
    Wdt = G.empty((f, d), torch.bfloat16)
    Y = G.empty((M, d), torch.bfloat16)
    out = dict(dX=G.empty((M, d), torch.float32), dW_g=G.empty((f, d), torch.float32),
               dW_u=G.empty((f, d), torch.float32), dW_d=G.empty((d, f), torch.float32),
               db_g=G.empty((f,), torch.float32))
    tw.transpose_wd(D["W_d"], out=Wdt)
    tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K, W_dt=Wdt, state=st, ws=wsf, Y=Y)
    return st, wsb, Wdt, Y, out


@pytest.mark.parametrize("name", sorted(CASES))
def test_bounds_checked_run_on_guarded_buffers(tw, name):
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    D = {k: to_dev(v) for k, v in make_inputs(w).items() if k != "meta"}
    Y0, st0 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
    g0 = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st0, D["dY"], lam=1e-3)
    G = Guarded()
    with tw.bounds_checked():
        st, wsb, Wdt, Y, out = _run(tw, D, w, G, K)
        tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3, W_dt=Wdt, ws=wsb, out=out)
        torch.cuda.synchronize()
        assert st.read_status() == 0, "an index out of range (or another device condition)"
    assert G.intact(), "a kernel wrote outside its arrays"
    # the checks change no arithmetic: the same results as the regular library
    assert torch.equal(Y, Y0)
    for k in out:
        assert torch.equal(out[k], g0[k]), k


@pytest.mark.parametrize("name", ["k64_split_rows", "heavy_small", "ovf_rows_8"])
def test_bounds_checked_passes_on_guarded_buffers(tw, name):
    """The same, under the multi-pass schedule with a 64 KiB L2 budget (the dot
    passes in many hidden-tile chunks, the axpy passes in column chunks with
    their own turnstile words in the workspace), and the 8-bit forward: guards
    intact, no bounds bit, the regular library's results."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    D = {k: to_dev(v) for k, v in make_inputs(w).items() if k != "meta"}
    try:
        tw.set_sparse_schedule(tw.SCHED_PASSES, 64 << 10)
        Y0, st0 = tw.ffn_fwd(D["X"], D["W_g"], D["b_g"], D["W_u"], D["W_d"], K=K)
        g0 = tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st0, D["dY"], lam=1e-3)
        q8 = tw.quantize_weights(D["W_u"], D["W_d"])
        Yq0, _ = tw.ffn_fwd_e4m3(D["X"], D["W_g"], D["b_g"], q8, K=K)
        G = Guarded()
        with tw.bounds_checked():
            tw.set_sparse_schedule(tw.SCHED_PASSES, 64 << 10)  # the checked library keeps its own setting
            st, wsb, Wdt, Y, out = _run(tw, D, w, G, K)
            tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3, W_dt=Wdt, ws=wsb, out=out)
            stq = tw.HybridState(M, f, 128, K, None, "cuda", alloc=G.empty)
            wsq = tw.workspace(tw.OP_FWD, M, d, f, 128, K, M, alloc=G.empty)
            Yq = G.empty((M, d), torch.bfloat16)
            tw.ffn_fwd_e4m3(D["X"], D["W_g"], D["b_g"], q8, K=K, state=stq, ws=wsq, Y=Yq)
            torch.cuda.synchronize()
            assert st.read_status() == 0 and stq.read_status() == 0
        assert G.intact(), "a kernel wrote outside its arrays"
        assert torch.equal(Y, Y0) and torch.equal(Yq, Yq0)
        for k in out:
            assert torch.equal(out[k], g0[k]), k
    finally:
        tw.set_sparse_schedule(tw.SCHED_AUTO, 0)
        with tw.bounds_checked():
            tw.set_sparse_schedule(tw.SCHED_AUTO, 0)


def test_bounds_checked_build_flags_a_corrupt_column(tw):
    """An in-tile column of 130 (>= T_n = 128) in an ELL slot of row r < 32,
    tile 0: the backward's kernels that read it (the sparse backward and the
    pair-list build) refuse it and set TWELL_STATUS_BOUNDS; no guard is touched.
    The value keeps every address in range even where it not checked (unit 130
    < d_ff; shared-memory row 0 of the pair-list counters), so the test cannot
    fault either way."""
    M, d, f, K, act, rs, seed = CASES["ragged"]
    w = Workload("ragged", M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    assert f >= 256
    D = {k: to_dev(v) for k, v in make_inputs(w).items() if k != "meta"}
    G = Guarded()
    with tw.bounds_checked():
        st, wsb, Wdt, Y, out = _run(tw, D, w, G, K)
        torch.cuda.synchronize()
        assert st.read_status() == 0
        count = st.count.cpu().numpy().view(np.uint16)
        row_ovf = st.row_ovf.cpu().numpy()[:M]
        rows = [r for r in range(32) if count[r, 0] >= 1 and not row_ovf[r]]
        assert rows, "no ELL row with an active unit in tile 0 among the first 32 rows"
        st.col[rows[0], 0, 0] = 130
        tw.ffn_bwd(D["X"], D["W_g"], D["W_u"], D["W_d"], st, D["dY"], lam=1e-3, W_dt=Wdt, ws=wsb, out=out)
        torch.cuda.synchronize()
        assert st.read_status() & tw.STATUS_BOUNDS
    assert G.intact()
