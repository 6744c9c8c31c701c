"""GPU parity of the 8-bit-weight forward (twell_quantize_e4m3_rows,
twell_ffn_fwd_e4m3) against the fp64 oracle, through the C ABI.

The quantisation is compared bit for bit with the oracle's (codes, scales and
dequantised weights, both for W_u's rows and for W_d's columns). The forward
must equal the oracle's FFN evaluated on the dequantised weights (the oracle
given the g values the GPU stored, within the stated tolerances; the plain
definition on the same weights to rel-L2), with the pack bit-exact; the gap
between the 8-bit-weight FFN and the bf16 one is printed.
"""

import numpy as np
import pytest

from synthetic import Workload, bf16_bits_from_f64, make_inputs, sweep_workload
from twell_testlib import (assert_matches_oracle, assert_pack_equal, bits_of, close_stats, f32_of_bits, gpu_gmat,
                           state_to_numpy, to_dev)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import activation_sparse_ffn_gemm_b200 as tw

    tw.lib()
    return tw


def test_quantize_matches_oracle(tw, orc):
    w = Workload("q", 8, 320, 1024, 128, 8, 0.05, seed=4)
    inp = make_inputs(w)
    Wu = inp["W_u"].copy()
    Wu[3] = 0  # a zero unit
    Wu[4] = bf16_bits_from_f64(np.linspace(-300.0, 300.0, Wu.shape[1]))  # a wide unit
    D = {k: to_dev(v) for k, v in (("W_u", Wu), ("W_d", inp["W_d"]))}
    q8 = tw.quantize_weights(D["W_u"], D["W_d"])
    torch.cuda.synchronize()
    ru = orc.quantize_e4m3(Wu, unit_axis=0)
    rd = orc.quantize_e4m3(inp["W_d"], unit_axis=1)
    assert np.array_equal(q8["W_u8"].cpu().numpy(), ru["q"])
    assert np.array_equal(q8["s_u"].cpu().numpy(), np.ldexp(1.0, ru["exp"]).astype(np.float32))
    assert np.array_equal(bits_of(q8["W_u"]), ru["deq"])
    assert np.array_equal(q8["W_dt8"].cpu().numpy(), rd["q"])
    assert np.array_equal(q8["s_d"].cpu().numpy(), np.ldexp(1.0, rd["exp"]).astype(np.float32))
    assert np.array_equal(bits_of(q8["W_d"]), rd["deq"])


CASES = {
    # name: (M, d, f, K, activity, row_scale, seed)
    "tiny": (64, 256, 1024, 16, 0.03, "none", 0),
    "ragged": (300, 192, 384, 8, 0.05, "lognormal", 1),
    "k64_split_rows": (130, 256, 2048, 64, 0.2, "lognormal", 4),
    "heavy_small": (1024, 1024, 4096, 8, 0.02, "lognormal", 23),
    "wide_d_w4": (40, 8192, 1024, 16, 0.05, "none", 8),
    "min_d_model": (50, 64, 256, 8, 0.05, "lognormal", 32),
}


def _check_q8_forward(tw, orc, w, sample=None):
    """Pack bit-exact; Y on every row, or (sample = n) on n seeded rows plus every overflow row."""
    inp = make_inputs(w)
    D = {k: to_dev(v) for k, v in inp.items() if k != "meta"}
    q8 = tw.quantize_weights(D["W_u"], D["W_d"])
    Y, st, z = tw.ffn_fwd_e4m3(D["X"], D["W_g"], D["b_g"], q8, K=w.K, z_debug=True)
    torch.cuda.synchronize()
    assert st.read_status() == 0
    p = state_to_numpy(st)
    assert_pack_equal(p, orc.pack(z.cpu().numpy().astype(np.float64), w.T_n, w.K))
    Wuq, Wdq = bits_of(q8["W_u"]), bits_of(q8["W_d"])
    M, f = w.M, w.d_ff
    if sample is None:
        rows = np.arange(M, dtype=np.int32)
    else:
        rng = np.random.default_rng(9)
        pick = set(rng.choice(M, sample, replace=False).tolist()) | set(p["ovf_rows"][:p["n_ovf"]].tolist())
        rows = np.array(sorted(pick), dtype=np.int32)
    G = gpu_gmat(p, M, f, w.T_n, w.K)[rows]
    a = (inp["X"], inp["W_g"], inp["b_g"], Wuq, Wdq)
    yg = f32_of_bits(bits_of(Y))[rows]
    per_row = w.row_scale == "lognormal"
    assert_matches_oracle(yg, orc.ffn_fwd(*a, rows=rows, gmat=G), orc.ffn_fwd(*a, rows=rows), f"{w.name} 8-bit Y",
                          bf16_out=True, per_row=per_row)
    # the gap to the FFN with the bf16 weights, for the record
    y_bf16 = orc.ffn_fwd(inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], rows=rows, gmat=G)
    gap = close_stats(yg, y_bf16)
    print(f"[8-bit weights] {w.name}: rel-L2 of Y against the bf16-weight FFN {gap['rel_l2']:.3e}")
    return gap


@pytest.mark.parametrize("name", sorted(CASES))
def test_fwd_e4m3_small(tw, orc, name):
    M, d, f, K, act, rs, seed = CASES[name]
    _check_q8_forward(tw, orc, Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed))


def test_fwd_e4m3_sweep_scale(tw, orc):
    """d_model=4096, d_ff=14336, M=8192, 99% sparsity, lognormal rows: Y on a
    seeded sample of rows plus every overflow row."""
    gap = _check_q8_forward(tw, orc, sweep_workload(8192, 0.01), sample=256)
    assert gap["rel_l2"] < 0.1  # E4M3 keeps 4 significant bits: a few percent, not a different function


@pytest.mark.parametrize("name", ["ragged", "heavy_small", "wide_d_w4", "min_d_model"])
def test_fwd_e4m3_schedules_agree(tw, name):
    """The 8-bit forward under the fused and the multi-pass schedule (the latter
    also with a 64 KiB L2 budget, so the passes run in many hidden-tile and
    column chunks): Y bit-identical, for an inference forward (u in the
    workspace) and with u saved."""
    M, d, f, K, act, rs, seed = CASES[name]
    w = Workload(name, M, d, f, 128, K, act, row_scale=rs, training=True, seed=seed)
    inp = make_inputs(w)
    D = {k: to_dev(v) for k, v in inp.items() if k != "meta"}
    q8 = tw.quantize_weights(D["W_u"], D["W_d"])
    outs = {}
    try:
        for label, mode, budget in (("fused", tw.SCHED_FUSED, 0), ("passes", tw.SCHED_PASSES, 0),
                                    ("chunked", tw.SCHED_PASSES, 64 << 10)):
            tw.set_sparse_schedule(mode, budget)
            Y, st = tw.ffn_fwd_e4m3(D["X"], D["W_g"], D["b_g"], q8, K=K)
            Ys, sts = tw.ffn_fwd_e4m3(D["X"], D["W_g"], D["b_g"], q8, K=K, save_for_backward=True)
            torch.cuda.synchronize()
            assert st.read_status() == 0 and sts.read_status() == 0, label
            outs[label] = (Y, Ys)
    finally:
        tw.set_sparse_schedule(tw.SCHED_AUTO, 0)
    for label in ("passes", "chunked"):
        for a, b in zip(outs["fused"], outs[label]):
            assert torch.equal(a, b), label
