"""Host logic of the ELL-width choice (activation_sparse_ffn_gemm_b200.kchoice):
the modelled time of each candidate K against values worked out by hand."""

import numpy as np
import pytest

from activation_sparse_ffn_gemm_b200.kchoice import CostModel, dense_min_for, modelled_times, suggest_k

T_n = 128


def _stats(rows_by_max, act_by_max, tiles_by_count):
    out = {}
    for k, v in (("rows_by_max", rows_by_max), ("act_by_max", act_by_max), ("tiles_by_count", tiles_by_count)):
        a = np.zeros(T_n + 2, np.int64)
        for c, n in v.items():
            a[c] = n
        out[k] = a
    return out


# unit coefficients, so each term can be read off: pair = 1 s per d element,
# dense row = 10 s per d*f element, 1 byte/s
UNIT = CostModel(pair_fwd_s=1.0, pair_bwd_s=0.0, dense_fwd_s=10.0, dense_bwd_s=0.0, hbm_bytes_s=1.0,
                 gemm_launch_s=0.0, weight_stream_bytes_s=1e300)


def test_row_routing_terms_by_hand():
    # 3 rows with largest count 5 (30 actives), 1 row with 20 (40 actives); T = 2 tiles
    st = _stats({5: 3, 20: 1}, {5: 30, 20: 40}, {5: 3, 3: 3, 20: 1, 1: 1})
    t = modelled_times(st, d_model=2, d_ff=256, candidates=(8, 32), training=False, model=UNIT)
    M, T = 4, 2
    # K=8: 30 pairs sparse, 1 row dense; K=32: all 70 pairs sparse, no dense row
    assert t[8] == 1.0 * 2 * 30 + 10.0 * 2 * 256 * 1 + M * T * (2 + 3 * 8)
    assert t[32] == 1.0 * 2 * 70 + M * T * (2 + 3 * 32)
    # a row routed dense by the threshold (bin T_n + 1) is dense at every K
    st2 = _stats({5: 3, T_n + 1: 1}, {5: 30, T_n + 1: 40}, {5: 3, 3: 3, 20: 1, 1: 1})
    t2 = modelled_times(st2, d_model=2, d_ff=256, candidates=(8, 32), training=False, model=UNIT)
    assert t2[8] == t[8] and t2[32] == 1.0 * 2 * 30 + 10.0 * 2 * 256 * 1 + M * T * (2 + 3 * 32)
    best, times = suggest_k(st, d_model=2, d_ff=256, candidates=(8, 32), training=False, model=UNIT)
    assert best == 32 and times == t


def test_tile_routing_terms_by_hand():
    st = _stats({5: 3, 20: 1}, {5: 30, 20: 40}, {5: 3, 3: 3, 20: 1, 1: 1})
    t = modelled_times(st, d_model=2, d_ff=256, candidates=(4, 8), training=False, routing="tiles", model=UNIT)
    # every active unit gathered; spilled tiles: count > 4 -> 4 tiles (three 5s, one 20); > 8 -> 1
    assert t[4] == 1.0 * 2 * 70 + 4 * 2 * (2 + 3 * 4) + 512 * 4
    assert t[8] == 1.0 * 2 * 70 + 4 * 2 * (2 + 3 * 8) + 512 * 1
    with pytest.raises(ValueError):
        modelled_times(st, 2, 256, training=True, routing="tiles")


def test_training_adds_backward_terms():
    st = _stats({10: 2}, {10: 12}, {10: 2, 1: 2})
    m = CostModel(pair_fwd_s=1.0, pair_bwd_s=2.0, dense_fwd_s=4.0, dense_bwd_s=5.0, hbm_bytes_s=1e30,
                  gemm_launch_s=0.0, weight_stream_bytes_s=1e300)
    t_inf = modelled_times(st, 1, 256, candidates=(8, 16), training=False, model=m)
    t_trn = modelled_times(st, 1, 256, candidates=(8, 16), training=True, model=m)
    assert t_inf[8] == pytest.approx(4.0 * 256 * 2) and t_trn[8] == pytest.approx(9.0 * 256 * 2)
    assert t_inf[16] == pytest.approx(1.0 * 12) and t_trn[16] == pytest.approx(3.0 * 12)


def test_no_overflow_prefers_smallest_k_and_ties_go_small():
    st = _stats({3: 100}, {3: 500}, {3: 100, 0: 100})
    best, times = suggest_k(st, 2048, 256)
    assert best == 8 and times[8] < times[16] < times[32] < times[64]
    free = CostModel(pair_fwd_s=0.0, pair_bwd_s=0.0, dense_fwd_s=0.0, dense_bwd_s=0.0, hbm_bytes_s=1e300,
                     gemm_launch_s=0.0, weight_stream_bytes_s=1e300)
    assert suggest_k(st, 2048, 256, model=free)[0] == 8


def test_heavy_rows_trade_slots_for_dense_rows():
    """Rows with many actives go dense at a small K when a dense row is cheap next
    to their gathers, and stay sparse at a large K when it is not."""
    st = _stats({4: 1000, 40: 10}, {4: 3000, 40: 10 * 2000}, {4: 1000, 40: 10, 0: 1010 * 111})
    d, f = 4096, 14336
    cheap_dense = CostModel(pair_fwd_s=1e-12, pair_bwd_s=0.0, dense_fwd_s=1e-17, dense_bwd_s=0.0, gemm_launch_s=0.0,
                            weight_stream_bytes_s=1e300)
    dear_dense = CostModel(pair_fwd_s=1e-12, pair_bwd_s=0.0, dense_fwd_s=1e-12, dense_bwd_s=0.0)
    assert suggest_k(st, d, f, training=False, model=cheap_dense)[0] == 8
    assert suggest_k(st, d, f, training=False, model=dear_dense)[0] == 64


def test_rejects_bad_statistics():
    st = _stats({3: 1}, {3: 3}, {3: 1})
    st["rows_by_max"] = st["rows_by_max"][:-1]
    with pytest.raises(ValueError):
        suggest_k(st, 64, 128)
    with pytest.raises(ValueError):
        modelled_times(_stats({3: 1}, {3: 3}, {3: 1}), 64, 128, candidates=(0,))


def test_dense_min_break_even():
    m = CostModel(pair_fwd_s=2.0, pair_bwd_s=3.0, dense_fwd_s=1.0, dense_bwd_s=4.0)
    # ceil(r * d_ff / a): inference 1 * 256 / 2, training 5 * 256 / 5
    assert dense_min_for(64, 256, training=False, model=m) == 128
    assert dense_min_for(64, 256, training=True, model=m) == 256
    # the measured coefficients: weights in L2 at d_model=2048, d_ff=8192, from HBM at 4096 x 14336
    assert CostModel.for_shape(2048, 8192).pair_fwd_s < CostModel.for_shape(4096, 14336).pair_fwd_s
    for d, f in ((2048, 8192), (4096, 14336)):
        for training in (False, True):
            a = dense_min_for(d, f, training)
            # about 1-3% of the row active: above the 1% rows of the uniform workload's mean
            assert 0.01 * f < a < 0.03 * f, (d, f, training, a)


def test_fixed_cost_of_the_first_overflow_row():
    """One overflowing row at K=8 costs the backup GEMMs' fixed time; K=16 keeps it in ELL
    slots for a few more slot bytes, so the uniform 1% batch picks K=16."""
    m = CostModel(pair_fwd_s=1.0, pair_bwd_s=0.0, dense_fwd_s=0.0, dense_bwd_s=0.0, hbm_bytes_s=1.0,
                  gemm_launch_s=3.0, weight_stream_bytes_s=2.0)
    # fixed: forward 2 * (3 + 2*d*f/2) = 2 * (3 + 512) with d=2, f=256
    assert m.dense_fixed_s(2, 256, False) == 2 * (3 + 512)
    assert m.dense_fixed_s(2, 256, True) == 2 * (3 + 512) + (3 + 512) + (3 + 1024)
    st = _stats({5: 3, 12: 1}, {5: 30, 12: 40}, {5: 3, 3: 3, 12: 1, 1: 1})
    t = modelled_times(st, 2, 256, candidates=(8, 16), training=False, model=m)
    assert t[8] == 1.0 * 2 * 30 + 4 * 2 * (2 + 3 * 8) + 2 * (3 + 512)
    assert t[16] == 1.0 * 2 * 70 + 4 * 2 * (2 + 3 * 16)
    # with the measured coefficients: 4095 rows of largest count <= 8, one row at 9
    M, f, d = 4096, 8192, 2048
    st = _stats({6: 4095, 9: 1}, {6: 4095 * 82, 9: 90}, {1: M * 64})
    assert suggest_k(st, d, f, training=True)[0] == 16
    assert suggest_k(st, d, f, training=False)[0] == 16


def test_choice_from_oracle_statistics(orc):
    """End to end on the host: the oracle packs a uniform 1% batch (the uniform
    workload's shape of d_ff) in which a few rows overflow K=8 but none overflows
    K=16; its statistics make suggest_k pick 16 (the backup GEMMs' fixed cost
    outweighs the wider slots). A 4% batch, whose rows are past the break-even of a
    dense row, keeps K=8 and sends its overflowing rows dense. With a row threshold
    of 1 every row with an active unit lands in the threshold bin."""
    rng = np.random.default_rng(3)
    M, d, f = 4096, 2048, 8192
    Z = rng.standard_normal((M, f)) - 2.326  # 1% active, 1.3 per 128-wide tile
    p8, p16 = orc.pack(Z, T_n, 8), orc.pack(Z, T_n, 16)
    assert p8["n_ovf_total"] > 0 and p16["n_ovf_total"] == 0
    st = orc.count_stats(p8["count"], T_n)
    assert st["rows_by_max"][9:].sum() == p8["n_ovf_total"]
    best, times = suggest_k(st, d, f, training=True)
    assert best == 16 and times[16] < times[8]
    dense = orc.count_stats(p8["count"], T_n, dense_min=1)
    assert dense["rows_by_max"][T_n + 1] == M - int((p8["count"].sum(1) == 0).sum())
    Z4 = rng.standard_normal((512, f)) - 1.75  # 4% active: 330 per row, above the break-even
    st4 = orc.count_stats(orc.pack(Z4, T_n, 8)["count"], T_n)
    assert dense_min_for(d, f, training=True) < 330
    assert suggest_k(st4, d, f, training=True)[0] == 8
