"""The seeded workload generator: determinism, rounding, and calibrated activity."""

import json
import os

import numpy as np
import pytest
import torch

import synthetic.workloads as W
from synthetic import WORKLOADS, Workload, bf16_bits_from_f64, gate_bias_for_activity, make_inputs, sweep_k

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_deterministic_and_stream_independent():
    w = Workload("t", 40, 64, 256, 128, 8, 0.05, training=True)
    a = make_inputs(w, seed=3)
    b = make_inputs(w, seed=3)
    c = make_inputs(w, seed=3, with_dY=False)
    for k in ("X", "W_g", "b_g", "W_u", "W_d"):
        assert np.array_equal(a[k], b[k]) and np.array_equal(a[k], c[k])
    assert np.array_equal(a["dY"], b["dY"]) and "dY" not in c
    d = make_inputs(w, seed=4)
    assert not np.array_equal(a["X"], d["X"])
    shapes = dict(X=(40, 64), W_g=(256, 64), b_g=(256,), W_u=(256, 64), W_d=(64, 256), dY=(40, 64))
    for k, s in shapes.items():
        assert a[k].shape == s and a[k].dtype == np.uint16


def test_chunked_draw_matches_single_draw(monkeypatch):
    w = Workload("t", 37, 32, 128, 128, 8, 0.05, row_scale="lognormal")
    whole = make_inputs(w, seed=5)
    monkeypatch.setattr(W, "_ROW_CHUNK", 5)
    chunked = make_inputs(w, seed=5)
    for k in ("X", "W_g", "W_u", "W_d"):
        assert np.array_equal(whole[k], chunked[k])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = rng.standard_normal(100000) * np.exp(3 * rng.standard_normal(100000))
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits_from_f64(a), ref)


def test_bias_values():
    assert gate_bias_for_activity(0.01) == pytest.approx(-2.3263, abs=1e-3)
    assert gate_bias_for_activity(0.03) == pytest.approx(-1.8808, abs=1e-3)
    b = gate_bias_for_activity(0.01, "lognormal", 0.75)
    assert -5.5 < b < -4.8
    assert sweep_k(0.10) == 64 and sweep_k(0.05) == 32 and sweep_k(0.01) == 8 and sweep_k(0.001) == 8


def test_calibrated_activity_tiny(orc):
    inp = make_inputs(WORKLOADS["tiny"])
    z = orc.gate(inp["X"], inp["W_g"], inp["b_g"])
    assert 0.025 < (z > 0).mean() < 0.035


def test_calibrated_activity_uniform_proxy(orc):
    w = Workload("proxy", 512, 2048, 2048, 128, 8, 0.01)
    inp = make_inputs(w, seed=1)
    z = orc.gate(inp["X"], inp["W_g"], inp["b_g"])
    assert 0.009 < (z > 0).mean() < 0.011


def test_calibrated_activity_heavy_tail_proxy(orc):
    """Lognormal row scale: ~1% mean activity with a max/mean count per row-tile >= 10."""
    w = Workload("proxy", 4096, 512, 1024, 128, 8, 0.01, row_scale="lognormal")
    inp = make_inputs(w, seed=2)
    z = orc.gate(inp["X"], inp["W_g"], inp["b_g"])
    act = (z > 0).mean()
    assert 0.008 < act < 0.012
    cnt = (z.reshape(4096, 8, 128) > 0).sum(-1)
    assert cnt.max() / cnt.mean() >= 10


def test_uniform_seed_file():
    with open(os.path.join(GOLDEN, "uniform_seed.json")) as fh:
        g = json.load(fh)
    w = WORKLOADS["uniform"]
    assert (g["M"], g["d_model"], g["d_ff"], g["T_n"], g["K"]) == (w.M, w.d_model, w.d_ff, w.T_n, w.K)
    assert g["seeds_tried"][-1]["seed"] == g["seed"] and g["seeds_tried"][-1]["n_ovf"] == 0
    assert all(s["n_ovf"] > 0 for s in g["seeds_tried"][:-1])
