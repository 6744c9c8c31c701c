"""Pins of the fp64 CPU oracle against things other than itself.

Each check ties one oracle function to the mathematics or to an independent
library routine: brute-force loops on tiny inputs, torch float64 matmuls and
autograd, a hand-built packing known by construction, closed forms of special
cases, and format invariants. A dropped term, a wrong sign, a transposed operand
or a wrong slot order in the oracle fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

from synthetic import bf16_bits_from_f64, bf16_bits_to_f32


def _rand_bf16(rng, shape, scale=1.0):
    return bf16_bits_from_f64(rng.standard_normal(shape) * scale)


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _problem(seed, M, d, f, bias):
    rng = np.random.default_rng(seed)
    X = _rand_bf16(rng, (M, d))
    Wg = _rand_bf16(rng, (f, d), 1 / math.sqrt(d))
    Wu = _rand_bf16(rng, (f, d), 1 / math.sqrt(d))
    Wd = _rand_bf16(rng, (d, f), 1 / math.sqrt(f))
    bg = bf16_bits_from_f64(np.full(f, bias))
    dY = _rand_bf16(rng, (M, d))
    return X, Wg, bg, Wu, Wd, dY


def _torch_ffn(X, Wg, bg, Wu, Wd, lam=0.0, dY=None):
    t = lambda a: torch.tensor(_f64(a), dtype=torch.float64, requires_grad=True)  # noqa: E731
    x, wg, b, wu, wd = t(X), t(Wg), t(bg), t(Wu), t(Wd)
    z = x @ wg.T + b
    g = torch.relu(z)
    y = (g * (x @ wu.T)) @ wd.T
    out = dict(Y=y.detach().numpy(), Z=z.detach().numpy())
    if dY is not None:
        loss = (y * torch.tensor(_f64(dY), dtype=torch.float64)).sum() + lam * g.sum()
        loss.backward()
        out.update(dX=x.grad.numpy(), dW_g=wg.grad.numpy(), dW_u=wu.grad.numpy(), dW_d=wd.grad.numpy(),
                   db_g=b.grad.numpy())
    return out


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ------------------------------------------------------------------ bfloat16


def test_bf16_round_matches_torch_cast(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # binary32 subnormals
        (rng.standard_normal(2000) * 1e37).astype(np.float32),
        # exact halfway cases: low 16 bits 0x8000, both parities of the kept bit
        (rng.integers(0x0080, 0x7F00, 4000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ])
    vals = np.concatenate([vals, -vals])
    ours = orc.bf16_round(vals.astype(np.float64))
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_round_double_inputs_by_hand(orc):
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0).
    assert orc.bf16_round([1.0 + 2.0**-8])[0] == 0x3F80
    # (1 + 2^-7) + 2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): rounds up.
    assert orc.bf16_round([1.0 + 2.0**-7 + 2.0**-8])[0] == 0x3F82
    # a hair above the first tie (not representable in binary32) rounds up.
    assert orc.bf16_round([1.0 + 2.0**-8 + 2.0**-40])[0] == 0x3F81
    assert orc.bf16_round([-(1.0 + 2.0**-8 + 2.0**-40)])[0] == 0xBF81
    assert orc.bf16_round([0.0])[0] == 0x0000 and orc.bf16_round([-0.0])[0] == 0x8000
    # largest finite bf16 and overflow to infinity
    assert orc.bf16_round([(2 - 2.0**-7) * 2.0**127])[0] == 0x7F7F
    assert orc.bf16_round([2.0**128])[0] == 0x7F80
    # smallest subnormal 2^-133, and half of it (a tie with 0, goes to 0)
    assert orc.bf16_round([2.0**-133])[0] == 0x0001
    assert orc.bf16_round([2.0**-134])[0] == 0x0000
    assert orc.bf16_round([1.5 * 2.0**-134 * 2])[0] == 0x0002  # 3 * 2^-134 = 1.5 ulp -> 2 ulp (even)
    b = np.arange(0, 0x7F80, 7, dtype=np.uint16)
    assert np.array_equal(orc.bf16_round(orc.bf16_to_f64(b)), b)


# ----------------------------------------------------------------------- gate


def test_gate_brute_force(orc):
    X, Wg, bg, *_ = _problem(2, 3, 8, 16, -0.25)
    Z = orc.gate(X, Wg, bg)
    x, w, b = _f64(X), _f64(Wg), _f64(bg)
    for i, j in itertools.product(range(3), range(16)):
        s = 0.0
        for k in range(8):
            s += x[i, k] * w[j, k]
        assert Z[i, j] == pytest.approx(s + b[j], rel=1e-14, abs=1e-14)


def test_gate_torch_and_rows(orc):
    X, Wg, bg, *_ = _problem(3, 40, 96, 384, 0.1)
    Z = orc.gate(X, Wg, bg)
    ref = _f64(X) @ _f64(Wg).T + _f64(bg)
    assert np.abs(Z - ref).max() < 1e-12
    rows = np.array([39, 0, 17], np.int32)
    assert np.array_equal(orc.gate(X, Wg, bg, rows=rows), Z[rows])


# ----------------------------------------------------------------------- pack


def test_pack_hand_built_identity_gate(orc):
    """W_g = I, b = 0 gives z = X exactly, so the packing is known by construction."""
    d = f = 256
    T_n, K = 128, 8
    Xv = np.zeros((4, d))
    Xv[0, [3, 7, 130]] = [1.5, 2.0, 0.75]
    Xv[0, [5, 200]] = [-1.0, -3.0]
    ten = [0, 1, 2, 10, 20, 30, 40, 50, 60, 127]               # 10 > K actives in tile 0 of row 1
    Xv[1, ten] = np.arange(1, 11, dtype=np.float64)
    Xv[1, 128 + 5] = 4.0
    Xv[2, :] = -1.0
    Xv[2, 9] = 0.0                                              # z == 0 is inactive
    Xv[3, 255] = 0.5
    X = bf16_bits_from_f64(Xv)
    Wg = bf16_bits_from_f64(np.eye(f, d))
    bg = np.zeros(f, np.uint16)
    Z = orc.gate(X, Wg, bg)
    assert np.array_equal(Z, _f64(X))
    p = orc.pack(Z, T_n, K)
    one = lambda v: int(bf16_bits_from_f64(np.array([v]))[0])  # noqa: E731

    assert p["count"].tolist() == [[2, 1], [10, 1], [0, 0], [0, 1]]
    assert p["col"][0, 0].tolist() == [3, 7, 0, 0, 0, 0, 0, 0]
    assert p["val"][0, 0].tolist() == [one(1.5), one(2.0), 0, 0, 0, 0, 0, 0]
    assert p["col"][0, 1].tolist() == [2, 0, 0, 0, 0, 0, 0, 0]
    assert p["val"][0, 1].tolist()[0] == one(0.75)
    assert p["col"][1, 0].tolist() == ten[:8]                   # first K in ascending column order
    assert p["val"][1, 0].tolist() == [one(v) for v in range(1, 9)]
    assert p["col"][1, 1].tolist()[0] == 5
    assert not p["val"][2].any() and not p["col"][2].any()
    assert p["col"][3, 1].tolist()[0] == 127
    assert p["row_ovf"].tolist() == [0, 1, 0, 0]
    assert p["n_ovf"] == 1 and p["ovf_rows"][:1].tolist() == [1]
    expect_row1 = np.zeros(f)
    expect_row1[ten] = np.arange(1, 11)
    expect_row1[133] = 4.0
    assert np.array_equal(p["g_ovf"][0], bf16_bits_from_f64(expect_row1))


@pytest.mark.parametrize("T_n,K", [(128, 8), (128, 16), (64, 4), (256, 8), (256, 256), (128, 128)])
def test_pack_roundtrip_and_invariants(orc, T_n, K):
    rng = np.random.default_rng(T_n + K)
    M, f = 37, 1024
    # heavy-tailed activity: a few rows dense enough to overflow
    Z = rng.standard_normal((M, f)) * np.exp(0.9 * rng.standard_normal((M, 1))) - 2.0
    Z[5, :] = 0.0
    p = orc.pack(Z, T_n, K)
    T = f // T_n
    # round trip to the dense bf16 ReLU
    G = orc.unpack(p, f, T_n, K)
    assert np.array_equal(G, orc.bf16_round(np.maximum(Z, 0.0) + 0.0))
    # counts by a different route
    cnt = (Z.reshape(M, T, T_n) > 0).sum(-1)
    assert np.array_equal(p["count"], cnt)
    assert p["count"].sum() == (Z > 0).sum()
    assert (p["count"] <= T_n).all()
    # slots: columns strictly ascending and < T_n, padding is (0, 0)
    for i in range(M):
        for t in range(T):
            n = min(int(p["count"][i, t]), K)
            c = p["col"][i, t, :n].astype(int)
            assert (np.diff(c) > 0).all() and (c < T_n).all()
            assert not p["col"][i, t, n:].any() and not p["val"][i, t, n:].any()
            assert (Z[i, t * T_n + c] > 0).all()
    # row routing and its order
    assert np.array_equal(p["row_ovf"].astype(bool), (cnt > K).any(1))
    rows = np.nonzero(cnt.max(1) > K)[0]
    assert p["n_ovf"] == rows.size and np.array_equal(p["ovf_rows"][: rows.size], rows)
    if K >= T_n:
        assert p["n_ovf"] == 0
    # with a row threshold, rows of many actives also go dense; same round trip
    dm = int(np.median(cnt.sum(1))) + 1
    q = orc.pack(Z, T_n, K, dense_min=dm)
    want = (cnt > K).any(1) | (cnt.sum(1) >= dm)
    assert np.array_equal(q["row_ovf"].astype(bool), want) and want.sum() > (cnt > K).any(1).sum() - 1
    assert np.array_equal(q["ovf_rows"][:q["n_ovf"]], np.nonzero(want)[0])
    assert np.array_equal(orc.unpack(q, f, T_n, K), G)
    for k in ("count", "val", "col"):
        assert np.array_equal(q[k], p[k])


def test_pack_single_tile_is_row_ellpack(orc):
    rng = np.random.default_rng(9)
    Z = rng.standard_normal((5, 64)) - 1.0
    p = orc.pack(Z, 64, 64)
    for i in range(5):
        nz = np.nonzero(Z[i] > 0)[0]
        assert p["count"][i, 0] == nz.size
        assert np.array_equal(p["col"][i, 0, : nz.size], nz)
        assert np.array_equal(p["val"][i, 0, : nz.size], orc.bf16_round(Z[i, nz]))


def test_pack_rejects_unpackable_shapes(orc):
    Z = np.ones((2, 1024))
    for T_n, K in [(512, 8), (1024, 64), (96, 8), (128, 0)]:
        with pytest.raises(ValueError):
            orc.pack(Z, T_n, K)


def test_pack_capacity(orc):
    Z = np.ones((6, 256))
    Z[2] = -1
    p = orc.pack(Z, 128, 8, cap=3)
    assert p["status"] == 3 and p["n_ovf_total"] == 5 and p["n_ovf"] == 3
    assert p["ovf_rows"].tolist() == [0, 1, 3]


# -------------------------------------------------------------------- forward


def test_fwd_brute_force(orc):
    X, Wg, bg, Wu, Wd, _ = _problem(4, 3, 8, 16, 0.05)
    Y = orc.ffn_fwd(X, Wg, bg, Wu, Wd)
    x, wg, b, wu, wd = map(_f64, (X, Wg, bg, Wu, Wd))
    for i in range(3):
        for c in range(8):
            acc = 0.0
            for j in range(16):
                z = sum(x[i, k] * wg[j, k] for k in range(8)) + b[j]
                if z > 0:
                    u = sum(x[i, k] * wu[j, k] for k in range(8))
                    acc += z * u * wd[c, j]
            assert Y[i, c] == pytest.approx(acc, rel=1e-12, abs=1e-14)


@pytest.mark.parametrize("bias", [-2.0, 0.0, 1.0])
def test_fwd_torch(orc, bias):
    X, Wg, bg, Wu, Wd, _ = _problem(5, 33, 64, 256, bias)
    Y = orc.ffn_fwd(X, Wg, bg, Wu, Wd)
    ref = _torch_ffn(X, Wg, bg, Wu, Wd)["Y"]
    assert _rel(Y, ref) < 1e-12
    rows = np.array([32, 1, 7], np.int32)
    assert np.array_equal(orc.ffn_fwd(X, Wg, bg, Wu, Wd, rows=rows), Y[rows])


def test_fwd_special_cases(orc):
    X, Wg, _, Wu, Wd, _ = _problem(6, 9, 32, 128, 0.0)
    f = 128
    # nothing active: Y == 0 exactly
    neg = bf16_bits_from_f64(np.full(f, -1e4))
    assert not orc.ffn_fwd(X, Wg, neg, Wu, Wd).any()
    # everything active: ReLU is the identity, a plain bilinear product (torch)
    pos = bf16_bits_from_f64(np.full(f, 1e4))
    x, wg, wu, wd, b = map(_f64, (X, Wg, Wu, Wd, pos))
    full = ((x @ wg.T + b) * (x @ wu.T)) @ wd.T
    assert _rel(orc.ffn_fwd(X, Wg, pos, Wu, Wd), full) < 1e-12
    # exactly one active unit j: y = (x.w_g[j] + b_j)(x.w_u[j]) W_d[:, j]
    j = 37
    bv = np.full(f, -1e4)
    bv[j] = 64.0
    one = bf16_bits_from_f64(bv)
    Y = orc.ffn_fwd(X, Wg, one, Wu, Wd)
    closed = np.outer((x @ wg[j] + 64.0) * (x @ wu[j]), wd[:, j])
    assert _rel(Y, closed) < 1e-13


def test_fwd_mask_override(orc):
    X, Wg, bg, Wu, Wd, _ = _problem(7, 12, 32, 256, -0.5)
    Z = orc.gate(X, Wg, bg)
    mask = (Z > 0).astype(np.uint8)
    Y = orc.ffn_fwd(X, Wg, bg, Wu, Wd)
    assert np.array_equal(orc.ffn_fwd(X, Wg, bg, Wu, Wd, mask=mask), Y)
    # flip one unit on: the definition evaluated with that active set (torch, masked)
    i, j = 3, int(np.argmin(Z[3]))
    mask[i, j] = 1
    x, wg, b, wu, wd = map(_f64, (X, Wg, bg, Wu, Wd))
    z = x @ wg.T + b
    ref = ((z * mask) * (x @ wu.T)) @ wd.T
    assert _rel(orc.ffn_fwd(X, Wg, bg, Wu, Wd, mask=mask), ref) < 1e-12


@pytest.mark.parametrize("K", [2, 8, 128])
def test_hybrid_equals_dense(orc, K):
    """Sparse (ELL rows + dense backup rows) equals the dense definition on bf16(g)."""
    rng = np.random.default_rng(K)
    M, d, f = 24, 64, 512
    X, Wg, bg, Wu, Wd, _ = _problem(K, M, d, f, -1.0)
    X = bf16_bits_from_f64(_f64(X) * np.exp(0.8 * rng.standard_normal((M, 1))))
    Z = orc.gate(X, Wg, bg)
    p = orc.pack(Z, 128, K)
    if K == 2:
        assert 0 < p["n_ovf"] < M
    Yh = orc.ffn_fwd_hybrid(X, Wu, Wd, p, 128, K)
    Yd = orc.ffn_fwd(X, Wg, bg, Wu, Wd, round_g=True)
    assert _rel(Yh, Yd) < 1e-12
    # and rounding g changes the result by about one bf16 half-ulp, not more
    assert _rel(Yd, orc.ffn_fwd(X, Wg, bg, Wu, Wd)) < 4e-3


# ------------------------------------------------------------------- backward


@pytest.mark.parametrize("lam", [0.0, 0.3])
@pytest.mark.parametrize("bias", [-0.7, 0.4])
def test_bwd_torch_autograd(orc, lam, bias):
    X, Wg, bg, Wu, Wd, dY = _problem(11, 10, 32, 128, bias)
    g = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, lam)
    ref = _torch_ffn(X, Wg, bg, Wu, Wd, lam, dY)
    for k in ("dX", "dW_g", "dW_u", "dW_d", "db_g"):
        assert _rel(g[k], ref[k]) < 1e-11, k


def test_bwd_l1_closed_form(orc):
    """With dY = 0 only the L1 term remains: dZ = lambda on active units."""
    X, Wg, bg, Wu, Wd, _ = _problem(12, 14, 32, 256, -0.3)
    dY = np.zeros((14, 32), np.uint16)
    lam = 0.125
    g = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, lam)
    act = (orc.gate(X, Wg, bg) > 0).astype(np.float64)
    x, wg = _f64(X), _f64(Wg)
    assert np.allclose(g["db_g"], lam * act.sum(0), rtol=0, atol=1e-12)
    assert _rel(g["dW_g"], lam * act.T @ x) < 1e-13
    assert _rel(g["dX"], lam * act @ wg) < 1e-13
    assert not g["dW_u"].any() and not g["dW_d"].any()


def test_bwd_special_and_mask(orc):
    X, Wg, bg, Wu, Wd, dY = _problem(13, 8, 32, 128, -0.4)
    neg = bf16_bits_from_f64(np.full(128, -1e4))
    g0 = orc.ffn_bwd(X, Wg, neg, Wu, Wd, dY, 0.5)
    assert all(not g0[k].any() for k in g0)
    mask = (orc.gate(X, Wg, bg) > 0).astype(np.uint8)
    a = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, 0.01)
    b = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, 0.01, mask=mask)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_gmat_input_equals_stored_g_definition(orc):
    """g given explicitly (the packed, bf16-rounded ReLU(z)) reproduces round_g exactly,
    and a perturbed g moves the result the way the definition says."""
    rng = np.random.default_rng(21)
    X, Wg, bg, Wu, Wd, dY = _problem(21, 16, 64, 256, -0.6)
    Z = orc.gate(X, Wg, bg)
    G = orc.unpack(orc.pack(Z, 128, 8), 256, 128, 8)
    assert np.array_equal(orc.ffn_fwd(X, Wg, bg, Wu, Wd, gmat=G), orc.ffn_fwd(X, Wg, bg, Wu, Wd, round_g=True))
    a = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, 0.01, gmat=G)
    b = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, 0.01, round_g=True)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    # doubling one stored g doubles that unit's contribution to Y (torch, float64)
    i, j = [int(v) for v in np.argwhere(G != 0)[0]]
    G2 = G.copy()
    G2[i, j] = bf16_bits_from_f64(2 * _f64(G[i:i + 1, j:j + 1]))[0, 0]
    x, wu, wd = _f64(X), _f64(Wu), _f64(Wd)
    delta = _f64(G[i:i + 1, j:j + 1])[0, 0] * (x[i] @ wu[j]) * wd[:, j]
    y1 = orc.ffn_fwd(X, Wg, bg, Wu, Wd, gmat=G)
    y2 = orc.ffn_fwd(X, Wg, bg, Wu, Wd, gmat=G2)
    assert np.abs(y2[i] - y1[i] - delta).max() < 1e-12
    rows = np.array([3, 0], np.int32)
    assert np.array_equal(orc.ffn_fwd(X, Wg, bg, Wu, Wd, rows=rows, gmat=G[rows]), y1[rows])


def test_bwd_units_equals_full_backward(orc):
    """ffn_bwd_units (the weight gradients of listed units, numpy) against the C
    oracle's full backward given the same stored g: the same numbers to rounding
    order, for units active in many rows, in one row and in none, and lambda != 0;
    and a unit's gradients move by the definition when its g doubles in one row."""
    X, Wg, bg, Wu, Wd, dY = _problem(31, 40, 64, 256, -0.5)
    Z = orc.gate(X, Wg, bg)
    G = orc.unpack(orc.pack(Z, 128, 8), 256, 128, 8)
    G[:, 7] = 0           # a unit active nowhere
    G[1:, 9] = 0          # a unit active in row 0 only (if at all)
    full = orc.ffn_bwd(X, Wg, bg, Wu, Wd, dY, 0.03, gmat=G)
    units = np.array([0, 5, 7, 9, 130, 255])
    part = orc.ffn_bwd_units(X, Wu, Wd, dY, 0.03, units, G[:, units])
    for k in ("dW_g", "dW_u"):
        ref = full[k][units]
        assert np.abs(part[k] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), k
    ref = full["dW_d"][:, units]
    assert np.abs(part["dW_d"] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    assert np.abs(part["db_g"] - full["db_g"][units]).max() <= 1e-12 * max(1.0, np.abs(full["db_g"]).max())
    assert not part["dW_u"][2].any() and part["db_g"][2] == 0.0
    # doubling g_ij doubles row i's term of dW_u[j] (dU = dH g) and of dW_d[:, j] (h = g u)
    i = int(np.nonzero(G[:, 5])[0][0])
    G2 = G.copy()
    G2[i, 5] = bf16_bits_from_f64(2 * _f64(G[i:i + 1, 5:6]))[0, 0]
    a = orc.ffn_bwd_units(X, Wu, Wd, dY, 0.03, [5], G[:, [5]])
    b = orc.ffn_bwd_units(X, Wu, Wd, dY, 0.03, [5], G2[:, [5]])
    x, wu, wd, dy = _f64(X), _f64(Wu), _f64(Wd), _f64(dY)
    gij = _f64(G[i:i + 1, 5:6])[0, 0]
    dh = dy[i] @ wd[:, 5]
    assert np.abs((b["dW_u"][0] - a["dW_u"][0]) - dh * gij * x[i]).max() < 1e-10
    assert np.abs((b["dW_d"][:, 0] - a["dW_d"][:, 0]) - gij * (x[i] @ wu[5]) * dy[i]).max() < 1e-10
    assert np.abs(b["dW_g"] - a["dW_g"]).max() == 0.0  # dZ does not depend on g's value


def test_count_stats_hand_counted(orc):
    """Bins counted by hand for a 3-row, 2-tile batch with T_n = 4."""
    count = np.array([[1, 3], [0, 0], [4, 2]], dtype=np.uint16)
    st = orc.count_stats(count, 4)
    # largest tile counts 3, 0, 4; row sums 4, 0, 6; tile counts 1, 3, 0, 0, 4, 2
    assert st["rows_by_max"].tolist() == [1, 0, 0, 1, 1, 0]
    assert st["act_by_max"].tolist() == [0, 0, 0, 4, 6, 0]
    assert st["tiles_by_count"].tolist() == [2, 1, 1, 1, 1, 0]
    # rows with at least 5 active units (the third, 6) go to the last bin
    st = orc.count_stats(count, 4, dense_min=5)
    assert st["rows_by_max"].tolist() == [1, 0, 0, 1, 0, 1]
    assert st["act_by_max"].tolist() == [0, 0, 0, 4, 0, 6]
    assert st["tiles_by_count"].tolist() == [2, 1, 1, 1, 1, 0]
    empty = orc.count_stats(np.zeros((0, 5), np.uint16), 128)
    assert all(v.shape == (130,) and not v.any() for v in empty.values())
    with pytest.raises(ValueError):
        orc.count_stats(np.array([[5]], np.uint16), 4)


def test_count_stats_brute_force_and_sums(orc):
    """Plain loops over rows and tiles on random counts, plus the sum identities
    (rows, actives and tiles are each counted once) and the link to routing:
    the rows of bins above K are exactly the rows the oracle's pack routes to
    the dense backup."""
    rng = np.random.default_rng(11)
    M, T, T_n = 57, 6, 128
    count = np.minimum(rng.geometric(0.3, size=(M, T)) - 1 + (rng.random((M, T)) < 0.05) * 40, T_n).astype(np.uint16)
    for dense_min in (0, 40):
        st = orc.count_stats(count, T_n, dense_min)
        rows = [0] * (T_n + 2)
        act = [0] * (T_n + 2)
        tiles = [0] * (T_n + 2)
        for i in range(M):
            m = 0
            s = 0
            for t in range(T):
                c = int(count[i, t])
                tiles[c] += 1
                m = max(m, c)
                s += c
            if dense_min and s >= dense_min:
                m = T_n + 1
            rows[m] += 1
            act[m] += s
        assert st["rows_by_max"].tolist() == rows
        assert st["act_by_max"].tolist() == act
        assert st["tiles_by_count"].tolist() == tiles
        assert st["rows_by_max"].sum() == M and st["tiles_by_count"].sum() == M * T
        assert st["act_by_max"].sum() == count.astype(np.int64).sum()
        assert (np.arange(T_n + 2) * st["tiles_by_count"]).sum() == count.astype(np.int64).sum()
    assert 0 < st["rows_by_max"][T_n + 1] < M  # the threshold splits this batch
    # a dense Z whose tile counts are `count`: the first c columns of each tile positive
    Z = -np.ones((M, T * T_n))
    for i in range(M):
        for t in range(T):
            Z[i, t * T_n:t * T_n + int(count[i, t])] = 1.0
    for K in (8, 16, 32):
        for dense_min in (0, 40):
            st = orc.count_stats(count, T_n, dense_min)
            p = orc.pack(Z, T_n, K, dense_min=dense_min)
            assert np.array_equal(p["count"], count)
            assert p["n_ovf_total"] == st["rows_by_max"][K + 1:].sum()
            flagged = (count.max(axis=1) > K) | ((count.astype(np.int64).sum(axis=1) >= dense_min) & (dense_min > 0))
            assert np.array_equal(p["row_ovf"].astype(bool), flagged)
            assert np.array_equal(p["ovf_rows"][:p["n_ovf"]], np.flatnonzero(flagged))


# ------------------------------------------------------------- 8-bit weights


def test_e4m3_values_match_torch(orc):
    """All 256 E4M3 codes read as torch's float8_e4m3fn reads them (NaN codes aside)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = orc.e4m3_value(c)
        if c & 0x7F == 0x7F:
            assert math.isnan(v) and math.isnan(ref[c])
        else:
            assert v == ref[c] and math.copysign(1.0, v) == math.copysign(1.0, ref[c]), c
    # the grid's landmarks
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9 and orc.e4m3_value(0x08) == 2.0 ** -6


def _nearest_code(x, values):
    """Brute force: the finite code nearest to x; on a tie the one with the even mantissa."""
    best = None
    for c, v in values:
        dist = abs(v - x)
        if best is None or dist < best[0] or (dist == best[0] and (c & 1) == 0 and (best[1] & 1) == 1):
            best = (dist, c)
    return best[1]


def test_e4m3_round_brute_force_and_torch(orc):
    """Nearest-even rounding to E4M3 against a brute-force search over the finite
    codes (with both signs, ties, subnormals, the binade edges) and against torch's
    float64 -> float8_e4m3fn cast."""
    finite = [(c, orc.e4m3_value(c)) for c in range(256) if c & 0x7F != 0x7F]
    pos = sorted({v for _, v in finite if v > 0})
    xs = [0.0, 448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -6, 1.0, 1.0625, 1.1875, 15.5, 240.0, 232.0,
          447.0, 2.0 ** -7 * 0.99]
    xs += [(a + b) / 2 for a, b in zip(pos, pos[1:])]  # every tie between neighbours
    rng = np.random.default_rng(3)
    xs += list(rng.uniform(0, 448, 400)) + list(np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448), 400)))
    for x in xs:
        for sx in (x, -x):
            got = orc.e4m3_round(sx)
            want = _nearest_code(sx, [(c, v) for c, v in finite if (v > 0) == (sx > 0) or v == 0])
            assert orc.e4m3_value(got) == orc.e4m3_value(want), (sx, got, want)
    t = torch.tensor(xs + [-x for x in xs], dtype=torch.float64)
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_round(float(v)) for v in t], np.uint8)
    assert np.array_equal(np.vectorize(orc.e4m3_value)(got), np.vectorize(orc.e4m3_value)(ref))
    assert orc.e4m3_round(500.0) == 0x7E and orc.e4m3_round(-1e9) == 0xFE


def test_quantize_units_scale_round_trip_idempotence(orc):
    """Per unit: amax <= 448 * 2^e < 2 * amax (the smallest such e); the dequantised
    weights are bf16 values equal to value(q) * 2^e; quantising them again gives the
    same codes and exponents; the two layouts (units as rows / columns) agree."""
    rng = np.random.default_rng(11)
    W = _rand_bf16(rng, (37, 96), 1 / math.sqrt(96))
    W[5] = 0  # a zero unit
    W[6, :] = bf16_bits_from_f64(np.linspace(-3.0, 5.0, 96))  # a wider range
    r = orc.quantize_e4m3(W, unit_axis=0)
    q, e, deq = r["q"], r["exp"], r["deq"]
    vals = np.vectorize(orc.e4m3_value)(q)
    Wf = _f64(W)
    for j in range(W.shape[0]):
        amax = np.abs(Wf[j]).max()
        if amax == 0:
            assert e[j] == 0 and not q[j].any() and not deq[j].any()
            continue
        assert amax <= 448.0 * 2.0 ** e[j] and amax > 448.0 * 2.0 ** (e[j] - 1)
        np.testing.assert_array_equal(_f64(deq[j]), vals[j] * 2.0 ** e[j])
        # each code is the nearest grid point of the scaled weight
        assert np.all(np.abs(vals[j] - Wf[j] / 2.0 ** e[j]) <= np.abs(
            np.vectorize(orc.e4m3_value)((q[j] ^ 1) & 0xFF) - Wf[j] / 2.0 ** e[j]) + 1e-300)
    again = orc.quantize_e4m3(deq, unit_axis=0)
    assert np.array_equal(again["q"], q) and np.array_equal(again["exp"], e) and np.array_equal(again["deq"], deq)
    cols = orc.quantize_e4m3(np.ascontiguousarray(W.T), unit_axis=1)
    assert np.array_equal(cols["q"], q) and np.array_equal(cols["exp"], e)
    assert np.array_equal(cols["deq"], np.ascontiguousarray(deq.T))


def test_quantize_grid_unit_is_exact(orc):
    """A unit whose weights already lie on the E4M3 grid times a power of two (with
    the largest one at 448 * 2^e) comes back unchanged."""
    e = -7
    codes = np.array([0x7E, 0x01, 0x38, 0xBA, 0x08, 0x00, 0x55, 0xD0], np.uint8)
    vals = np.array([orc.e4m3_value(c) for c in codes]) * 2.0 ** e
    W = bf16_bits_from_f64(vals)[None, :]
    r = orc.quantize_e4m3(W, unit_axis=0)
    assert r["exp"][0] == e
    assert np.array_equal(np.vectorize(orc.e4m3_value)(r["q"][0]) * 2.0 ** e, vals)
    assert np.array_equal(r["deq"], W)
