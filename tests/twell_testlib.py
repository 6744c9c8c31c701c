"""Helpers shared by the GPU parity tests, the smoke check and the benchmark's checks.

Tolerances (bf16 inputs, fp32 accumulation) for every floating-point output,
compared with the fp64 oracle evaluated on the g values the GPU stored:
  * relative L2 error of the whole tensor <= 1e-2;
  * every element: |a - o| <= 2e-2 * rms(o) + r(o), rms over the whole tensor,
    where r(o) = |bf16(o) - o| for outputs the contract stores in bf16 (Y) and
    0 for fp32 outputs (the gradients). r is the rounding the output format
    itself imposes on that element: bf16 keeps 8 significant bits, so rounding
    the exact result alone moves an element by up to 2^-8 of its magnitude, more
    than 2e-2 * rms wherever |o| > 5.12 rms (Gaussian-like outputs of a few
    million elements reach 5.5 rms). The plain bound would fail for the exact
    result rounded to bf16, so it is read with the element's own rounding added.
These bounds apply to every workload whose tokens share one scale. Under the
heavy-tailed (lognormal) per-token scaling a row's outputs can be tens of times
the tensor's rms, and the roundings the format prescribes (stored g, stored Y)
are relative to that row's scale, so there the element bound is read per row:
|a - o| <= 2e-2 * max(rms(o), rms(o_row)) + r(o), o_row the element's row (a
token row of Y or dX, a unit row of a weight gradient); the excess over the
plain bound is reported.
Whether a unit is active and how its z rounds to bf16 are decisions the GPU
takes in fp32 (the stored g is part of the format), so the reference for these
bounds is the oracle given the g values the GPU stored (unpacked by gpu_gmat).
The plain definition (fp64 z, unrounded g, the GPU's active set) must agree to
rel-L2 <= 1e-2: its element-wise gap is the bf16 rounding of g itself, up to
2^-9 of a term, which exceeds 2e-2 * rms wherever one term dominates an
outlier element.
The gate output z that the GPU exports is compared element by element with the
oracle's fp64 z under the summation bound of fp32 arithmetic (assert_gate_close).
Packed counts, columns, values, row flags and the overflow list are compared
bit for bit with the oracle's pack of the GPU's own fp32 gate output; the GPU
active set may differ from the fp64 one only where |z| < 1e-3 * rms(z).
"""

from __future__ import annotations

import numpy as np

REL_L2 = 1e-2
MAX_ABS_RMS = 2e-2
ACTIVE_BAND = 1e-3


def to_dev(bits: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t) -> np.ndarray:
    import torch

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32_of_bits(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def state_to_numpy(st) -> dict:
    n_store, n_flag = st.n_overflow()
    return dict(count=st.count.cpu().numpy().view(np.uint16), val=bits_of(st.val), col=st.col.cpu().numpy(),
                row_ovf=st.row_ovf.cpu().numpy()[: st.M], ovf_rows=st.ovf_rows.cpu().numpy()[:n_store],
                n_ovf=n_store, n_ovf_total=n_flag, g_ovf=bits_of(st.g_ovf)[:n_store])


def assert_pack_equal(gpu: dict, ref: dict) -> None:
    """Bit-exact comparison of two packed hybrid representations."""
    for k in ("count", "val", "col", "row_ovf"):
        assert np.array_equal(gpu[k], ref[k]), f"pack field {k} differs"
    assert gpu["n_ovf_total"] == ref["n_ovf_total"], "number of overflow rows differs"
    assert gpu["n_ovf"] == ref["n_ovf"]
    n = gpu["n_ovf"]
    assert np.array_equal(gpu["ovf_rows"][:n], ref["ovf_rows"][:n]), "overflow row list differs"
    assert np.array_equal(gpu["g_ovf"][:n], ref["g_ovf"][:n]), "dense backup rows differ"


def assert_plan_valid(st, groups_hint=None) -> dict:
    """The row plan of the sparse kernels, checked on the host from the pack.

    Every non-overflow row appears as pieces q = 0..P-1 with P = max(1,
    ceil(kept / S)), rows ascending; overflow rows have no piece; S lies in
    [32, 256]; every turnstile word is back at zero between passes.
    """
    plan = st.row_plan.cpu().numpy()
    M, K = st.M, st.K
    npieces, S, total = int(plan[0]), int(plan[1]), int(plan[2])
    count = st.count.cpu().numpy().view(np.uint16).astype(np.int64)
    row_ovf = st.row_ovf.cpu().numpy()[:M]
    kept = np.minimum(count, K).sum(axis=1)
    assert 32 <= S <= 256, S
    assert total == int(kept[row_ovf == 0].sum())
    # weight gradients of the overflow rows as dense GEMMs when their P active pairs
    # over n rows satisfy the cost model P * 1000 > d_ff * (24 n + 30000)
    n_rows, pairs = int((row_ovf != 0).sum()), int(count[row_ovf != 0].sum())
    dense = n_rows > 0 and pairs * 1000 > st.d_ff * (24 * n_rows + 30000)
    assert int(plan[3]) == int(dense)
    assert not plan[4:4 + M].any(), "turnstile words must be zero between passes"
    slots = plan[4 + M:4 + 2 * M]
    want_slot = np.full(M, -1)
    ovf_list = st.ovf_rows.cpu().numpy()[:st.n_overflow()[0]]
    want_slot[ovf_list] = np.arange(ovf_list.size)
    assert np.array_equal(slots, want_slot), "row_slot: dense slot of each row"
    pieces = plan[4 + 2 * M:4 + 2 * M + 2 * npieces].reshape(-1, 2)
    want = [(r, q) for r in range(M) if not row_ovf[r]
            for q in range(max(1, -(-int(kept[r]) // S)))]
    assert [tuple(x) for x in pieces.tolist()] == want
    return dict(pieces=npieces, S=S, total=total, split_rows=int(sum(1 for r, q in want if q == 1)),
                dense_wgrad=dense)


def gpu_mask(p: dict, M: int, f: int, T_n: int, K: int) -> np.ndarray:
    """Active set [M, f] as the GPU's hybrid representation records it."""
    T = f // T_n
    mask = np.zeros((M, f), np.uint8)
    cnt = np.minimum(p["count"].astype(np.int64), K)
    ii, tt, ss = np.nonzero(np.arange(K)[None, None, :] < cnt[:, :, None])
    ell = p["row_ovf"][ii] == 0
    ii, tt, ss = ii[ell], tt[ell], ss[ell]
    mask[ii, tt * T_n + p["col"][ii, tt, ss].astype(np.int64)] = 1
    for s in range(p["n_ovf"]):
        mask[p["ovf_rows"][s]] = p["g_ovf"][s] != 0
    return mask


def gpu_gmat(p: dict, M: int, f: int, T_n: int, K: int) -> np.ndarray:
    """Dense bf16 bits [M, f] of the g values the GPU's hybrid representation stores."""
    G = np.zeros((M, f), np.uint16)
    cnt = np.minimum(p["count"].astype(np.int64), K)
    ii, tt, ss = np.nonzero(np.arange(K)[None, None, :] < cnt[:, :, None])
    ell = p["row_ovf"][ii] == 0
    ii, tt, ss = ii[ell], tt[ell], ss[ell]
    G[ii, tt * T_n + p["col"][ii, tt, ss].astype(np.int64)] = p["val"][ii, tt, ss]
    for s in range(p["n_ovf"]):
        G[p["ovf_rows"][s]] = p["g_ovf"][s]
    return G


def gpu_gmat_rows(p: dict, rows, f: int, T_n: int, K: int) -> np.ndarray:
    """gpu_gmat restricted to the listed rows ([len(rows), f] bf16 bits)."""
    rows = np.asarray(rows, np.int64)
    G = np.zeros((rows.size, f), np.uint16)
    cnt = np.minimum(p["count"][rows].astype(np.int64), K)
    rr, tt, ss = np.nonzero(np.arange(K)[None, None, :] < cnt[:, :, None])
    ell = p["row_ovf"][rows[rr]] == 0
    rr, tt, ss = rr[ell], tt[ell], ss[ell]
    G[rr, tt * T_n + p["col"][rows[rr], tt, ss].astype(np.int64)] = p["val"][rows[rr], tt, ss]
    n = p["n_ovf"]
    is_ovf = p["row_ovf"][rows] != 0
    slots = np.searchsorted(p["ovf_rows"][:n], rows[is_ovf])
    G[np.nonzero(is_ovf)[0]] = p["g_ovf"][slots]
    return G


def gpu_gmat_cols(p: dict, units, M: int, T_n: int, K: int) -> np.ndarray:
    """gpu_gmat restricted to the listed units ([M, len(units)] bf16 bits)."""
    units = np.asarray(units, np.int64)
    G = np.zeros((M, units.size), np.uint16)
    ell = p["row_ovf"][:M] == 0
    for k, j in enumerate(units):
        t, c = divmod(int(j), T_n)
        cnt = np.minimum(p["count"][:, t].astype(np.int64), K)
        hit = (np.arange(K)[None, :] < cnt[:, None]) & (p["col"][:, t, :] == c) & ell[:, None]
        ii, ss = np.nonzero(hit)
        G[ii, k] = p["val"][ii, t, ss]
    n = p["n_ovf"]
    G[p["ovf_rows"][:n]] = p["g_ovf"][:n][:, units]
    return G


def output_rounding(o: np.ndarray) -> np.ndarray:
    """|bf16(o) - o| per element: how far rounding the exact value to the bf16
    output format moves it (round to nearest even, by the oracle's rounding)."""
    from oracle import oracle as O

    o = np.asarray(o, np.float64)
    return np.abs(f32_of_bits(O.bf16_round(o)).astype(np.float64) - o)


def close_stats(a: np.ndarray, o: np.ndarray, bf16_out: bool = False, per_row: bool = False) -> dict:
    a = np.asarray(a, np.float64)
    o = np.asarray(o, np.float64)
    diff = a - o
    no = float(np.linalg.norm(o))
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    o2 = o.reshape(o.shape[0], -1) if o.ndim > 1 else o.reshape(-1, 1)
    ad = np.abs(diff.reshape(o2.shape))
    rnd = output_rounding(o2) if bf16_out and o2.size else 0.0
    plain_excess = ad - MAX_ABS_RMS * rms - rnd
    if per_row:
        row_rms = np.sqrt(np.mean(o2 * o2, axis=1, keepdims=True)) if o2.size else o2
        excess = ad - (MAX_ABS_RMS * np.maximum(rms, row_rms) + rnd)
    else:
        excess = plain_excess
    return dict(rel_l2=float(np.linalg.norm(diff)) / no if no > 0 else float(np.linalg.norm(diff)),
                max_abs=float(ad.max()) if ad.size else 0.0, rms=rms,
                worst_excess=float(excess.max()) if excess.size else 0.0,
                plain_excess=float(plain_excess.max()) if plain_excess.size else 0.0,
                max_abs_over_rms=float(ad.max() / rms) if rms > 0 and ad.size else 0.0)


def assert_close(a: np.ndarray, o: np.ndarray, name: str, bf16_out: bool = False, per_row: bool = False) -> dict:
    s = close_stats(a, o, bf16_out, per_row)
    if s["rms"] == 0.0:
        assert s["max_abs"] == 0.0, f"{name}: expected exact zeros, max abs {s['max_abs']}"
        return s
    assert s["rel_l2"] <= REL_L2, f"{name}: rel-L2 {s['rel_l2']:.3e} > {REL_L2}"
    what = "its per-row bound" if per_row else f"{MAX_ABS_RMS} x rms" + (" + its bf16 rounding" if bf16_out else "")
    assert s["worst_excess"] <= 0.0, (f"{name}: an element exceeds {what} by {s['worst_excess']:.3e} "
                                      f"(max-abs {s['max_abs']:.3e}, rms {s['rms']:.3e})")
    if per_row and s["plain_excess"] > 0.0:
        print(f"[per-row bound] {name}: max-abs / rms = {s['max_abs_over_rms']:.3e} "
              f"(plain bound exceeded by {s['plain_excess']:.3e})")
    return s


def assert_active_set(z_gpu: np.ndarray, z64: np.ndarray, rms_z: float) -> int:
    """Active sets agree except where |z| < 1e-3 rms(z). Returns the number of flips."""
    flips = (z_gpu > 0) != (z64 > 0)
    if flips.any():
        assert np.all(np.abs(z64[flips]) < ACTIVE_BAND * rms_z), "active set differs outside the rounding band"
    return int(flips.sum())


def gate_error_bound(X_bits, W_g_bits, b_g_bits, rows=None) -> np.ndarray:
    """Bound on |z_gpu - z| for the gate z_ij = sum_k x_ik W_g[j,k] + b_j computed
    with fp32 additions: the products of bf16 values are exact in fp32, and any
    order of d additions, each rounded (to nearest or toward zero) with relative
    error at most u = 2^-23, is off by at most gamma_d * sum_k |x_ik W_g[j,k]|;
    the bias addition adds u |z|. With d <= 16384, (d + 1) u < 0.002, so
    (d + 2) u (sum_k |x_ik W_g[j,k]| + |b_j|) covers both. [len(rows) or M, d_ff]."""
    X = f32_of_bits(np.asarray(X_bits) if rows is None else np.asarray(X_bits)[rows]).astype(np.float64)
    W = f32_of_bits(W_g_bits).astype(np.float64)
    b = f32_of_bits(b_g_bits).astype(np.float64)
    d = X.shape[1]
    return (d + 2) * 2.0 ** -23 * (np.abs(X) @ np.abs(W).T + np.abs(b)[None, :])


def assert_gate_close(z_gpu: np.ndarray, z64: np.ndarray, bound: np.ndarray) -> float:
    """Element-wise gate check; returns max |dz| / bound (<= 1)."""
    err = np.abs(np.asarray(z_gpu, np.float64) - z64)
    ratio = float((err / bound).max()) if err.size else 0.0
    assert ratio <= 1.0, f"gate z exceeds the fp32 summation bound (max |dz| / bound = {ratio:.3e})"
    return ratio


def assert_matches_oracle(a: np.ndarray, o_stored_g: np.ndarray, o_plain: np.ndarray, name: str,
                          bf16_out: bool = False, per_row: bool = False) -> dict:
    """Both bounds against the oracle on stored g; rel-L2 against the unrounded definition."""
    st = assert_close(a, o_stored_g, name, bf16_out, per_row)
    p = close_stats(a, o_plain, bf16_out, per_row)
    if p["rms"] > 0:
        assert p["rel_l2"] <= REL_L2, f"{name}: rel-L2 vs unrounded-g definition {p['rel_l2']:.3e} > {REL_L2}"
    st["rel_l2_plain"] = p["rel_l2"]
    return st
