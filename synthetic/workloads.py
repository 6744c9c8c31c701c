"""Seeded input recipes for the activation-sparse gated FFN (TwELL) workloads.

The pages describing TwELL ("Sakana AI и NVIDIA представили TwELL — формат и
CUDA-ядра, превращающие активную разреженность в реальные ускорения LLM",
paragraphs 1 and 3) characterise the regime only as batched, thousands-of-token
GEMMs over multi-billion-parameter LLM FFN blocks whose hidden units are more
than 99% zero after L1 training. No dataset or trained weights exist here, so
every tensor is drawn from a seeded generator with the shapes of the five
workload rows below:

* X    ~ N(0, 1) per element, optionally scaled per token by s_i ~ lognormal(0, sigma)
* W_g, W_u ~ N(0, 1/d_model); W_d ~ N(0, 1/d_ff)  (fan-in scaling)
* dY   ~ N(0, 1)
* b_g  = one constant, set so that P(z > 0) equals the target activity p for the
         distribution z0 = x . w_g that these draws induce (see gate_bias_for_activity)

Every value is drawn in float64 from numpy's PCG64, rounded to float32 (RNE) and
then to bfloat16 (RNE); arrays are returned as uint16 bit patterns. The streams
are independent children of one SeedSequence, spawned in the fixed order
X, s, W_g, W_u, W_d, dY, so adding dY never changes X or the weights.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

_STREAMS = ("X", "s", "W_g", "W_u", "W_d", "dY")
_ROW_CHUNK = 2048  # rows drawn per call; the PCG64 stream is consumed in order either way


@dataclasses.dataclass(frozen=True)
class Workload:
    """One workload shape. `activity` is the target mean fraction of active hidden units."""

    name: str
    M: int
    d_model: int
    d_ff: int
    T_n: int
    K: int
    activity: float
    row_scale: str = "none"  # "none" or "lognormal"
    sigma: float = 0.75
    training: bool = False
    seed: int = 0


WORKLOADS = {
    # tiny gated ReLU FFN forward, ~3% active units
    "tiny": Workload("tiny", 64, 256, 1024, 128, 16, 0.03),
    # inference forward, uniform i.i.d. 1% activity; seed fixed by tests/golden/select_uniform_seed.py
    "uniform": Workload("uniform", 4096, 2048, 8192, 128, 8, 0.01),
    # inference forward, heavy-tailed per-token activity (lognormal row scale)
    "heavy": Workload("heavy", 16384, 4096, 14336, 128, 8, 0.01, row_scale="lognormal"),
    # one training step of a sparse FFN layer
    "train": Workload("train", 8192, 2048, 8192, 128, 8, 0.01, training=True),
    # the largest single-GPU point of the d_model=4096, d_ff=14336 sweep at 99% sparsity,
    # run as a training step (the throughput workload of bench.py)
    "large": Workload("large", 65536, 4096, 14336, 128, 8, 0.01, row_scale="lognormal", training=True),
    # the M=8192 point of the same sweep at 99% sparsity, as a training step
    "sweep8k": Workload("sweep8k", 8192, 4096, 14336, 128, 8, 0.01, row_scale="lognormal", training=True),
    # the sweep's small batches at 99% sparsity, as training steps
    "sweep2k": Workload("sweep2k", 2048, 4096, 14336, 128, 8, 0.01, row_scale="lognormal", training=True),
    "sweep512": Workload("sweep512", 512, 4096, 14336, 128, 8, 0.01, row_scale="lognormal", training=True),
}


def sweep_k(activity: float, T_n: int = 128) -> int:
    """ELL width for the sweep: smallest power of two >= 4x the mean count per tile, at least 8."""
    mean = activity * T_n
    return max(8, 1 << math.ceil(math.log2(4.0 * mean)))


def sweep_workload(M: int, activity: float, seed: int = 0) -> Workload:
    """Sweep point at d_model=4096, d_ff=14336 with lognormal row scaling."""
    return Workload(
        f"sweep_M{M}_p{activity:g}", M, 4096, 14336, 128, sweep_k(activity), activity,
        row_scale="lognormal", training=True, seed=seed,
    )


def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bfloat16 (RNE), returned as uint16 bit patterns.

    Inputs are finite draws; the bfloat16 step adds 0x7FFF plus the lowest kept bit
    to the float32 pattern and truncates, which is round-half-to-even on finite values.
    """
    f32 = np.ascontiguousarray(a, dtype=np.float32)
    u = f32.view(np.uint32)
    # finite patterns are at most 0xFF7FFFFF, so the sum below stays within 32 bits
    r = (u >> 16) & 1
    r += 0x7FFF
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _norm_isf(p: float) -> float:
    from scipy.stats import norm

    return float(norm.isf(p))


def gate_bias_for_activity(activity: float, row_scale: str = "none", sigma: float = 0.75) -> float:
    """Constant gate bias b with P(z0 + b > 0) = activity.

    With x_k ~ N(0,1) and w_k ~ N(0, 1/d), z0 = sum_k x_k w_k is N(0, 1) to first
    order, so b = -Q^{-1}(p). With a per-token scale s ~ lognormal(0, sigma),
    z0 = s * N(0,1) and b solves E_s[Q(-b/s)] = p (one-dimensional integral over
    the log-scale, solved by bracketing). The realised fraction on a given seed is
    measured by the caller and reported next to every result.
    """
    if not (0.0 < activity < 1.0):
        raise ValueError("activity must be in (0, 1)")
    if row_scale == "none":
        return -_norm_isf(activity)
    if row_scale != "lognormal":
        raise ValueError(f"unknown row_scale {row_scale!r}")
    from scipy import integrate, optimize
    from scipy.stats import norm

    def active_fraction(b: float) -> float:
        f = lambda t: norm.pdf(t) * norm.sf(-b * math.exp(-sigma * t))  # noqa: E731
        return integrate.quad(f, -12.0, 12.0, limit=400)[0]

    return float(optimize.brentq(lambda b: active_fraction(b) - activity, -200.0, 0.0, xtol=1e-10))


def _draw_rows(rng: np.random.Generator, rows: int, cols: int, scale: float,
               row_scale: Optional[np.ndarray] = None) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.uint16)
    buf = np.empty((min(rows, _ROW_CHUNK), cols), dtype=np.float64)
    for r0 in range(0, rows, _ROW_CHUNK):
        r1 = min(rows, r0 + _ROW_CHUNK)
        a = buf[: r1 - r0]
        rng.standard_normal(out=a)
        if scale != 1.0:
            a *= scale
        if row_scale is not None:
            a *= row_scale[r0:r1, None]
        out[r0:r1] = bf16_bits_from_f64(a)
    return out


def make_inputs(w: Workload, seed: Optional[int] = None, with_dY: Optional[bool] = None,
                M: Optional[int] = None, shard: int = 0) -> dict:
    """Draw one workload. Returns uint16 (bf16 bit) arrays and the recipe metadata.

    Keys: X [M, d], W_g [f, d], b_g [f], W_u [f, d], W_d [d, f], dY [M, d] (training),
    plus "meta" with the seed, the calibrated bias value (as float) and the shapes.
    `M` overrides the token count (the weights do not depend on it). `shard` > 0
    draws another batch of tokens for the same weights (the per-token streams X,
    s and dY come from the children of SeedSequence([seed, shard]); the weights
    from the seed's own), as the ranks of a data-parallel step hold; shard 0 is
    the plain draw.
    """
    seed = w.seed if seed is None else int(seed)
    with_dY = w.training if with_dY is None else bool(with_dY)
    M = w.M if M is None else int(M)
    d, f = w.d_model, w.d_ff
    streams = dict(zip(_STREAMS, np.random.SeedSequence(seed).spawn(len(_STREAMS))))
    if shard:
        tok = dict(zip(_STREAMS, np.random.SeedSequence([seed, int(shard)]).spawn(len(_STREAMS))))
        streams.update({k: tok[k] for k in ("X", "s", "dY")})
    g = {k: np.random.Generator(np.random.PCG64(v)) for k, v in streams.items()}

    s = None
    if w.row_scale == "lognormal":
        s = np.exp(w.sigma * g["s"].standard_normal(M))
    # each tensor has its own stream, so the draws run concurrently (numpy releases
    # the GIL in bulk fills) and give the same values as drawing them one by one
    jobs = {"X": (g["X"], M, d, 1.0, s), "W_g": (g["W_g"], f, d, 1.0 / math.sqrt(d)),
            "W_u": (g["W_u"], f, d, 1.0 / math.sqrt(d)), "W_d": (g["W_d"], d, f, 1.0 / math.sqrt(f))}
    if with_dY:
        jobs["dY"] = (g["dY"], M, d, 1.0)
    big = M * d + 3 * f * d > (1 << 24)
    if big:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
            futs = {k: ex.submit(_draw_rows, *a) for k, a in jobs.items()}
            drawn = {k: fu.result() for k, fu in futs.items()}
    else:
        drawn = {k: _draw_rows(*a) for k, a in jobs.items()}
    b = gate_bias_for_activity(w.activity, w.row_scale, w.sigma)
    b_bits = bf16_bits_from_f64(np.full(f, b))
    out = dict(X=drawn["X"], W_g=drawn["W_g"], b_g=b_bits, W_u=drawn["W_u"], W_d=drawn["W_d"])
    if with_dY:
        out["dY"] = drawn["dY"]
    out["meta"] = dict(
        workload=w.name, seed=seed, shard=int(shard), M=M, d_model=d, d_ff=f, T_n=w.T_n, K=w.K,
        target_activity=w.activity, row_scale=w.row_scale, sigma=w.sigma,
        b_g=float(bf16_bits_to_f32(b_bits[:1])[0]),
    )
    return out
