"""Choice of the ELL width K and of the dense-row threshold from measured costs.

The pages fix no K. [aivizor] paragraph 4 only warns that in training the
largest number of nonzeros per row can be far above the mean, so one fixed K
either wastes slots or sends many rows to the dense backup. Two knobs follow:

* dense_min (struct twell_hybrid): a row with at least this many active units
  goes to the dense backup even when no tile overflows, because its gathers
  would cost more than a dense row on the tensor cores. ``dense_min_for`` gives
  the break-even from the cost model: r * d_ff / a active units.
* K: ``suggest_k`` turns the statistics of ``twell_count_stats`` (bins
  c = 0..T_n of per-row largest tile count, with those rows' active units, plus
  bin T_n + 1 for rows routed dense by dense_min; and per-tile counts) into a
  modelled time per candidate K and returns the cheapest. A training loop calls
  it on one batch's statistics to set K for the next batches; an inference
  server calls it on a calibration batch.

Row routing, candidate K:
    rows(K)  = sum of rows_by_max[c] over c > K        (dense backup rows)
    pairs(K) = sum of act_by_max[c] over c <= K        (units kept in ELL slots)
    t(K) = a * d * pairs(K) + r * d * f * rows(K) + (bytes of the slots) / BW
           + [rows(K) > 0] * (fixed cost of the dense backup GEMMs)
The fixed cost is what the backup GEMMs take beyond their empty launch as soon
as one row overflows: per GEMM a launch and one pass over its weight matrix
(the forward has two, the backward two more, dX with two matrices). The model
takes a lower bound, 3 us plus the matrix at the HBM copy rate; B200 measured
16-28 us per GEMM for a single row at d_model=2048, d_ff=8192. A bound keeps
the heavy-tailed batches, where the model's pair cost is itself low for long
rows, on the measured best K.
Tile routing (inference only), every active unit is gathered and each tile
over K is read from its spilled dense slice:
    t(K) = a * d * total + (bytes of the slots + 512 bytes per spilled tile) / BW
with the slot bytes M * T * (2 + 3K) (count, values, columns), written by the
gate epilogue and read back once. Terms that do not depend on K (the gate
GEMM) are left out.

The coefficients are B200 measurements of this library: ``a`` is the time of
one (token, unit) pair per d_model element in the sparse kernels (forward: the
fused up+down; training adds the sparse backward, the pair list and the weight
gradients), ``r`` the time per d_model * d_ff element of one dense backup row
on the tensor cores (forward: up and down GEMMs; training adds dH, dX and the
dense weight gradients). ``a`` depends on whether the three weight matrices
stay in L2 (d_model=2048, d_ff=8192: the uniform training step) or stream
from HBM (d_model=4096, d_ff=14336: a least-squares fit over the K sweep at
M in {2048, 8192}, sparsity in {95, 99, 99.9}%, K in {8, 16, 32, 64}).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Iterable, Mapping, Sequence

import numpy as np

CANDIDATES = (8, 16, 32, 64)
L2_BYTES = 126 << 20


@dataclass(frozen=True)
class CostModel:
    pair_fwd_s: float = 4.2e-13      # fused up+down, per pair per d_model element
    pair_bwd_s: float = 9.1e-13      # sparse backward + pair list + weight gradients
    dense_fwd_s: float = 6.5e-15     # per dense row per d_model * d_ff element, forward
    dense_bwd_s: float = 1.04e-14    # the same, backward
    hbm_bytes_s: float = 6.5e12
    gemm_launch_s: float = 3e-6        # a dense backup GEMM with any row, beyond its empty launch
    weight_stream_bytes_s: float = 6.5e12  # one pass over a weight matrix by a few-row GEMM (bound)

    def dense_fixed_s(self, d_model: int, d_ff: int, training: bool) -> float:
        """Cost of the dense backup GEMMs as soon as one row overflows: up and
        down in the forward, dH and dX (two weight matrices) in the backward."""
        w = 2.0 * d_model * d_ff / self.weight_stream_bytes_s
        fwd = 2 * (self.gemm_launch_s + w)
        return fwd + ((self.gemm_launch_s + w) + (self.gemm_launch_s + 2 * w) if training else 0.0)

    @classmethod
    def for_shape(cls, d_model: int, d_ff: int) -> "CostModel":
        """Coefficients for a shape: gathers from L2 when the three bf16 weight
        matrices fit in it, else from HBM (the default coefficients)."""
        if 3 * 2 * d_model * d_ff <= L2_BYTES:
            return cls(pair_fwd_s=2.5e-13, pair_bwd_s=8.1e-13)
        return cls()


def dense_min_for(d_model: int, d_ff: int, training: bool = True, model: CostModel | None = None) -> int:
    """Active units per row above which a dense backup row is cheaper than the
    row's gathers: ceil(r * d_ff / a)."""
    m = model or CostModel.for_shape(d_model, d_ff)
    a = m.pair_fwd_s + (m.pair_bwd_s if training else 0.0)
    r = m.dense_fwd_s + (m.dense_bwd_s if training else 0.0)
    return max(1, int(math.ceil(r * d_ff / a)))


def _np(stats: Mapping[str, object], key: str) -> np.ndarray:
    v = stats[key]
    if hasattr(v, "detach"):
        v = v.detach().cpu().numpy()
    return np.asarray(v, dtype=np.int64)


def modelled_times(stats: Mapping[str, object], d_model: int, d_ff: int, T_n: int = 128,
                   candidates: Iterable[int] = CANDIDATES, training: bool = True, routing: str = "rows",
                   model: CostModel | None = None) -> dict:
    """Modelled seconds per candidate K (see the module docstring)."""
    if routing not in ("rows", "tiles"):
        raise ValueError("routing is 'rows' or 'tiles'")
    if training and routing == "tiles":
        raise ValueError("tile routing is an inference-only format")
    rows_by_max = _np(stats, "rows_by_max")
    act_by_max = _np(stats, "act_by_max")
    tiles_by_count = _np(stats, "tiles_by_count")
    if not (rows_by_max.shape == act_by_max.shape == tiles_by_count.shape == (T_n + 2,)):
        raise ValueError(f"statistics must have T_n + 2 = {T_n + 2} bins")
    model = model or CostModel.for_shape(d_model, d_ff)
    M = int(rows_by_max.sum())
    T = d_ff // T_n
    total = int(act_by_max.sum())
    a = model.pair_fwd_s + (model.pair_bwd_s if training else 0.0)
    r = model.dense_fwd_s + (model.dense_bwd_s if training else 0.0)
    out = {}
    for K in candidates:
        K = int(K)
        if not 1 <= K <= T_n:
            raise ValueError(f"K={K} outside [1, T_n]")
        slots = M * T * (2 + 3 * K)
        if routing == "rows":
            pairs = int(act_by_max[:K + 1].sum())
            rows = int(rows_by_max[K + 1:].sum())
            out[K] = (a * d_model * pairs + r * d_model * d_ff * rows + slots / model.hbm_bytes_s
                      + (model.dense_fixed_s(d_model, d_ff, training) if rows > 0 else 0.0))
        else:
            spilled = int(tiles_by_count[K + 1:].sum())
            out[K] = a * d_model * total + (slots + 512 * spilled) / model.hbm_bytes_s
    return out


def suggest_k(stats: Mapping[str, object], d_model: int, d_ff: int, T_n: int = 128,
              candidates: Sequence[int] = CANDIDATES, training: bool = True, routing: str = "rows",
              model: CostModel | None = None) -> tuple[int, dict]:
    """The candidate K of least modelled time (the smaller K on a tie) and the table of times."""
    times = modelled_times(stats, d_model, d_ff, T_n, candidates, training, routing, model)
    best = min(sorted(times), key=lambda k: times[k])
    return best, times
