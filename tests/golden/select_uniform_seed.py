"""Pick the seed of the uniform-sparsity inference workload.

The workload (M=4096, d_model=2048, d_ff=8192, T_n=128, K=8, 1% i.i.d. activity)
is specified with no row overflowing K. At 1.28 actives per tile on average some
seeds do produce a tile with more than 8, so this script walks seeds 0, 1, 2, ...
and keeps the first one whose oracle packing (fp64 gate, exact z > 0 test) has
no overflowing row. It calls only the CPU oracle and the seeded generator, and
writes uniform_seed.json next to itself with the per-seed statistics it saw.

Run from the repository root:  python tests/golden/select_uniform_seed.py
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle as O  # noqa: E402
from synthetic import WORKLOADS, make_inputs  # noqa: E402


def main(max_seed: int = 20) -> None:
    w = WORKLOADS["uniform"]
    seen = []
    chosen = None
    for seed in range(max_seed):
        inp = make_inputs(w, seed=seed)
        Z = O.gate(inp["X"], inp["W_g"], inp["b_g"])
        p = O.pack(Z, w.T_n, w.K)
        stats = dict(seed=seed, n_ovf=p["n_ovf_total"], activity=float((Z > 0).mean()),
                     max_count=int(p["count"].max()), mean_count=float(p["count"].mean()),
                     b_g=inp["meta"]["b_g"])
        print(stats, flush=True)
        seen.append(stats)
        if p["n_ovf_total"] == 0:
            chosen = seed
            break
    if chosen is None:
        raise SystemExit("no seed without overflow found")
    out = dict(workload=w.name, M=w.M, d_model=w.d_model, d_ff=w.d_ff, T_n=w.T_n, K=w.K,
               target_activity=w.activity, seed=chosen, seeds_tried=seen,
               written_by="tests/golden/select_uniform_seed.py (CPU oracle only)")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "uniform_seed.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", path, "seed", chosen)


if __name__ == "__main__":
    main()
