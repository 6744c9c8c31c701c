#!/usr/bin/env python
"""Throughput of the TwELL activation-sparse gated FFN training step on B200.

One step = the whole hot path over one batch: W_d transposed for the step's
weights, the gate GEMM with the TwELL pack epilogue, row routing, the sparse
up+down for ELL rows and the dense backup for overflow rows, then the backward
over the hybrid format (L1 term on the gate activations). Workload: M=65536
tokens, d_model=4096, d_ff=14336, T_n=128, K=8, 99% sparsity (1% target
activity) with lognormal(0, 0.75) per-token row scaling, synthetic seeded data
drawn on the host, inputs resident in HBM. The line also carries the forward
half and the inference forward of that workload, the dense bf16 FFN on the
same inputs, and two smaller workloads beside it (the uniform 1% inference
forward at M=4096, d_model=2048, d_ff=8192, and the uniform training step at
M=8192 of the same shape).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
    python bench.py --sweep [--steps K --warmup W]
    python bench.py --block [--steps K --warmup W]

--sweep times the forward and forward+backward of TwELL and of the dense bf16
FFN over token counts M in {512, 2048, 8192, 32768, 65536} and mean sparsity in
{90, 95, 99, 99.5, 99.9}% at d_model=4096, d_ff=14336, with per-token
lognormal(0, 0.75) row scaling, K = max(8, 2^ceil(log2(4 p T_n))), one JSON
line per point (1 GPU). Each point also times adaptive routing: the dense-row
threshold of the cost model and the K chosen from the batch's count statistics
(activation_sparse_ffn_gemm_b200.kchoice). With --sweep-k 8,16,32,64 each point is timed for every
listed K instead, next to the K that the batch's count statistics and the cost
model of activation_sparse_ffn_gemm_b200.kchoice choose.

Prints one JSON line (rank 0). With N > 1 (torchrun) the step is the
token-sharded (data-parallel) training step: every rank holds its own batch of
tokens for the same weights and the weight gradients are summed over the ranks
by NCCL all-reduce inside every timed step (activation_sparse_ffn_gemm_b200.sharded);
the time is the max over ranks and the value counts the tokens of all ranks
(weak scaling).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse FFN tokens/s fwd & fwd+bwd at 99% sparsity vs dense; % of roofline"
L2_FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["twell", "reference"], default="twell")
    p.add_argument("--lam", type=float, default=1e-3)
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-trace", action="store_true")
    p.add_argument("--workload", default=MAIN_WORKLOAD, choices=["large", "sweep8k", "sweep2k", "sweep512", "train", "heavy"],
                   help="workload of the timed training step (synthetic.WORKLOADS)")
    p.add_argument("--no-extra", action="store_true", help="skip the two smaller workloads of the line")
    p.add_argument("--step-only", action="store_true",
                   help="time the training step alone (no trace, inference, 8-bit, end-to-end, dense or CPU legs, "
                        "no smaller workloads): the command profiler captures run")
    p.add_argument("--sweep", action="store_true",
                   help="token-count x sparsity sweep at d_model=4096, d_ff=14336 (one JSON line per point)")
    p.add_argument("--sweep-m", default="512,2048,8192,32768,65536")
    p.add_argument("--sweep-sparsity", default="0.9,0.95,0.99,0.995,0.999")
    p.add_argument("--block", action="store_true",
                   help="one transformer block with the dense or the TwELL FFN, forward and forward+backward")
    p.add_argument("--sweep-k", default="",
                   help="with --sweep: time every K of this list at each point (e.g. 8,16,32,64) next to the "
                        "K chosen from the count statistics")
    p.add_argument("--sched", default="auto", choices=["auto", "fused", "passes"],
                   help="schedule of the sparse kernels (twell_set_sparse_schedule)")
    p.add_argument("--l2-budget-mib", type=int, default=0,
                   help="L2 budget of one chunk of the multi-pass schedule, MiB (0: the library default)")
    p.add_argument("--overlap", default="auto", choices=["auto", "on", "off"],
                   help="dense-backup GEMMs on the library's side stream beside the sparse kernels "
                        "(twell_set_overlap; auto: below 4096 rows)")
    return p.parse_args()


def apply_schedule(args):
    """Sets the sparse-kernel schedule the command line asks for (process-wide)."""
    import activation_sparse_ffn_gemm_b200 as tw

    mode = {"auto": tw.SCHED_AUTO, "fused": tw.SCHED_FUSED, "passes": tw.SCHED_PASSES}[args.sched]
    tw.set_sparse_schedule(mode, args.l2_budget_mib << 20)
    tw.set_overlap({"auto": tw.OVERLAP_AUTO, "on": tw.OVERLAP_ON, "off": tw.OVERLAP_OFF}[args.overlap])


def reduce_max(x: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


# the workload of the timed training step, and the smaller ones reported beside it
MAIN_WORKLOAD = "large"
OTHER_WORKLOADS = (("uniform_d2048_f8192_M4096_inference", "uniform", "infer"),
                   ("uniform_d2048_f8192_M8192_training", "train", "train"))
CPU_SLICE_ROWS = 256  # token rows of the CPU baseline's slice of the main workload


def workload(name=MAIN_WORKLOAD):
    from synthetic import WORKLOADS

    w = WORKLOADS[name]
    seed = w.seed
    if name == "uniform":
        with open(os.path.join(ROOT, "tests", "golden", "uniform_seed.json")) as fh:
            seed = json.load(fh)["seed"]
    return w, seed


def workload_desc(w, seed, mode="train"):
    rows = (f"lognormal(0, {w.sigma:g}) per-token row scale" if w.row_scale == "lognormal"
            else "i.i.d. activity across tokens")
    what = "training step (forward + backward)" if mode == "train" else "inference forward"
    return (f"{100.0 * (1.0 - w.activity):g}% sparsity ({100.0 * w.activity:g}% target activity), {rows}: "
            f"M={w.M} tokens, d_model={w.d_model}, d_ff={w.d_ff}, T_n={w.T_n}, K={w.K}, seed {seed}, {what}")


def ovf_cap_for(w):
    """Dense-backup capacity of the timed runs: a quarter of the rows (the heavy-tailed
    99% batches route about 10% of their rows dense; the status word is checked)."""
    return max(1, w.M // 4)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs.

    NVML is polled every 2 ms from a thread (a timed region of a few tens of
    milliseconds still gets samples under load); without NVML, nvidia-smi
    samples every 200 ms. Reading clocks changes no GPU setting."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.nvml = None
        self.samples = []
        self.max_mhz = None
        self.stop = threading.Event()
        self.thread = None

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        try:
            self.nvml, h = self._nvml_handle()
            self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(h, self.nvml.NVML_CLOCK_SM))

            def poll():
                while not self.stop.is_set():
                    self.samples.append((float(self.nvml.nvmlDeviceGetClockInfo(h, self.nvml.NVML_CLOCK_SM)),
                                         int(self.nvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        time.sleep(0.25)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.nvml is not None:
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0,
                        "source": "nvml"}
            reasons = sorted(n for n, bit in self.REASONS.items() if any(r & bit for _, r in self.samples))
            return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(self.samples), "source": "nvml, every 2 ms"}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, every 200 ms"}


# ------------------------------------------------------ algorithmic work


def kernel_work(name, M, d, f, T, K, kept, pairs, n_ovf=0, dense_wgrad=0):
    """Algorithmic flops (tensor-bound kernels) or bytes (memory-bound) of one launch.

    kept = stored slots of ELL rows (all their active units), pairs = all active
    (row, unit) pairs, n_ovf = stored dense backup rows, dense_wgrad = 1 when the
    overflow rows' weight gradients run as GEMMs (their pairs then stay out of
    the pair list). The dense backup GEMMs count the plain contraction (the
    weight-gradient GEMMs run it twice, over hi and lo halves of their operand)."""
    m_ell = M - n_ovf
    listed = kept + (0 if dense_wgrad else pairs - kept)
    if name == "gate_pack_gemm":
        return "tensor", 2.0 * M * d * f
    if name in ("ovf_up_gemm", "ovf_down_gemm", "ovf_dh_gemm", "dense_wgrad_d"):
        return "tensor", 2.0 * n_ovf * d * f
    if name in ("ovf_dx_gemm", "dense_wgrad_ug"):
        return "tensor", 4.0 * n_ovf * d * f
    if name == "ell_updown":
        return "hbm", (2 * m_ell * d            # X
                       + m_ell * T * (2 + 3 * K)  # TwELL count/val/col
                       + 4 * kept                 # u written
                       + 2 * m_ell * d            # Y written
                       + 2 * 2 * f * d)           # W_u, W_dt read once
    if name == "ell_updown_q8":
        # as ell_updown, with the two gathered weights read as 1-byte codes (plus a scale per unit)
        return "hbm", (2 * m_ell * d + m_ell * T * (2 + 3 * K) + 4 * kept + 2 * m_ell * d + 2 * f * d + 2 * 4 * f)
    if name == "ell_up":
        # the up pass: X, TwELL, u written, W_u once
        return "hbm", 2 * m_ell * d + m_ell * T * (2 + 3 * K) + 4 * kept + 2 * f * d
    if name == "ell_down":
        # the down pass: TwELL, u read, Y written, W_dt once
        return "hbm", m_ell * T * (2 + 3 * K) + 4 * kept + 2 * m_ell * d + 2 * f * d
    if name == "ell_dh":
        # the dH pass: dY, TwELL, u read, (h, dU, dZ) per slot written, W_dt once
        return "hbm", 2 * m_ell * d + m_ell * T * (2 + 3 * K) + 4 * kept + 16 * kept + 2 * f * d
    if name == "ell_dx":
        # the dX pass: counts and columns, (h, dU, dZ) per slot read, dX (fp32) written, W_u and W_g once
        return "hbm", m_ell * T * (2 + K) + 16 * kept + 4 * m_ell * d + 2 * 2 * f * d
    if name == "ell_bwd":
        # dY, TwELL, u read; (h, dU, dZ) per slot written; dX (fp32) written; W_u, W_g, W_dt once
        return "hbm", (2 * m_ell * d + m_ell * T * (2 + 3 * K) + 4 * kept + 16 * kept + 4 * m_ell * d
                       + 3 * 2 * f * d)
    if name == "weight_grads":
        # X and dY rows once, the pair list (row + (h, dU, dZ)), three fp32 gradients written
        # (and read back when the dense GEMMs wrote the overflow rows' part first), db_g
        return "hbm", (2 * 2 * M * d + 20 * listed + (2 if dense_wgrad else 1) * 3 * 4 * f * d + 4 * f)
    if name == "transpose_wd":
        return "hbm", 2 * 2 * f * d
    if name in ("csc_count", "csc_fill"):
        return "hbm", M * T * (2 + K) + (20 * listed if name == "csc_fill" else 0)
    return None, None


# Source files that define each traced kernel's code (its own translation unit
# and the headers it compiles in); a committed DRAM capture applies only while
# these files are unchanged.
KERNEL_SOURCES = {
    "gate_pack_gemm": ("gemm_kernels.cu", "umma_gemm.cuh", "umma_gemm_pair.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_updown": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_bwd": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_up": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_down": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_dh": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "ell_dx": ("token_kernels.cu", "token_common.cuh", "sm100.cuh", "twell_internal.cuh"),
    "weight_grads": ("pairlist_kernels.cu", "twell_internal.cuh"),
    "csc_fill": ("pairlist_kernels.cu", "twell_internal.cuh"),
    "transpose_wd": ("route_kernels.cu", "twell_internal.cuh"),
}


def path_roofline(M, d, f, T, K, kept, n_ovf, peaks, ms_fwd, ms_step):
    """Whole-step roofline: the time the step's algorithmic work takes at the
    measured peaks (dense flops at the sustained bf16 rate, algorithmic bytes
    at the HBM copy rate), against the measured times.

    forward:  gate GEMM 2 M d f flops; dense backup 4 M_ovf d f flops; bytes:
              X, TwELL (2 + 3K bytes per row tile), Y, u saved, W_u and W_dt
              once, the W_d transpose (read + write)
    backward: 12 d flops per kept pair (dH, dX, three weight gradients) and
              12 M_ovf d f for dense rows; bytes: X, dY, TwELL, u, dX (fp32),
              W_u, W_g, W_dt once, the three fp32 weight gradients written
    """
    P = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12
    B = peaks["hbm_gbs"] * 1e9
    tw_bytes = M * T * (2 + 3 * K)
    f_flops = 2.0 * M * d * f + 4.0 * n_ovf * d * f
    f_bytes = 2 * M * d + tw_bytes + 2 * M * d + 4 * kept + 2 * 2 * f * d + 2 * 2 * f * d
    b_flops = 12.0 * d * kept + 12.0 * n_ovf * d * f
    b_bytes = 2 * M * d + 2 * M * d + tw_bytes + 4 * kept + 4 * M * d + 3 * 2 * f * d + 3 * 4 * f * d
    t_f = f_flops / P + f_bytes / B
    t_s = t_f + b_flops / P + b_bytes / B
    return {"fwd_ms": t_f * 1e3, "step_ms": t_s * 1e3, "fwd_frac": t_f * 1e3 / ms_fwd, "step_frac": t_s * 1e3 / ms_step,
            "note": "algorithmic time at measured peaks (sustained bf16, HBM copy) / measured time"}


def source_hash(kernel):
    files = KERNEL_SOURCES.get(kernel)
    if not files:
        return None
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_sparse_ffn_gemm_b200", "csrc")
    for fn in files:
        with open(os.path.join(csrc, fn), "rb") as fh:
            h.update(fn.encode() + fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel, wname=MAIN_WORKLOAD):
    """DRAM bytes per launch of `kernel` on workload `wname` from the committed ncu
    capture, if the kernel's sources still match the ones captured."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    rec = d.get("workloads", {}).get(wname, {}).get("kernels", {}).get(kernel)
    if not rec or rec.get("source_sha") != source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------ CPU oracle


def _oracle_rows(O, inp, n, lam):
    """One oracle step on the first n token rows: forward (Y of those rows) and
    backward (dX of those rows, weight gradients over them); returns seconds."""
    import numpy as np

    rows = np.arange(n, dtype=np.int32)
    t0 = time.perf_counter()
    O.ffn_fwd(inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], rows=rows)
    O.ffn_bwd(inp["X"][:n], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], inp["dY"][:n], lam)
    return time.perf_counter() - t0


def cpu_baseline_slice(inp, lam, n):
    """The fp64 oracle as it stands, forward + backward on a fixed slice of n token rows."""
    from oracle import oracle as O

    O.build()
    M = inp["X"].shape[0]
    n = min(n, M)
    t = _oracle_rows(O, inp, n, lam)
    return {"value": n / t, "unit": "tokens/s", "cores": O.get_threads(), "kind": "oracle",
            "sample": f"slice: first {n} of {M} token rows, forward + backward (weight gradients over the "
                      f"slice), {t:.1f} s"}


def cpu_baseline(inp, lam, target_s):
    """The fp64 oracle as it stands, forward + backward on a sample of token rows
    sized towards target_s seconds; returns (line, rows, seconds)."""
    from oracle import oracle as O

    O.build()
    M = inp["X"].shape[0]
    n = 8
    t = _oracle_rows(O, inp, n, lam)
    for _ in range(3):  # grow the sample towards target_s (the oracle's cost is not quite linear in rows)
        if t >= target_s / 2 or n >= M:
            break
        n = int(min(M, max(2 * n, n * target_s / max(t, 1e-3))))
        t = _oracle_rows(O, inp, n, lam)
    return {"value": n / t, "unit": "tokens/s", "cores": O.get_threads(), "kind": "oracle",
            "sample": f"first {n} of {M} token rows, forward + backward (weight gradients over the sample), "
                      f"{t:.1f} s"}, n, t


# --------------------------------------------------------------- arms


def run_reference(args, world, rank):
    if rank != 0:
        return
    import numpy as np

    from oracle import oracle as O
    from synthetic import make_inputs

    w, seed = workload(args.workload)
    inp = make_inputs(w, seed=seed, with_dY=True)
    O.build()
    # each step: the oracle's forward + backward on a bounded sample of rows
    # the whole run is sized to about 5 x --cpu-seconds (60 s by default) of oracle work
    probe = cpu_baseline(inp, args.lam, target_s=max(0.05, 5.0 * args.cpu_seconds / max(1, args.steps + args.warmup)))
    n = probe[1]
    rows = np.arange(n, dtype=np.int32)

    def step():
        O.ffn_fwd(inp["X"], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], rows=rows)
        O.ffn_bwd(inp["X"][:n], inp["W_g"], inp["b_g"], inp["W_u"], inp["W_d"], inp["dY"][:n], args.lam)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = n / dt
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_desc(w, seed, "train"), "sample_rows_per_step": n,
                   "reference": "fp64 CPU oracle (oracle/twell_oracle.c), OpenMP over rows"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": O.get_threads(), "kind": "oracle",
                         "sample": f"first {n} of {w.M} token rows per step, forward + backward"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _dense_arm(torch, X, W_g, b_g, W_u, W_d, dY, lam, timed, train):
    """The dense bf16 gated FFN in torch (cuBLAS) on the same inputs, in two forms:
    three GEMMs, and one GEMM against the stacked [W_g; W_u] (the concatenation is
    made once, outside the timed region, as a model storing the fused weight
    would). The backward goes through autograd with the L1 term's gradient fed
    in directly (lambda on every gate activation), so no extra reduction is timed.
    Returns per-form times and the faster form for each measure."""
    f = W_g.shape[0]
    M = X.shape[0]
    W_gu = torch.cat([W_g, W_u]).contiguous()

    def fwd3(e_mid):
        with torch.no_grad():
            (torch.relu(X @ W_g.T + b_g) * (X @ W_u.T)) @ W_d.T
        e_mid.record()

    def fwd_fused(e_mid):
        with torch.no_grad():
            zu = X @ W_gu.T
            (torch.relu(zu[:, :f] + b_g) * zu[:, f:]) @ W_d.T
        e_mid.record()

    res = {"fwd_ms": {"three_gemms": timed(fwd3), "fused_gate_up": timed(fwd_fused)}}
    if train:
        Xr = X.clone().requires_grad_()
        Wg_r, Wu_r, Wd_r, Wgu_r = (t.clone().requires_grad_() for t in (W_g, W_u, W_d, W_gu))
        lam_g = torch.full((1, 1), lam, dtype=torch.bfloat16, device=X.device).expand(M, f)

        def fb3(e_mid):
            g = torch.relu(Xr @ Wg_r.T + b_g)
            y = (g * (Xr @ Wu_r.T)) @ Wd_r.T
            torch.autograd.backward((y, g), (dY, lam_g))
            Xr.grad = Wg_r.grad = Wu_r.grad = Wd_r.grad = None
            e_mid.record()

        def fb_fused(e_mid):
            zu = Xr @ Wgu_r.T
            g = torch.relu(zu[:, :f] + b_g)
            y = (g * zu[:, f:]) @ Wd_r.T
            torch.autograd.backward((y, g), (dY, lam_g))
            Xr.grad = Wgu_r.grad = Wd_r.grad = None
            e_mid.record()

        res["fwd_bwd_ms"] = {"three_gemms": timed(fb3), "fused_gate_up": timed(fb_fused)}
    for k in ("fwd_ms", "fwd_bwd_ms"):
        if k in res:
            best = min(res[k], key=res[k].get)
            res[k.replace("_ms", "_best")] = {"form": best, "ms": res[k][best], "tokens_per_s": M / (res[k][best] / 1e3)}
    return res


def run_twell(args, world, rank, local):
    import numpy as np
    import torch

    import activation_sparse_ffn_gemm_b200 as tw
    from activation_sparse_ffn_gemm_b200.sharded import allreduce_grads
    from synthetic import make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, dist, dev)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed_pair(n, body):
        """Per-step CUDA events on the launching stream, L2 flushed before each
        step (outside the events); returns the mean step time and the mean time
        to the event the body records part-way (body(e_mid))."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier()
        torch.cuda.synchronize(dev)
        for e0, e1, e2 in ev:
            flush.zero_()
            e0.record(stream)
            body(e1)
            e2.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return sum(a.elapsed_time(c) for a, _, c in ev) / n, sum(a.elapsed_time(b) for a, b, _ in ev) / n

    def warm_and_time(body):
        for _ in range(max(3, args.warmup)):
            body(torch.cuda.Event())
        return max_over_ranks(timed_pair(args.steps, body)[0])

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    def measure(name, mode, full):
        """Times one workload: mode "train" = forward + backward per step, "infer"
        = the inference forward (W_dt prepared once, u not saved). `full` adds the
        per-kernel trace, the inference forward of a training workload, the
        end-to-end run with host copies, and the CPU baseline."""
        w, seed = workload(name)
        # with N ranks each rank holds its own tokens for the same weights (shard = rank)
        inp = make_inputs(w, seed=seed, with_dY=True, shard=rank if world > 1 else 0)
        X, W_g, b_g, W_u, W_d, dY = (dev_bf16(inp[k]) for k in ("X", "W_g", "b_g", "W_u", "W_d", "dY"))
        M, d, f, K, T = w.M, w.d_model, w.d_ff, w.K, w.d_ff // w.T_n
        cap = ovf_cap_for(w)
        train = mode == "train"
        st = tw.HybridState(M, f, w.T_n, K, cap, dev, with_u=train)
        wsf = tw.workspace(tw.OP_FWD, M, d, f, w.T_n, K, cap, dev)
        wsb = tw.workspace(tw.OP_BWD, M, d, f, w.T_n, K, cap, dev) if train else None
        Wdt = torch.empty((f, d), dtype=torch.bfloat16, device=dev)
        Y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
        grads = (dict(dX=torch.empty((M, d), device=dev), dW_g=torch.empty((f, d), device=dev),
                      dW_u=torch.empty((f, d), device=dev), dW_d=torch.empty((d, f), device=dev),
                      db_g=torch.empty(f, device=dev)) if train else None)
        res = {"workload": workload_desc(w, seed, mode), "M": M, "ovf_cap": cap}

        def fwd_train():
            tw.transpose_wd(W_d, out=Wdt)
            tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=w.T_n, K=K, W_dt=Wdt, state=st, ws=wsf, Y=Y)

        def bwd():
            tw.ffn_bwd(X, W_g, W_u, W_d, st, dY, lam=args.lam, W_dt=Wdt, ws=wsb, out=grads)
            allreduce_grads(grads)  # data parallel over ranks: weight gradients summed (NCCL); no-op on one rank

        def train_step(e_mid):
            fwd_train()
            e_mid.record(stream)
            bwd()

        def infer(st_i):
            def body(e_mid):
                tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=w.T_n, K=K, W_dt=Wdt, state=st_i, ws=wsf, Y=Y)
                e_mid.record(stream)
            return body

        if not train:
            tw.transpose_wd(W_d, out=Wdt)  # fixed weights: transposed once, outside the timed region
        step = train_step if train else infer(st)
        for _ in range(max(3, args.warmup)):
            step(torch.cuda.Event())
        torch.cuda.synchronize(dev)
        assert st.read_status() == 0, f"device status word set during warm-up ({name})"
        launches0 = tw.launch_count()
        clk = ClockSampler(local) if full else None
        if clk:
            clk.__enter__()
        ms_step, ms_mid = timed_pair(args.steps, step)
        if clk:
            clk.__exit__(None, None, None)
        res["gpu_launches"] = tw.launch_count() - launches0
        ms_step, ms_mid = max_over_ranks(ms_step), max_over_ranks(ms_mid)
        assert st.read_status() == 0, f"device status word set during timing ({name})"
        res["ms_step"] = ms_step
        if train:
            res["ms_fwd"] = ms_mid
        cnt = st.count.float()
        nst, nfl = st.n_overflow()
        ell_rows = (st.row_ovf[:M] == 0).unsqueeze(1)
        res["kept"] = int((torch.minimum(st.count.int(), torch.tensor(K, device=dev)) * ell_rows).sum().item())
        res["pairs"] = int(st.count.int().sum().item())
        res["n_ovf"] = nst
        res["dense_wgrad"] = int(st.row_plan[3].item())
        res["sparsity"] = {"activity": res["pairs"] / (M * f), "overflow_rows": nfl,
                           "max_count": float(cnt.max().item()), "mean_count": float(cnt.mean().item()),
                           "max_over_mean_count": float(cnt.max().item()) / max(float(cnt.mean().item()), 1e-30)}
        res["shape"] = (M, d, f, T, K)
        if full and args.step_only:
            res["clocks"] = clk.summary()
            return res
        if full:
            res["clocks"] = clk.summary()
            # per-kernel breakdown: the same steps again with event tracing
            breakdown = {}
            if not args.no_trace:
                tw.trace_collect()
                tw.trace_enable(True)
                timed_pair(args.steps, step)
                tw.trace_enable(False)
                for kname, ms in tw.trace_collect():
                    b = breakdown.setdefault(kname, {"launches": 0, "ms": 0.0})
                    b["launches"] += 1
                    b["ms"] += ms
                for b in breakdown.values():
                    b["ms_per_launch"] = b["ms"] / b["launches"]
                    b["ms_per_step"] = b["ms"] / args.steps
            res["breakdown"] = breakdown
            if train:
                # the inference forward with fixed weights: W_d transposed once, u not saved
                st_inf = tw.HybridState(M, f, w.T_n, K, cap, dev, with_u=False)
                res["ms_infer"] = warm_and_time(infer(st_inf))
                assert st_inf.read_status() == 0, "device status word set during the inference timing"
                Y_ref = Y.clone()
                # the same inference forward with the gathers reading 8-bit (E4M3) weights, quantised
                # once outside the timed region; the FFN it computes uses the dequantised weights
                q8 = tw.quantize_weights(W_u, W_d)
                Yq = torch.empty_like(Y)

                def infer_q8(e_mid):
                    tw.ffn_fwd_e4m3(X, W_g, b_g, q8, T_n=w.T_n, K=K, state=st_inf, ws=wsf, Y=Yq)
                    e_mid.record(stream)

                res["ms_infer_e4m3"] = warm_and_time(infer_q8)
                assert st_inf.read_status() == 0, "device status word set during the 8-bit inference timing"
                res["e4m3_rel_l2"] = float((Yq.float() - Y_ref.float()).norm() / Y_ref.float().norm())
                del st_inf, q8, Yq, Y_ref
            res["e2e"] = e2e(M, d, X, dY, Y, lambda Xi, dYi, Yi: (
                tw.transpose_wd(W_d, out=Wdt),
                tw.ffn_fwd(Xi, W_g, b_g, W_u, W_d, T_n=w.T_n, K=K, W_dt=Wdt, state=st, ws=wsf, Y=Yi),
                tw.ffn_bwd(Xi, W_g, W_u, W_d, st, dYi, lam=args.lam, W_dt=Wdt, ws=wsb, out=grads),
                allreduce_grads(grads)))
            assert st.read_status() == 0, "device status word set during the end-to-end timing"
        del st, wsf, wsb, Wdt, Y, grads
        torch.cuda.empty_cache()
        if not args.no_dense:
            res["dense"] = _dense_arm(torch, X, W_g, b_g, W_u, W_d, dY, args.lam, warm_and_time, train)
        del X, W_g, b_g, W_u, W_d, dY
        torch.cuda.empty_cache()
        if full and not args.no_cpu_baseline and world == 1 and rank == 0:
            res["cpu_baseline"] = cpu_baseline_slice(inp, args.lam, CPU_SLICE_ROWS)
        return res

    def e2e(M, d, X, dY, Y, run_step):
        """The same step end to end: every step copies its inputs (X, dY) from
        pinned host memory and reads its result Y back, inside the timed region.
        As a training loop that prefetches its next batch does, the copies run on
        two copy streams (host->device, device->host) into double-buffered device
        tensors, so step i+1's inputs and step i-1's result move while step i
        computes. The step's working set is far larger than L2, so no extra flush
        is inserted."""
        hX = torch.empty((M, d), dtype=torch.bfloat16, pin_memory=True)
        hdY = torch.empty((M, d), dtype=torch.bfloat16, pin_memory=True)
        hY = [torch.empty((M, d), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        hX.copy_(X.cpu())
        hdY.copy_(dY.cpu())
        Xb, dYb, Yb = [X, torch.empty_like(X)], [dY, torch.empty_like(dY)], [Y, torch.empty_like(Y)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def run(n):
            ev_in = [torch.cuda.Event() for _ in range(2)]
            ev_done = [torch.cuda.Event() for _ in range(2)]
            ev_out = [torch.cuda.Event() for _ in range(2)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize(dev)
            t0.record(stream)
            up.wait_stream(stream)
            down.wait_stream(stream)

            def load(b):
                with torch.cuda.stream(up):
                    Xb[b].copy_(hX, non_blocking=True)
                    dYb[b].copy_(hdY, non_blocking=True)
                    ev_in[b].record(up)

            load(0)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    if i >= 1:
                        up.wait_event(ev_done[1 - b])  # step i-1 has finished reading these buffers
                    load(1 - b)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # step i-2's result has left Yb[b]
                run_step(Xb[b], dYb[b], Yb[b])
                ev_done[b].record(stream)
                down.wait_event(ev_done[b])
                with torch.cuda.stream(down):
                    hY[b].copy_(Yb[b], non_blocking=True)
                    ev_out[b].record(down)
            stream.wait_stream(down)
            stream.wait_stream(up)
            t1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return t0.elapsed_time(t1) / n

        run(max(3, args.warmup))
        ms = max_over_ranks(run(args.steps))
        assert torch.equal(hY[(args.steps - 1) % 2].to(dev), Y), "end-to-end result differs from the resident run"

        def copy_ms(body, reps=5):
            """Mean time of one step's host<->device copies alone (no compute), for context."""
            body()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                body()
            e1.record(stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / reps

        ms_h2d = copy_ms(lambda: (Xb[1].copy_(hX, non_blocking=True), dYb[1].copy_(hdY, non_blocking=True)))
        ms_d2h = copy_ms(lambda: hY[1].copy_(Yb[0], non_blocking=True))
        return {"ms_per_step": ms, "h2d_bytes_per_step": 2 * M * d * 2, "d2h_bytes_per_step": M * d * 2,
                "copy_alone_ms": {"h2d": ms_h2d, "d2h": ms_d2h}}

    main = measure(args.workload, "train", full=True)
    others = {}
    if args.step_only:
        if dist is not None:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": main["M"] * world / (main["ms_step"] / 1e3),
                              "unit": "tokens/s", "ms_per_step": main["ms_step"], "fwd_ms": main["ms_fwd"],
                              "steps": args.steps, "warmup": max(3, args.warmup), "config": {
                                  "workload": main["workload"], "note": "training step alone (profiling run)",
                                  "sparse_schedule": args.sched, "l2_budget_mib": args.l2_budget_mib or None,
                                  "overlap": args.overlap},
                              "sparsity": main["sparsity"], "gpu_launches": main["gpu_launches"]}), flush=True)
        return
    if not args.no_extra:
        for key, wname, mode in OTHER_WORKLOADS:
            if wname != args.workload:
                others[key] = measure(wname, mode, full=False)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps(bench_line(args, world, main, others)), flush=True)


def bench_line(args, world, main, others):
    """The JSON line of the TwELL arm from the measurements (host arithmetic only)."""
    peaks, peak_src = load_peaks()
    M, d, f, T, K = main["shape"]
    tokens = M * world
    ms_step, ms_fwd = main["ms_step"], main["ms_fwd"]
    kernels, roofline = kernel_table(main["breakdown"], main, peaks, peak_src, args.steps, ms_step, args.workload)
    dense = main.get("dense")
    e = main["e2e"]

    def summary(r, train):
        out = {"workload": r["workload"], "ovf_cap": r["ovf_cap"], "sparsity": r["sparsity"]}
        tok = r["M"] * world
        if train:
            out["fwd_bwd"] = {"tokens_per_s": tok / (r["ms_step"] / 1e3), "ms": r["ms_step"]}
            out["fwd"] = {"tokens_per_s": tok / (r["ms_fwd"] / 1e3), "ms": r["ms_fwd"]}
        else:
            out["fwd_inference"] = {"tokens_per_s": tok / (r["ms_step"] / 1e3), "ms": r["ms_step"]}
        dn = r.get("dense")
        if dn:
            out["dense_bf16"] = dn
            out["speedup_vs_dense"] = ({"fwd": dn["fwd_best"]["ms"] / r["ms_fwd"],
                                        "fwd_bwd": dn["fwd_bwd_best"]["ms"] / r["ms_step"]} if train else
                                       {"fwd_inference": dn["fwd_best"]["ms"] / r["ms_step"]})
        return out

    return {
        "metric": METRIC,
        "value": tokens / (ms_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": main["workload"], "global_batch": tokens, "lambda_l1": args.lam,
                   "l2": "flushed before every timed step (256 MiB device write, outside the events); "
                         "the step's inputs are also larger than L2",
                   "accumulation": "fp32", "ovf_cap": main["ovf_cap"],
                   "sparse_schedule": (args.sched + (f", L2 budget {args.l2_budget_mib} MiB" if args.l2_budget_mib
                                                     else "")),
                   "dense_overlap": args.overlap,
                   "parallelism": (f"dp{world}: every rank its own {M} tokens, weight gradients summed over "
                                   "ranks (NCCL all-reduce) inside each step" if world > 1 else "dp1")},
        "fwd": {"tokens_per_s": tokens / (ms_fwd / 1e3), "ms": ms_fwd,
                "note": "forward half of the training step (W_d transposed, u saved)"},
        "fwd_inference": {"tokens_per_s": tokens / (main["ms_infer"] / 1e3), "ms": main["ms_infer"],
                          "note": "forward alone with fixed weights (W_dt prepared once, u not saved)"},
        "fwd_inference_e4m3": {"tokens_per_s": tokens / (main["ms_infer_e4m3"] / 1e3), "ms": main["ms_infer_e4m3"],
                               "rel_l2_vs_bf16_weights": main["e4m3_rel_l2"],
                               "note": "the inference forward with the sparse kernel gathering E4M3 weights (per-unit "
                                       "power-of-two scales, quantised once); the FFN computed is the one with the "
                                       "dequantised weights; rel_l2 is its Y against the bf16-weight Y"},
        "dense_bf16": dense,
        "speedup_vs_dense": ({"fwd": dense["fwd_best"]["ms"] / ms_fwd,
                              "fwd_inference": dense["fwd_best"]["ms"] / main["ms_infer"],
                              "fwd_bwd": dense["fwd_bwd_best"]["ms"] / ms_step} if dense else None),
        "e2e": {"value": tokens / (e["ms_per_step"] / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                "ms_per_step": e["ms_per_step"], "copy_alone_ms": e["copy_alone_ms"],
                "copies": "pinned host X and dY in and Y out every step, on two copy streams, overlapping the "
                          "neighbouring steps' compute (double-buffered device inputs and outputs)"},
        "gpu_launches": main["gpu_launches"],
        "roofline": roofline,
        "path_roofline": path_roofline(M, d, f, T, K, main["kept"], main["n_ovf"], peaks, ms_fwd, ms_step),
        "kernels": kernels,
        "sparsity": main["sparsity"],
        "clocks": main["clocks"],
        "cpu_baseline": main.get("cpu_baseline"),
        "other_workloads": {k: summary(r, r.get("ms_fwd") is not None) for k, r in others.items()},
    }


def kernel_table(breakdown, r, peaks, peak_src, steps, ms_step, wname):
    """Per-kernel time per step from the event trace, with the algorithmic work
    and roofline fraction of every kernel whose work is defined; and the
    roofline object of the dominant kernel (the one with the most time). Work
    and time are per step: a dense-backup GEMM is launched on both GEMM engines
    (the one that does not own the device-side row count returns at once), so
    its per-step work is set against both launches' time."""
    M, d, f, T, K = r["shape"]
    table = {}
    for k, v in sorted(breakdown.items(), key=lambda kv: -kv[1]["ms"]):
        row = {"launches_per_step": v["launches"] / steps, "ms_per_step": v["ms_per_step"]}
        bound, work = kernel_work(k, M, d, f, T, K, r["kept"], r["pairs"], r["n_ovf"], r["dense_wgrad"])
        if bound:
            peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) if bound == "tensor" else peaks["hbm_gbs"]
            achieved = work / (v["ms_per_step"] / 1e3) / (1e12 if bound == "tensor" else 1e9)
            row.update({"bound": bound, "work_per_step": work, "achieved": achieved,
                        "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": achieved / peak})
        table[k] = row
    roofline = None
    if breakdown:
        top = max(breakdown, key=lambda k: breakdown[k]["ms"])
        row = table[top]
        bound = row.get("bound")
        peak = None
        if bound:
            peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) if bound == "tensor" else peaks["hbm_gbs"]
        roofline = {"kernel": top, "bound": bound, "achieved": row.get("achieved"), "peak": peak,
                    "unit": row.get("unit"), "frac": row.get("frac"), "traffic": committed_traffic(top, wname),
                    "peak_source": f"{peak_src} ({'sustained bf16' if bound == 'tensor' else 'HBM copy'}, "
                                   "MEASURED_PEAKS.json)",
                    "work_per_step": row.get("work_per_step"),
                    "share_of_step": breakdown[top]["ms_per_step"] / ms_step if ms_step else None}
    return table, roofline


# ---------------------------------------------------------------- sweep


def _sweep_inputs(torch, dev, M, sp, d, f, sigma, bias):
    """Seeded sweep-point inputs drawn on the device: X rows scaled by lognormal(0, sigma)."""
    g = torch.Generator(device=dev)
    g.manual_seed(1000003 * M + int(round(sp * 1e4)))
    rs = torch.exp(sigma * torch.randn(M, 1, device=dev, generator=g))
    X = (torch.randn(M, d, device=dev, generator=g) * rs).to(torch.bfloat16)
    W_g = (torch.randn(f, d, device=dev, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W_u = (torch.randn(f, d, device=dev, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W_d = (torch.randn(d, f, device=dev, generator=g) / math.sqrt(f)).to(torch.bfloat16)
    dY = torch.randn(M, d, device=dev, generator=g).to(torch.bfloat16)
    b_g = torch.full((f,), bias, device=dev).to(torch.bfloat16)
    return X, W_g, W_u, W_d, dY, b_g, rs


def run_ksweep(args, local):
    """At each sweep point, the TwELL forward and forward+backward for every K of
    --sweep-k, next to the K that the count statistics and the cost model
    (activation_sparse_ffn_gemm_b200.kchoice) choose for training and inference."""
    import torch

    import activation_sparse_ffn_gemm_b200 as tw
    from synthetic import gate_bias_for_activity

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    d, f, T_n, sigma = 4096, 14336, 128, 0.75
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    steps, warm = max(1, args.steps), max(3, args.warmup)
    ks = [int(v) for v in args.sweep_k.split(",")]

    def timed(body):
        for _ in range(warm):
            body()
        torch.cuda.synchronize(dev)
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            body()
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / steps

    for sp in (float(v) for v in args.sweep_sparsity.split(",")):
        bias = gate_bias_for_activity(1.0 - sp, "lognormal", sigma)
        for M in (int(v) for v in args.sweep_m.split(",")):
            X, W_g, W_u, W_d, dY, b_g, rs = _sweep_inputs(torch, dev, M, sp, d, f, sigma, bias)
            Wdt = tw.transpose_wd(W_d)
            Y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
            per_k, stats = {}, None
            for K in ks:
                st = tw.HybridState(M, f, T_n, K, M, dev, with_u=True)
                wsf = tw.workspace(tw.OP_FWD, M, d, f, T_n, K, M, dev)
                wsb = tw.workspace(tw.OP_BWD, M, d, f, T_n, K, M, dev)
                grads = dict(dX=torch.empty((M, d), device=dev), dW_g=torch.empty((f, d), device=dev),
                             dW_u=torch.empty((f, d), device=dev), dW_d=torch.empty((d, f), device=dev),
                             db_g=torch.empty(f, device=dev))

                def fwd():
                    tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=T_n, K=K, W_dt=Wdt, state=st, ws=wsf, Y=Y)

                def fwd_bwd():
                    fwd()
                    tw.ffn_bwd(X, W_g, W_u, W_d, st, dY, lam=args.lam, W_dt=Wdt, ws=wsb, out=grads)

                t_fwd, t_fb = timed(fwd), timed(fwd_bwd)
                assert st.read_status() == 0, "device status word set"
                if stats is None:
                    stats = {k: v.cpu().numpy() for k, v in tw.count_stats(st).items()}
                per_k[K] = {"fwd_ms": t_fwd, "fwd_bwd_ms": t_fb, "overflow_rows": st.n_overflow()[1],
                            "dense_wgrad_for_overflow_rows": int(st.row_plan[3].item())}
                del st, wsf, wsb, grads
            del X, W_g, W_u, W_d, dY, b_g, rs, Wdt, Y
            torch.cuda.empty_cache()
            k_train, m_train = tw.suggest_k(stats, d, f, T_n, ks, training=True)
            k_inf, m_inf = tw.suggest_k(stats, d, f, T_n, ks, training=False)
            print(json.dumps({
                "point": {"M": M, "sparsity": sp, "d_model": d, "d_ff": f, "T_n": T_n},
                "per_k": per_k,
                "measured_best": {"fwd_bwd": min(per_k, key=lambda k: per_k[k]["fwd_bwd_ms"]),
                                  "fwd": min(per_k, key=lambda k: per_k[k]["fwd_ms"])},
                "suggested": {"fwd_bwd": k_train, "fwd": k_inf},
                "modelled_ms": {"fwd_bwd": {k: v * 1e3 for k, v in m_train.items()},
                                "fwd": {k: v * 1e3 for k, v in m_inf.items()}},
                "steps": steps, "warmup": warm, "l2": "flushed before every timed step",
                "data": "synthetic (seeded torch CUDA generator)"}), flush=True)


def run_sweep(args, local):
    """Forward and forward+backward time of TwELL and dense bf16 per (M, sparsity) point."""
    import torch

    import activation_sparse_ffn_gemm_b200 as tw
    from synthetic import gate_bias_for_activity, sweep_k

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    d, f, T_n, sigma = 4096, 14336, 128, 0.75
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    steps, warm = max(1, args.steps), max(3, args.warmup)

    def timed(body):
        for _ in range(warm):
            body()
        torch.cuda.synchronize(dev)
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            body()
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / steps

    for sp in (float(v) for v in args.sweep_sparsity.split(",")):
        p = 1.0 - sp
        K = sweep_k(p, T_n)
        bias = gate_bias_for_activity(p, "lognormal", sigma)
        for M in (int(v) for v in args.sweep_m.split(",")):
            X, W_g, W_u, W_d, dY, b_g, rs = _sweep_inputs(torch, dev, M, sp, d, f, sigma, bias)
            st = tw.HybridState(M, f, T_n, K, M, dev, with_u=True)
            wsf = tw.workspace(tw.OP_FWD, M, d, f, T_n, K, M, dev)
            wsb = tw.workspace(tw.OP_BWD, M, d, f, T_n, K, M, dev)
            Wdt = torch.empty((f, d), dtype=torch.bfloat16, device=dev)
            Y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
            grads = dict(dX=torch.empty((M, d), device=dev), dW_g=torch.empty((f, d), device=dev),
                         dW_u=torch.empty((f, d), device=dev), dW_d=torch.empty((d, f), device=dev),
                         db_g=torch.empty(f, device=dev))

            def fwd():
                tw.transpose_wd(W_d, out=Wdt)
                tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=T_n, K=K, W_dt=Wdt, state=st, ws=wsf, Y=Y)

            def fwd_bwd():
                fwd()
                tw.ffn_bwd(X, W_g, W_u, W_d, st, dY, lam=args.lam, W_dt=Wdt, ws=wsb, out=grads)

            t_fwd = timed(fwd)
            t_fb = timed(fwd_bwd)
            assert st.read_status() == 0, "device status word set"
            n_ovf = st.n_overflow()[1]
            cnt = st.count.float()
            activity = float(cnt.sum().item()) / (M * f)
            ratio = float(cnt.max().item()) / max(float(cnt.mean().item()), 1e-30)
            dense_wgrad = int(st.row_plan[3].item())

            # the same forward with per-(row, tile) overflow routing (inference only)
            st_t = tw.HybridState(M, f, T_n, K, M, dev, with_u=False)

            def fwd_tiles():
                tw.transpose_wd(W_d, out=Wdt)
                tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=T_n, K=K, W_dt=Wdt, state=st_t, ws=wsf, Y=Y, tile_routing=True)

            t_fwd_tiles = timed(fwd_tiles)
            assert st_t.read_status() == 0, "device status word set"
            del st, st_t, wsf, wsb

            # adaptive routing: the cost model's dense-row threshold and the K that the
            # batch's count statistics choose (kchoice), for training and for inference
            adaptive = {}
            for mode, training in (("fwd_bwd", True), ("fwd", False)):
                dm = tw.dense_min_for(d, f, training)
                probe = tw.HybridState(M, f, T_n, 8, M, dev, with_u=False, dense_min=dm)
                tw.pack(X, W_g, b_g, T_n=T_n, K=8, state=probe)
                K_a = tw.suggest_k(tw.count_stats(probe), d, f, T_n, training=training)[0]
                del probe
                st_a = tw.HybridState(M, f, T_n, K_a, M, dev, with_u=training, dense_min=dm)
                wsf_a = tw.workspace(tw.OP_FWD, M, d, f, T_n, K_a, M, dev)
                wsb_a = tw.workspace(tw.OP_BWD, M, d, f, T_n, K_a, M, dev) if training else None

                def body():
                    tw.transpose_wd(W_d, out=Wdt)
                    tw.ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=T_n, K=K_a, W_dt=Wdt, state=st_a, ws=wsf_a, Y=Y)
                    if training:
                        tw.ffn_bwd(X, W_g, W_u, W_d, st_a, dY, lam=args.lam, W_dt=Wdt, ws=wsb_a, out=grads)

                adaptive[mode] = {"ms": timed(body), "K": K_a, "dense_min": dm,
                                  "overflow_rows": st_a.n_overflow()[1]}
                assert st_a.read_status() == 0, "device status word set"
                del st_a, wsf_a, wsb_a
            del grads, Wdt, Y

            Wg_r, Wu_r, Wd_r = (t.clone().requires_grad_() for t in (W_g, W_u, W_d))
            Xr = X.clone().requires_grad_()

            def dense_fwd():
                with torch.no_grad():
                    (torch.relu(X @ W_g.T + b_g) * (X @ W_u.T)) @ W_d.T

            def dense_fb():
                z = Xr @ Wg_r.T + b_g
                gg = torch.relu(z)
                y = (gg * (Xr @ Wu_r.T)) @ Wd_r.T
                (y.float() * dY.float()).sum().add(gg.float().sum() * args.lam).backward()
                Xr.grad = Wg_r.grad = Wu_r.grad = Wd_r.grad = None

            t_dfwd = timed(dense_fwd)
            t_dfb = timed(dense_fb)
            del Wg_r, Wu_r, Wd_r, Xr, X, W_g, W_u, W_d, dY, b_g, rs
            torch.cuda.empty_cache()
            print(json.dumps({
                "point": {"M": M, "sparsity": sp, "d_model": d, "d_ff": f, "T_n": T_n, "K": K},
                "twell": {"fwd_ms": t_fwd, "fwd_bwd_ms": t_fb, "fwd_tokens_per_s": M / (t_fwd / 1e3),
                          "fwd_bwd_tokens_per_s": M / (t_fb / 1e3), "dense_wgrad_for_overflow_rows": dense_wgrad},
                "twell_tile_routing": {"fwd_ms": t_fwd_tiles, "fwd_tokens_per_s": M / (t_fwd_tiles / 1e3)},
                "twell_adaptive": adaptive,
                "dense_bf16": {"fwd_ms": t_dfwd, "fwd_bwd_ms": t_dfb},
                "speedup_vs_dense": {"fwd": t_dfwd / t_fwd, "fwd_bwd": t_dfb / t_fb,
                                     "adaptive_fwd": t_dfwd / adaptive["fwd"]["ms"],
                                     "adaptive_fwd_bwd": t_dfb / adaptive["fwd_bwd"]["ms"]},
                "measured": {"activity": activity, "overflow_rows": n_ovf, "max_over_mean_count": ratio},
                "steps": steps, "warmup": warm, "data": "synthetic (seeded torch CUDA generator)",
                "l2": "flushed before every timed step"}), flush=True)


def run_block(args, local):
    """One pre-norm transformer block (RMSNorm, causal multi-head attention, RMSNorm,
    gated ReLU FFN, residuals) with random weights, its FFN either the dense bf16
    FFN or the TwELL FFN (twell_ffn, K=8, L1 lambda), forward and forward+backward.
    Puts the FFN-level speed-up in the context of a whole block: the pages quote
    end-to-end model speed-ups (+20.5% inference, +21.9% training on H100)."""
    import torch
    import torch.nn.functional as F

    import activation_sparse_ffn_gemm_b200 as tw
    from synthetic import gate_bias_for_activity

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    B, S, d, heads, f, K = 2, 2048, 2048, 16, 8192, 8
    M = B * S
    g = torch.Generator(device=dev)
    g.manual_seed(20250)

    def param(*shape, scale):
        return (torch.randn(*shape, device=dev, generator=g) * scale).to(torch.bfloat16).requires_grad_()

    W_qkv, W_o = param(3 * d, d, scale=d ** -0.5), param(d, d, scale=d ** -0.5)
    W_g, W_u, W_d = param(f, d, scale=d ** -0.5), param(f, d, scale=d ** -0.5), param(d, f, scale=f ** -0.5)
    b_g = torch.full((f,), gate_bias_for_activity(0.01), device=dev).to(torch.bfloat16).requires_grad_()
    n1, n2 = torch.ones(d, device=dev, dtype=torch.bfloat16), torch.ones(d, device=dev, dtype=torch.bfloat16)
    x = torch.randn(B, S, d, device=dev, generator=g).to(torch.bfloat16)
    dY = torch.randn(B, S, d, device=dev, generator=g).to(torch.bfloat16)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def rms(t, w):
        return (t.float() * torch.rsqrt(t.float().pow(2).mean(-1, keepdim=True) + 1e-6)).to(torch.bfloat16) * w

    def block(inp, ffn):
        q, k, v = (rms(inp, n1) @ W_qkv.T).view(B, S, 3, heads, d // heads).permute(2, 0, 3, 1, 4)
        a = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B, S, d)
        h = inp + a @ W_o.T
        return h + ffn(rms(h, n2))

    def dense_ffn(t):
        return (torch.relu(t @ W_g.T + b_g) * (t @ W_u.T)) @ W_d.T

    def twell_k(k_):
        def ffn(t):
            return tw.twell_ffn(t, W_g, b_g, W_u, W_d, K=k_, lam=args.lam)
        return ffn

    def timed(body):
        for _ in range(max(3, args.warmup)):
            body()
        torch.cuda.synchronize(dev)
        tot = 0.0
        for _ in range(max(1, args.steps)):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            body()
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / max(1, args.steps)

    def fwd(ffn):
        def body():
            with torch.no_grad():
                block(x, ffn)
        return body

    def train(ffn):
        def body():
            xi = x.detach().requires_grad_()
            (block(xi, ffn).float() * dY.float()).sum().backward()
            for p_ in (W_qkv, W_o, W_g, W_u, W_d, b_g):
                p_.grad = None
        return body

    with torch.no_grad():
        hn = rms(block(x, lambda t: torch.zeros_like(t)), n2).reshape(M, d)  # the FFN input of this block
        activity = float(((hn @ W_g.T + b_g) > 0).float().mean().item())
        # adaptive K: the count statistics of this batch's pack and the cost model (kchoice)
        probe = tw.HybridState(M, f, 128, K, M, dev, with_u=False)
        tw.pack(hn.contiguous(), W_g.detach(), b_g.detach(), T_n=128, K=K, state=probe)
        stats = tw.count_stats(probe)
        k_train = tw.suggest_k(stats, d, f, training=True)[0]
        k_inf = tw.suggest_k(stats, d, f, training=False)[0]
        overflow_k8 = probe.n_overflow()[1]
        del probe
    res = {}
    arms = (("dense_ffn", dense_ffn, dense_ffn), ("twell_ffn_k8", twell_k(K), twell_k(K)),
            ("twell_ffn_adaptive_k", twell_k(k_inf), twell_k(k_train)))
    for name, ffn_inf, ffn_train in arms:
        res[name] = {"fwd_ms": timed(fwd(ffn_inf)), "fwd_bwd_ms": timed(train(ffn_train))}
        res[name]["fwd_tokens_per_s"] = M / (res[name]["fwd_ms"] / 1e3)
        res[name]["fwd_bwd_tokens_per_s"] = M / (res[name]["fwd_bwd_ms"] / 1e3)
    res["twell_ffn_adaptive_k"]["K"] = {"fwd": k_inf, "fwd_bwd": k_train}
    print(json.dumps({
        "workload": f"pre-norm transformer block, batch {B} x seq {S} (M={M} tokens), d_model={d}, {heads} heads, "
                    f"causal SDPA attention (torch), gated ReLU FFN d_ff={f}; TwELL FFN with T_n=128, K={K} or the "
                    f"K chosen from the batch's count statistics, L1 lambda={args.lam}",
        "ffn_gate_activity": activity,
        "ffn_overflow_rows_at_k8": overflow_k8,
        "block": res,
        "speedup_vs_dense_block": {
            arm: {"fwd": res["dense_ffn"]["fwd_ms"] / res[arm]["fwd_ms"],
                  "fwd_bwd": res["dense_ffn"]["fwd_bwd_ms"] / res[arm]["fwd_bwd_ms"]}
            for arm in ("twell_ffn_k8", "twell_ffn_adaptive_k")},
        "steps": args.steps, "warmup": max(3, args.warmup), "l2": "flushed before every timed step",
        "data": "synthetic (random weights, seeded torch CUDA generator)"}), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_env()
    if args.impl != "reference" and (args.sched != "auto" or args.l2_budget_mib or args.overlap != "auto"):
        apply_schedule(args)
    if args.block:
        run_block(args, local)
    elif args.sweep and args.sweep_k:
        run_ksweep(args, local)
    elif args.sweep:
        run_sweep(args, local)
    elif args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_twell(args, world, rank, local)


if __name__ == "__main__":
    main()
