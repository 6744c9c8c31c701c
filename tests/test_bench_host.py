"""Host logic of bench.py, without a GPU: the clock sampler's summary (with a
fake NVML), the algorithmic work per kernel, the whole-step roofline and the
committed DRAM-traffic records."""

import json
import sys
import time
import types

import pytest

import bench


class _FakeNVML(types.ModuleType):
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons):
        super().__init__("pynvml")
        self.clocks, self.reasons, self.i = clocks, reasons, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        raise RuntimeError("no CUDA device here")

    def nvmlDeviceGetHandleByIndex(self, index):
        return ("gpu", index)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.clocks[min(self.i, len(self.clocks) - 1)]
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        r = self.reasons[min(self.i, len(self.reasons) - 1)]
        self.i += 1
        return r


def test_clock_sampler_polls_nvml(monkeypatch):
    fake = _FakeNVML([1800, 1950, 1965, 1965, 1965], [0, 0x4, 0, 0, 0])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as clk:
        t0 = time.time()
        while len(clk.samples) < 5 and time.time() - t0 < 5:
            time.sleep(0.005)
    s = clk.summary()
    assert s["source"].startswith("nvml") and s["samples"] >= 5
    assert s["sm_max_mhz"] == 1965.0 and s["sm_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_reasons_by_bit():
    clk = bench.ClockSampler(0)
    clk.nvml = object()
    clk.max_mhz = 1965.0
    clk.samples = [(1300.0, 0x8 | 0x40), (1310.0, 0x20), (1320.0, 0)]
    s = clk.summary()
    assert s["sm_mhz"] == 1310.0
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_kernel_work_by_hand():
    M, d, f, T, K, kept, pairs = 4, 8, 256, 2, 8, 10, 12
    assert bench.kernel_work("gate_pack_gemm", M, d, f, T, K, kept, pairs) == ("tensor", 2.0 * 4 * 8 * 256)
    # X + TwELL + u + Y + W_u and W_dt once
    assert bench.kernel_work("ell_updown", M, d, f, T, K, kept, pairs) == (
        "hbm", 2 * 32 + 4 * 2 * 26 + 40 + 2 * 32 + 4 * 256 * 8)
    # dY, TwELL, u, (h, dU, dZ, 0) per slot, dX fp32, three weight matrices once
    assert bench.kernel_work("ell_bwd", M, d, f, T, K, kept, pairs) == (
        "hbm", 2 * 32 + 4 * 2 * 26 + 40 + 160 + 4 * 32 + 6 * 256 * 8)
    # one overflow row: the ELL rows are the other three
    assert bench.kernel_work("ell_updown", M, d, f, T, K, kept, pairs, n_ovf=1) == (
        "hbm", 2 * 24 + 3 * 2 * 26 + 40 + 2 * 24 + 4 * 256 * 8)
    assert bench.kernel_work("ovf_dx_gemm", M, d, f, T, K, kept, pairs, n_ovf=3) == ("tensor", 4.0 * 3 * 8 * 256)
    assert bench.kernel_work("ovf_up_gemm", M, d, f, T, K, kept, pairs, n_ovf=3) == ("tensor", 2.0 * 3 * 8 * 256)
    # the pair list holds the overflow rows' pairs unless their gradients run as GEMMs
    sparse = bench.kernel_work("weight_grads", M, d, f, T, K, kept, pairs, n_ovf=1, dense_wgrad=0)[1]
    dense = bench.kernel_work("weight_grads", M, d, f, T, K, kept, pairs, n_ovf=1, dense_wgrad=1)[1]
    assert sparse == 4 * 32 + 20 * 12 + 12 * 256 * 8 + 4 * 256
    assert dense == 4 * 32 + 20 * 10 + 24 * 256 * 8 + 4 * 256
    assert bench.kernel_work("transpose_wd", M, d, f, T, K, kept, pairs) == ("hbm", 4 * 256 * 8)
    # the passes of the multi-pass schedule: the fused kernels' bytes split by pass (the
    # per-slot records written by one pass and read by the next counted on both sides)
    up = bench.kernel_work("ell_up", M, d, f, T, K, kept, pairs)[1]
    down = bench.kernel_work("ell_down", M, d, f, T, K, kept, pairs)[1]
    assert up == 2 * 32 + 4 * 2 * 26 + 40 + 2 * 256 * 8
    assert down == 4 * 2 * 26 + 40 + 2 * 32 + 2 * 256 * 8
    assert up + down == bench.kernel_work("ell_updown", M, d, f, T, K, kept, pairs)[1] + 4 * 2 * 26 + 40
    dh = bench.kernel_work("ell_dh", M, d, f, T, K, kept, pairs)[1]
    dx = bench.kernel_work("ell_dx", M, d, f, T, K, kept, pairs)[1]
    assert dh == 2 * 32 + 4 * 2 * 26 + 40 + 160 + 2 * 256 * 8
    assert dx == 4 * 2 * 10 + 160 + 4 * 32 + 4 * 256 * 8
    assert bench.kernel_work("row_flags", M, d, f, T, K, kept, pairs) == (None, None)


def test_path_roofline_fractions():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 2.0, "bf16_tflops_sustained": 1.0}
    r = bench.path_roofline(M=128, d=64, f=256, T=2, K=8, kept=100, n_ovf=0, peaks=peaks, ms_fwd=2.0, ms_step=5.0)
    assert r["step_ms"] > r["fwd_ms"] > 0
    assert r["fwd_frac"] == pytest.approx(r["fwd_ms"] / 2.0) and r["step_frac"] == pytest.approx(r["step_ms"] / 5.0)
    # the gate GEMM's flops at the sustained rate are part of the forward's floor
    assert r["fwd_ms"] >= 2.0 * 128 * 64 * 256 / 1e12 * 1e3


def test_committed_traffic_follows_the_sources(monkeypatch):
    with open(bench.os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as fh:
        wls = json.load(fh)["workloads"]
    assert wls
    for wname, wrec in wls.items():
        for k, v in wrec["kernels"].items():
            got = bench.committed_traffic(k, wname)
            if v["source_sha"] == bench.source_hash(k):
                assert got == v["dram_bytes_per_launch"]
            else:
                assert got is None
    assert bench.committed_traffic("gate_pack_gemm", "no such workload") is None
    monkeypatch.setattr(bench, "source_hash", lambda kernel: "changed")
    assert all(bench.committed_traffic(k, wname) is None for wname, wrec in wls.items() for k in wrec["kernels"])


def test_workloads_of_the_line():
    """The timed training step runs the largest single-GPU sweep point at 99% sparsity;
    the uniform inference workload keeps its golden seed."""
    w, seed = bench.workload()
    assert (w.M, w.d_model, w.d_ff, w.T_n, w.K, w.activity, w.row_scale) == (
        65536, 4096, 14336, 128, 8, 0.01, "lognormal")
    assert "M=65536" in bench.workload_desc(w, seed) and "99% sparsity" in bench.workload_desc(w, seed)
    for name, M in (("sweep8k", 8192), ("sweep2k", 2048), ("sweep512", 512)):
        w, _ = bench.workload(name)
        assert (w.M, w.d_model, w.d_ff, w.K, w.activity, w.row_scale, w.training) == (
            M, 4096, 14336, 8, 0.01, "lognormal", True)
    w, seed = bench.workload("uniform")
    assert (w.M, w.d_model, w.d_ff, w.T_n, w.K, w.activity) == (4096, 2048, 8192, 128, 8, 0.01)
    with open(bench.os.path.join(bench.ROOT, "tests", "golden", "uniform_seed.json")) as fh:
        assert seed == json.load(fh)["seed"]
    assert bench.ovf_cap_for(w) == 1024


def test_kernel_table_and_dominant_kernel():
    """Per-kernel fractions from the event trace; the roofline object is the kernel with the most time."""
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 2.0, "bf16_tflops_sustained": 1.0}
    r = {"shape": (128, 64, 256, 2, 8), "kept": 100, "pairs": 120, "n_ovf": 2, "dense_wgrad": 0}
    bd = {"gate_pack_gemm": {"launches": 2, "ms": 4.0, "ms_per_launch": 2.0, "ms_per_step": 2.0},
          "ovf_up_gemm": {"launches": 4, "ms": 1.0, "ms_per_launch": 0.25, "ms_per_step": 0.5},
          "ell_updown": {"launches": 2, "ms": 1.0, "ms_per_launch": 0.5, "ms_per_step": 0.5},
          "row_flags": {"launches": 2, "ms": 0.1, "ms_per_launch": 0.05, "ms_per_step": 0.05}}
    table, roof = bench.kernel_table(bd, r, peaks, "measured", 2, 4.0, "large")
    assert list(table) == ["gate_pack_gemm", "ovf_up_gemm", "ell_updown", "row_flags"]
    # two launches per step (both GEMM engines): the step's work against the step's time
    assert table["ovf_up_gemm"]["achieved"] == pytest.approx(2.0 * 2 * 64 * 256 / 0.5e-3 / 1e12)
    flops = 2.0 * 128 * 64 * 256
    assert table["gate_pack_gemm"]["achieved"] == pytest.approx(flops / 2e-3 / 1e12)
    assert table["gate_pack_gemm"]["frac"] == pytest.approx(flops / 2e-3 / 1e12 / 1.0)
    assert "frac" not in table["row_flags"]
    assert roof["kernel"] == "gate_pack_gemm" and roof["bound"] == "tensor" and roof["peak"] == 1.0
    assert roof["share_of_step"] == pytest.approx(0.5)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON
    line with the contract's keys; a tiny --cpu-seconds keeps the sample small."""
    import subprocess

    out = subprocess.run([sys.executable, bench.os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "train", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.05"],
                         capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_schedule_flags_reach_the_library(monkeypatch):
    """--sched, --l2-budget-mib and --overlap set the process-wide schedule and overlap
    through the binding (no GPU: the binding's setters are replaced)."""
    import activation_sparse_ffn_gemm_b200 as tw

    calls = []
    monkeypatch.setattr(tw, "set_sparse_schedule", lambda mode, budget: calls.append(("sched", mode, budget)))
    monkeypatch.setattr(tw, "set_overlap", lambda mode: calls.append(("overlap", mode)))
    for argv, want in ((["--sched", "passes", "--l2-budget-mib", "32", "--overlap", "on"],
                        [("sched", tw.SCHED_PASSES, 32 << 20), ("overlap", tw.OVERLAP_ON)]),
                       (["--sched", "fused", "--overlap", "off"],
                        [("sched", tw.SCHED_FUSED, 0), ("overlap", tw.OVERLAP_OFF)]),
                       ([], [("sched", tw.SCHED_AUTO, 0), ("overlap", tw.OVERLAP_AUTO)])):
        calls.clear()
        monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
        bench.apply_schedule(bench.parse_args())
        assert calls == want, argv
