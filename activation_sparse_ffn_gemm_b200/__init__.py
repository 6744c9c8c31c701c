"""Python binding of libtwell, the sm_100a TwELL activation-sparse gated FFN.

Argument marshalling only: every step runs in the CUDA library declared in
include/twell.h. PyTorch supplies device memory and the current CUDA stream.
There is no fallback: if libtwell.so is missing or a call fails, an exception
is raised.

    Y, st = ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=128, K=8)
    grads = ffn_bwd(X, W_g, W_u, W_d, st, dY, lam=1e-3)
"""

from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Optional

import torch

from .kchoice import CostModel, dense_min_for, modelled_times, suggest_k  # noqa: F401

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtwell.so")
# the same library compiled with -DTWELL_BOUNDS (index checks, STATUS_BOUNDS); see bounds_checked()
BOUNDS_LIB_PATH = os.path.join(_PKG, "libtwell_bounds.so")

OP_PACK, OP_FWD, OP_BWD = 0, 1, 2
STATUS_OVERFLOW_CAP = 1 << 3
STATUS_TIMEOUT = 1 << 5
STATUS_BAD_STATE = 1 << 1  # a tile-routed (inference) state given to the backward
STATUS_BOUNDS = 1 << 7  # bounds-checked build only: an index read from a buffer was out of range
_STATUS_NAMES = {0: "TWELL_OK", 1: "TWELL_EINVAL", 2: "TWELL_EUNSUPPORTED", 3: "TWELL_EOVERFLOW_CAP",
                 4: "TWELL_ECUDA", 5: "TWELL_ETIMEOUT", 6: "TWELL_EWORKSPACE", 7: "TWELL_EBOUNDS"}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


class TwellError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_STATUS_NAMES.get(code, code)} ({lib().twell_status_string(code).decode()})")


class TwellTraceRec(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("ms", ctypes.c_float)]


class TwellHybrid(ctypes.Structure):
    """Mirror of struct twell_hybrid."""

    _fields_ = [("M", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("T_n", ctypes.c_int32), ("K", ctypes.c_int32),
                ("ovf_cap", ctypes.c_int32), ("dense_min", ctypes.c_int32), ("count", _vp), ("val", _vp),
                ("col", _vp), ("row_ovf", _vp), ("ovf_rows", _vp), ("n_ovf", _vp), ("g_ovf", _vp), ("u_ell", _vp),
                ("u_ovf", _vp), ("status", _vp), ("row_plan", _vp)]


_lock = threading.RLock()
_libs = {}
_use_bounds = 0


def lib():
    """Loads libtwell.so (built in-tree by activation_sparse_ffn_gemm_b200.build),
    or libtwell_bounds.so inside a bounds_checked() block."""
    with _lock:
        path = BOUNDS_LIB_PATH if _use_bounds else LIB_PATH
        L = _libs.get(path)
        if L is None:
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m activation_sparse_ffn_gemm_b200.build`")
            L = ctypes.CDLL(path)
            L.twell_status_string.restype = ctypes.c_char_p
            L.twell_status_string.argtypes = [ctypes.c_int]
            L.twell_query_support.restype = ctypes.c_int
            L.twell_query_support.argtypes = [_i64] * 6
            L.twell_plan_ints.restype = ctypes.c_size_t
            L.twell_plan_ints.argtypes = [_i64] * 4
            L.twell_workspace_bytes.restype = ctypes.c_size_t
            L.twell_workspace_bytes.argtypes = [ctypes.c_int] + [_i64] * 6
            L.twell_transpose_wd.restype = ctypes.c_int
            L.twell_transpose_wd.argtypes = [_vp, _i64, _i64, _vp, _vp]
            L.twell_pack.restype = ctypes.c_int
            L.twell_pack.argtypes = [_vp, _vp, _vp, _i64, ctypes.POINTER(TwellHybrid), _vp, _vp, ctypes.c_size_t, _vp]
            L.twell_pack_noalloc.restype = ctypes.c_int
            L.twell_pack_noalloc.argtypes = [_vp, _vp, _vp, _i64, ctypes.POINTER(TwellHybrid), _vp, _vp]
            L.twell_ffn_fwd.restype = ctypes.c_int
            L.twell_ffn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, ctypes.POINTER(TwellHybrid), _vp,
                                        _vp, ctypes.c_size_t, _vp]
            L.twell_ffn_fwd_tiles.restype = ctypes.c_int
            L.twell_ffn_fwd_tiles.argtypes = L.twell_ffn_fwd.argtypes
            L.twell_quantize_e4m3_rows.restype = ctypes.c_int
            L.twell_quantize_e4m3_rows.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp]
            L.twell_ffn_fwd_e4m3.restype = ctypes.c_int
            L.twell_ffn_fwd_e4m3.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp,
                                             ctypes.POINTER(TwellHybrid), _vp, _vp, ctypes.c_size_t, _vp]
            L.twell_ffn_bwd.restype = ctypes.c_int
            L.twell_ffn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, ctypes.POINTER(TwellHybrid), _vp,
                                        ctypes.c_float, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
            L.twell_launch_count.restype = ctypes.c_uint64
            L.twell_launch_count.argtypes = []
            L.twell_trace_enable.restype = None
            L.twell_trace_enable.argtypes = [ctypes.c_int]
            L.twell_trace_collect.restype = ctypes.c_int
            L.twell_trace_collect.argtypes = [ctypes.POINTER(TwellTraceRec), ctypes.c_int]
            L.twell_count_stats.restype = ctypes.c_int
            L.twell_count_stats.argtypes = [ctypes.POINTER(TwellHybrid), _vp, _vp, _vp, _vp]
            L.twell_test_withhold_epilogue_arrival.restype = None
            L.twell_test_withhold_epilogue_arrival.argtypes = [ctypes.c_int]
            L.twell_set_sparse_schedule.restype = ctypes.c_int
            L.twell_set_sparse_schedule.argtypes = [ctypes.c_int, _i64]
            L.twell_set_overlap.restype = ctypes.c_int
            L.twell_set_overlap.argtypes = [ctypes.c_int]
            L.twell_status_read.restype = ctypes.c_int
            L.twell_status_read.argtypes = [ctypes.POINTER(TwellHybrid), ctypes.POINTER(ctypes.c_uint32),
                                            ctypes.c_int, _vp]
            _libs[path] = L
    return L


@contextlib.contextmanager
def bounds_checked():
    """Within the block every call of this binding runs in libtwell_bounds.so, the
    library compiled with index checks: each index a kernel reads from a buffer
    (in-tile column, piece row, overflow row, dense slot, pair-list row and
    position) is checked against the extent it addresses, and an index out of
    range sets STATUS_BOUNDS in the state's status word instead of being used.
    Results are otherwise those of libtwell.so (the checks change no arithmetic).
    A test and debugging aid (compute-sanitizer stands in for nothing here)."""
    global _use_bounds
    with _lock:
        _use_bounds += 1
    try:
        yield lib()
    finally:
        with _lock:
            _use_bounds -= 1


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, what: str) -> None:
    if code != 0:
        raise TwellError(code, what)


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous CUDA bfloat16 tensor")
    return t


def launch_count() -> int:
    """Kernels this library has launched in the process so far."""
    return int(lib().twell_launch_count())


def test_withhold_epilogue_arrival(launches: int) -> None:
    """Failure-detection test aid (twell_test_withhold_epilogue_arrival): the next
    `launches` split-capable dense-backup GEMM launches run with one epilogue warp
    that never reaches the split-K barrier, so its bounded wait runs out and the
    kernel sets TWELL_STATUS_TIMEOUT."""
    lib().twell_test_withhold_epilogue_arrival(int(launches))


SCHED_AUTO, SCHED_FUSED, SCHED_PASSES = 0, 1, 2


def set_sparse_schedule(mode: int = SCHED_AUTO, l2_budget_bytes: int = 0) -> None:
    """Schedule of the sparse kernels (twell_set_sparse_schedule): SCHED_FUSED,
    SCHED_PASSES (one pass per gathered weight matrix, chunked to
    l2_budget_bytes; 0 = the library's default) or SCHED_AUTO. Process-wide;
    the results are the same under every schedule."""
    _check(lib().twell_set_sparse_schedule(int(mode), int(l2_budget_bytes)), "twell_set_sparse_schedule")


OVERLAP_OFF, OVERLAP_ON, OVERLAP_AUTO = 0, 1, 2


def set_overlap(mode: int = OVERLAP_ON) -> None:
    """twell_set_overlap: run the dense-backup GEMMs on the library's side stream
    beside the sparse kernels (OVERLAP_ON, or True), everything on the caller's
    stream (OVERLAP_OFF, or False), or OVERLAP_AUTO (the default: on below 4096
    rows). Process-wide; the results are the same either way."""
    _check(lib().twell_set_overlap(int(mode)), "twell_set_overlap")


def trace_enable(on: bool = True) -> None:
    lib().twell_trace_enable(1 if on else 0)


def trace_collect(max_recs: int = 1 << 16) -> list:
    """[(kernel name, ms), ...] for the launches recorded since the last collect."""
    buf = (TwellTraceRec * max_recs)()
    n = lib().twell_trace_collect(buf, max_recs)
    return [(buf[i].name.decode(), float(buf[i].ms)) for i in range(min(n, max_recs))]


def query_support(M, d_model, d_ff, T_n, K, ovf_cap) -> int:
    return int(lib().twell_query_support(M, d_model, d_ff, T_n, K, ovf_cap))


def workspace_bytes(op: int, M: int, d_model: int, d_ff: int, T_n: int, K: int, ovf_cap: int) -> int:
    return int(lib().twell_workspace_bytes(op, M, d_model, d_ff, T_n, K, ovf_cap))


def workspace(op: int, M: int, d_model: int, d_ff: int, T_n: int, K: int, ovf_cap: int, device=None,
              alloc=None) -> torch.Tensor:
    """Workspace of `op` for this shape; alloc(shape, dtype), when given, supplies
    the (256-byte aligned) memory instead of torch.empty on `device`."""
    n = workspace_bytes(op, M, d_model, d_ff, T_n, K, ovf_cap)
    if n == 0 and query_support(M, d_model, d_ff, T_n, K, ovf_cap) != 0:
        _check(query_support(M, d_model, d_ff, T_n, K, ovf_cap), "workspace")
    if alloc is not None:
        return alloc((max(n, 256),), torch.uint8)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


class HybridState:
    """Device buffers of one hybrid TwELL representation (see struct twell_hybrid)."""

    def __init__(self, M: int, d_ff: int, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None,
                 device=None, with_u: bool = True, dense_min: int = 0, alloc=None):
        """dense_min > 0 also routes rows with at least that many active units to
        the dense backup (kchoice.dense_min_for gives the measured break-even).
        alloc(shape, dtype), when given, supplies each array's (16-byte aligned)
        memory instead of torch.empty on `device`."""
        dev = torch.device(device or "cuda")
        if alloc is None:
            def alloc(shape, dtype):
                return torch.empty(shape, dtype=dtype, device=dev)
        T = d_ff // T_n
        cap = M if ovf_cap is None else int(ovf_cap)
        cap1 = max(cap, 1)
        self.M, self.d_ff, self.T_n, self.K, self.ovf_cap, self.dense_min = M, d_ff, T_n, K, cap, int(dense_min)
        self.count = alloc((M, T), torch.int16)
        self.val = alloc((M, T, K), torch.bfloat16)
        self.col = alloc((M, T, K), torch.uint8)
        self.row_ovf = alloc((max(M, 1),), torch.uint8)
        self.ovf_rows = alloc((cap1,), torch.int32)
        # n_ovf, the status word and the row plan start at zero: one buffer, one fill,
        # each part 16-byte aligned
        n_plan = max(int(lib().twell_plan_ints(M, d_ff, T_n, K)), 1)
        self._zeroed = alloc((8 + n_plan,), torch.int32)
        self._zeroed.zero_()
        self.n_ovf = self._zeroed[0:2]
        self.g_ovf = alloc((cap1, d_ff), torch.bfloat16)
        self.u_ell = alloc((M, T, K), torch.float32) if with_u else None
        self.u_ovf = alloc((cap1, d_ff), torch.float32) if with_u else None
        self.status = self._zeroed[4:8]
        self.row_plan = self._zeroed[8:]
        self.c = TwellHybrid(M, d_ff, T_n, K, cap, int(dense_min), *(
            (t.data_ptr() if t is not None else None) for t in
            (self.count, self.val, self.col, self.row_ovf, self.ovf_rows, self.n_ovf, self.g_ovf, self.u_ell,
             self.u_ovf, self.status, self.row_plan)))

    def read_status(self, clear: bool = False, stream=None) -> int:
        out = ctypes.c_uint32(0)
        _check(lib().twell_status_read(ctypes.byref(self.c), ctypes.byref(out), int(clear), _stream(stream)),
               "twell_status_read")
        return int(out.value)

    def n_overflow(self) -> tuple[int, int]:
        v = self.n_ovf.cpu().tolist()
        return int(v[0]), int(v[1])


def count_stats(state: HybridState, stream=None) -> dict:
    """Count statistics of a packed batch (twell_count_stats): int64 CUDA tensors
    rows_by_max, act_by_max, tiles_by_count of T_n + 2 bins each (bin T_n + 1:
    rows routed dense by the state's dense_min)."""
    n = state.T_n + 2
    dev = state.count.device
    out = {k: torch.empty(n, dtype=torch.int64, device=dev) for k in ("rows_by_max", "act_by_max", "tiles_by_count")}
    _check(lib().twell_count_stats(ctypes.byref(state.c), _ptr(out["rows_by_max"]), _ptr(out["act_by_max"]),
                                   _ptr(out["tiles_by_count"]), _stream(stream)), "twell_count_stats")
    return out


def transpose_wd(W_d: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _bf16(W_d, "W_d")
    d, f = W_d.shape
    out = torch.empty((f, d), dtype=torch.bfloat16, device=W_d.device) if out is None else out
    _check(lib().twell_transpose_wd(_ptr(W_d), d, f, _ptr(out), _stream(stream)), "twell_transpose_wd")
    return out


def pack(X, W_g, b_g, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None, z_debug: bool = False,
         state: Optional[HybridState] = None, ws: Optional[torch.Tensor] = None, stream=None, dense_min: int = 0):
    """Gate GEMM + TwELL pack + row routing. Returns (state, z or None)."""
    for t, n in ((X, "X"), (W_g, "W_g"), (b_g, "b_g")):
        _bf16(t, n)
    M, d = X.shape
    f = W_g.shape[0]
    st = state or HybridState(M, f, T_n, K, ovf_cap, X.device, with_u=False, dense_min=dense_min)
    z = torch.empty((M, f), dtype=torch.float32, device=X.device) if z_debug else None
    if ws is None:
        ws = workspace(OP_PACK, M, d, f, T_n, K, st.ovf_cap, X.device)
    _check(lib().twell_pack(_ptr(X), _ptr(W_g), _ptr(b_g), d, ctypes.byref(st.c), _ptr(z), _ptr(ws), ws.numel(),
                            _stream(stream)), "twell_pack")
    return st, z


NOALLOC_SCRATCH_BYTES = 16 << 20


def pack_noalloc(X, W_g, b_g, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None, z_debug: bool = False,
                 state: Optional[HybridState] = None, stream=None, dense_min: int = 0):
    """twell_pack_noalloc: the same result as pack() without a workspace; the
    library's own fixed scratch is used instead (M * d_ff * 2 bytes at most
    NOALLOC_SCRATCH_BYTES). Returns (state, z or None)."""
    for t, n in ((X, "X"), (W_g, "W_g"), (b_g, "b_g")):
        _bf16(t, n)
    M, d = X.shape
    f = W_g.shape[0]
    st = state or HybridState(M, f, T_n, K, ovf_cap, X.device, with_u=False, dense_min=dense_min)
    z = torch.empty((M, f), dtype=torch.float32, device=X.device) if z_debug else None
    _check(lib().twell_pack_noalloc(_ptr(X), _ptr(W_g), _ptr(b_g), d, ctypes.byref(st.c), _ptr(z), _stream(stream)),
           "twell_pack_noalloc")
    return st, z


def ffn_fwd(X, W_g, b_g, W_u, W_d, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None, W_dt=None,
            save_for_backward: bool = True, z_debug: bool = False, state: Optional[HybridState] = None,
            ws: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None, stream=None,
            tile_routing: bool = False, dense_min: int = 0):
    """Sparse gated FFN forward. Returns (Y, state) or (Y, state, z) with z_debug.

    tile_routing: per-(row, tile) overflow routing (twell_ffn_fwd_tiles), an
    inference-only state; otherwise the row-level hybrid (twell_ffn_fwd).
    dense_min: for a state made here, rows with at least this many active
    units also go to the dense backup (0: only rows with a tile over K)."""
    for t, n in ((X, "X"), (W_g, "W_g"), (b_g, "b_g"), (W_u, "W_u"), (W_d, "W_d")):
        _bf16(t, n)
    M, d = X.shape
    f = W_g.shape[0]
    st = state or HybridState(M, f, T_n, K, ovf_cap, X.device, with_u=save_for_backward, dense_min=dense_min)
    Y = torch.empty((M, d), dtype=torch.bfloat16, device=X.device) if Y is None else Y
    z = torch.empty((M, f), dtype=torch.float32, device=X.device) if z_debug else None
    if ws is None:
        ws = workspace(OP_FWD, M, d, f, T_n, K, st.ovf_cap, X.device)
    fn = lib().twell_ffn_fwd_tiles if tile_routing else lib().twell_ffn_fwd
    _check(fn(_ptr(X), _ptr(W_g), _ptr(b_g), _ptr(W_u), _ptr(W_d), _ptr(W_dt), d, _ptr(Y), ctypes.byref(st.c),
              _ptr(z), _ptr(ws), ws.numel(), _stream(stream)),
           "twell_ffn_fwd_tiles" if tile_routing else "twell_ffn_fwd")
    return (Y, st, z) if z_debug else (Y, st)


def quantize_e4m3_rows(W, with_deq: bool = True, stream=None):
    """twell_quantize_e4m3_rows: E4M3 codes [rows, len] (uint8), per-row scales
    2^e [rows] (float32) and, with_deq, the dequantised bf16 rows."""
    _bf16(W, "W")
    rows, length = W.shape
    q = torch.empty((rows, length), dtype=torch.uint8, device=W.device)
    sc = torch.empty(rows, dtype=torch.float32, device=W.device)
    deq = torch.empty_like(W) if with_deq else None
    _check(lib().twell_quantize_e4m3_rows(_ptr(W), rows, length, _ptr(q), _ptr(sc), _ptr(deq), _stream(stream)),
           "twell_quantize_e4m3_rows")
    return q, sc, deq


def quantize_weights(W_u, W_d, stream=None) -> dict:
    """8-bit copies of the gathered weights for ffn_fwd_e4m3: W_u8 / s_u (rows of
    W_u), W_dt8 / s_d (rows of W_d^T), and the dequantised bf16 W_u, W_d (the
    weights the computed FFN uses)."""
    W_u8, s_u, W_uq = quantize_e4m3_rows(W_u, stream=stream)
    W_dt8, s_d, W_dtq = quantize_e4m3_rows(transpose_wd(W_d, stream=stream), stream=stream)
    W_dq = torch.empty_like(W_d)
    d, f = W_d.shape
    # [d_ff][d_model] -> [d_model][d_ff]: the same transpose kernel with the roles of the extents swapped
    _check(lib().twell_transpose_wd(_ptr(W_dtq), f, d, _ptr(W_dq), _stream(stream)), "twell_transpose_wd")
    return dict(W_u8=W_u8, s_u=s_u, W_dt8=W_dt8, s_d=s_d, W_u=W_uq, W_d=W_dq)


def ffn_fwd_e4m3(X, W_g, b_g, q8: dict, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None,
                 save_for_backward: bool = False, z_debug: bool = False, state: Optional[HybridState] = None,
                 ws: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None, stream=None, dense_min: int = 0):
    """twell_ffn_fwd_e4m3: the forward with the sparse kernel's gathers reading the
    8-bit weights of q8 (from quantize_weights); the FFN computed is the one with
    weights (W_g, q8["W_u"], q8["W_d"]). Returns (Y, state) or (Y, state, z)."""
    for t, n in ((X, "X"), (W_g, "W_g"), (b_g, "b_g"), (q8["W_u"], "W_u"), (q8["W_d"], "W_d")):
        _bf16(t, n)
    M, d = X.shape
    f = W_g.shape[0]
    st = state or HybridState(M, f, T_n, K, ovf_cap, X.device, with_u=save_for_backward, dense_min=dense_min)
    Y = torch.empty((M, d), dtype=torch.bfloat16, device=X.device) if Y is None else Y
    z = torch.empty((M, f), dtype=torch.float32, device=X.device) if z_debug else None
    if ws is None:
        ws = workspace(OP_FWD, M, d, f, T_n, K, st.ovf_cap, X.device)
    _check(lib().twell_ffn_fwd_e4m3(_ptr(X), _ptr(W_g), _ptr(b_g), _ptr(q8["W_u"]), _ptr(q8["W_d"]), _ptr(q8["W_u8"]),
                                    _ptr(q8["s_u"]), _ptr(q8["W_dt8"]), _ptr(q8["s_d"]), d, _ptr(Y), ctypes.byref(st.c),
                                    _ptr(z), _ptr(ws), ws.numel(), _stream(stream)), "twell_ffn_fwd_e4m3")
    return (Y, st, z) if z_debug else (Y, st)


def ffn_bwd(X, W_g, W_u, W_d, state: HybridState, dY, lam: float = 0.0, W_dt=None, with_db: bool = True,
            ws: Optional[torch.Tensor] = None, out: Optional[dict] = None, stream=None) -> dict:
    """Backward over the hybrid format. Returns dict dX, dW_g, dW_u, dW_d[, db_g] (fp32)."""
    for t, n in ((X, "X"), (W_g, "W_g"), (W_u, "W_u"), (W_d, "W_d"), (dY, "dY")):
        _bf16(t, n)
    M, d = X.shape
    f = W_g.shape[0]
    dev = X.device
    if out is None:
        out = dict(dX=torch.empty((M, d), dtype=torch.float32, device=dev),
                   dW_g=torch.empty((f, d), dtype=torch.float32, device=dev),
                   dW_u=torch.empty((f, d), dtype=torch.float32, device=dev),
                   dW_d=torch.empty((d, f), dtype=torch.float32, device=dev))
        if with_db:
            out["db_g"] = torch.empty(f, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(OP_BWD, M, d, f, state.T_n, state.K, state.ovf_cap, dev)
    _check(lib().twell_ffn_bwd(_ptr(X), _ptr(W_g), _ptr(W_u), _ptr(W_d), _ptr(W_dt), d, ctypes.byref(state.c),
                               _ptr(dY), float(lam), _ptr(out["dX"]), _ptr(out["dW_g"]), _ptr(out["dW_u"]),
                               _ptr(out["dW_d"]), _ptr(out.get("db_g")), _ptr(ws), ws.numel(), _stream(stream)),
           "twell_ffn_bwd")
    return out


from .autograd import TwellFFNFunction, twell_ffn  # noqa: E402,F401
