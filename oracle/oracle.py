"""ctypes front end of the fp64 CPU oracle (twell_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product path. All arrays are numpy;
bfloat16 tensors are passed as uint16 bit patterns.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  bf16_round        pinned: torch's float32->bfloat16 RNE cast, hand-made ties
  gate              pinned: brute-force loops, torch float64 matmul
  pack / unpack     pinned: round trip, invariants, hand-built identity-gate case
  count_stats       pinned: hand-counted bins, brute-force loops, sum invariants
  ffn_fwd           pinned: brute-force loops, torch float64, closed forms
  ffn_fwd_hybrid    pinned: equals ffn_fwd (round_g=1) on the same active set
  ffn_bwd           pinned: torch float64 autograd, closed form of the L1 term
  ffn_bwd_units     pinned: equals ffn_bwd (C) on the listed units, given the same g
  gmat input        pinned: with gmat = the oracle's own packed g, equals round_g
  e4m3_value        pinned: torch's float8_e4m3fn reading of all 256 codes
  e4m3_round        pinned: brute-force nearest code with the tie rule; torch's cast
  quantize_e4m3     pinned: scale bounds, exact round trip, idempotence, a unit
                    already on the grid, zero units, both layouts agree
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "twell_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libtwell_oracle.so")
_lock = threading.Lock()
_lib = None

_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O3, no fused or re-associated arithmetic)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.oracle_bf16_round.restype = ctypes.c_uint16
            L.oracle_bf16_round.argtypes = [ctypes.c_double]
            L.oracle_bf16_round_array.argtypes = [_f64p, _u16p, _i64]
            L.oracle_bf16_to_double_array.argtypes = [_u16p, _f64p, _i64]
            L.oracle_e4m3_value.restype = ctypes.c_double
            L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_round.restype = ctypes.c_uint8
            L.oracle_e4m3_round.argtypes = [ctypes.c_double]
            L.oracle_quantize_units.restype = None
            L.oracle_quantize_units.argtypes = [_u16p, _i64, _i64, _i64, _i64, _u8p, _i32p, _u16p]
            L.oracle_set_threads.argtypes = [ctypes.c_int]
            L.oracle_get_threads.restype = ctypes.c_int
            L.oracle_gate.restype = ctypes.c_int
            L.oracle_gate.argtypes = [_u16p, _u16p, _u16p, _i64, _i64, _i64, _vp, _i64, _f64p]
            L.oracle_pack.restype = ctypes.c_int
            L.oracle_pack.argtypes = [_f64p, _i64, _i64, _i32, _i32, _i64, _i64, _u16p, _u16p, _u8p, _u8p,
                                      _i32p, ctypes.POINTER(ctypes.c_int64), _u16p]
            L.oracle_unpack.argtypes = [_u16p, _u16p, _u8p, _u8p, _i32p, _i64, _u16p, _i64, _i64, _i32,
                                        _i32, _u16p]
            L.oracle_ffn_fwd.restype = ctypes.c_int
            L.oracle_ffn_fwd.argtypes = [_u16p, _u16p, _u16p, _u16p, _u16p, _i64, _i64, _i64, _vp, _i64,
                                         _vp, _i32, _vp, _f64p]
            L.oracle_ffn_fwd_hybrid.restype = ctypes.c_int
            L.oracle_ffn_fwd_hybrid.argtypes = [_u16p, _u16p, _u16p, _u16p, _u16p, _u8p, _u8p, _i32p, _i64,
                                                _u16p, _i64, _i64, _i64, _i32, _i32, _f64p]
            L.oracle_ffn_bwd.restype = ctypes.c_int
            L.oracle_ffn_bwd.argtypes = [_u16p, _u16p, _u16p, _u16p, _u16p, _u16p, ctypes.c_double, _i64,
                                         _i64, _i64, _vp, _i32, _vp, _f64p, _f64p, _f64p, _f64p, _vp]
            _lib = L
    return _lib


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def bf16_round(x) -> np.ndarray:
    """float64 values -> bfloat16 bits (RNE)."""
    a = _c(x, np.float64)
    out = np.empty(a.shape, np.uint16)
    lib().oracle_bf16_round_array(a.reshape(-1), out.reshape(-1), a.size)
    return out


def bf16_to_f64(b) -> np.ndarray:
    a = _c(b, np.uint16)
    out = np.empty(a.shape, np.float64)
    lib().oracle_bf16_to_double_array(a.reshape(-1), out.reshape(-1), a.size)
    return out


def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 code (NaN for 0x7F / 0xFF)."""
    return float(lib().oracle_e4m3_value(int(code) & 0xFF))


def e4m3_round(x: float) -> int:
    """Nearest E4M3 code of x, ties to even; |x| >= 448 saturates."""
    return int(lib().oracle_e4m3_round(float(x)))


def quantize_e4m3(W, unit_axis: int) -> dict:
    """8-bit copy of a bf16 weight matrix, one power-of-two scale per hidden unit.

    unit_axis = 0: units are rows (W_u [d_ff, d_model]); 1: units are columns
    (W_d [d_model, d_ff]). Returns q [units, len] uint8 codes (unit-major), exp
    [units] int32 (scale 2^exp) and deq: bf16 bits of the dequantised weights in
    W's own layout."""
    W = _c(W, np.uint16)
    R, C = W.shape
    units, length = (R, C) if unit_axis == 0 else (C, R)
    su, sk = (C, 1) if unit_axis == 0 else (1, C)
    q = np.empty((units, length), np.uint8)
    e = np.empty(units, np.int32)
    deq = np.empty_like(W)
    lib().oracle_quantize_units(W, units, length, su, sk, q, e, deq)
    return {"q": q, "exp": e, "deq": deq}


def gate(X, W_g, b_g, rows=None) -> np.ndarray:
    """z = X W_g^T + b_g in float64, for all rows or for the listed rows."""
    X, W_g, b_g = _c(X, np.uint16), _c(W_g, np.uint16), _c(b_g, np.uint16)
    M, d = X.shape
    f = W_g.shape[0]
    r = None if rows is None else _c(rows, np.int32)
    n = M if r is None else r.size
    Z = np.empty((n, f), np.float64)
    if lib().oracle_gate(X, W_g, b_g, M, d, f, _ptr(r), n, Z):
        raise MemoryError("oracle_gate")
    return Z


def pack(Z, T_n: int, K: int, cap=None, dense_min: int = 0) -> dict:
    """TwELL + hybrid routing of a dense float64 Z [M, f]; with dense_min > 0 a
    row with at least that many active units is also routed to the dense backup."""
    Z = _c(Z, np.float64)
    M, f = Z.shape
    if f % T_n or not (1 <= T_n <= 256) or K < 1:
        raise ValueError("need d_ff % T_n == 0, 1 <= T_n <= 256 and K >= 1")
    T = f // T_n
    cap = M if cap is None else int(cap)
    out = dict(
        count=np.empty((M, T), np.uint16), val=np.empty((M, T, K), np.uint16),
        col=np.empty((M, T, K), np.uint8), row_ovf=np.empty(M, np.uint8),
        ovf_rows=np.zeros(max(cap, 1), np.int32), g_ovf=np.zeros((max(cap, 1), f), np.uint16),
    )
    n = ctypes.c_int64(0)
    rc = lib().oracle_pack(Z, M, f, T_n, K, cap, int(dense_min), out["count"], out["val"], out["col"], out["row_ovf"],
                           out["ovf_rows"], ctypes.byref(n), out["g_ovf"])
    if rc == 1:
        raise ValueError("oracle_pack rejected the shape")
    out["n_ovf_total"] = int(n.value)
    out["n_ovf"] = min(int(n.value), cap)
    out["status"] = int(rc)
    out["ovf_rows"] = out["ovf_rows"][:cap]
    out["g_ovf"] = out["g_ovf"][:cap]
    return out


def count_stats(count, T_n: int, dense_min: int = 0) -> dict:
    """Count statistics of a packed batch from its true per-tile counts [M, T]
    (the definitions of twell_count_stats), T_n + 2 bins each: rows binned by
    their largest tile count c (bin c), and those rows' active units summed in
    the same bins, except that with dense_min > 0 a row with at least dense_min
    active units goes to bin T_n + 1; (row, tile) pairs binned by count (bin
    T_n + 1 stays empty)."""
    c = np.asarray(count).astype(np.int64)
    if c.ndim != 2 or (c.size and (c.min() < 0 or c.max() > T_n)):
        raise ValueError("count must be [M, T] with entries in [0, T_n]")
    M = c.shape[0]
    act = c.sum(axis=1)
    b = c.max(axis=1) if c.shape[1] else np.zeros(M, np.int64)
    if dense_min > 0:
        b = np.where(act >= dense_min, T_n + 1, b)
    act_by_max = np.zeros(T_n + 2, np.int64)
    np.add.at(act_by_max, b, act)
    return {"rows_by_max": np.bincount(b, minlength=T_n + 2).astype(np.int64),
            "act_by_max": act_by_max,
            "tiles_by_count": np.bincount(c.ravel(), minlength=T_n + 2).astype(np.int64)}


def unpack(p: dict, f: int, T_n: int, K: int) -> np.ndarray:
    """Dense bf16 bits of ReLU(z) [M, f] rebuilt from a packed dict."""
    M = p["count"].shape[0]
    G = np.empty((M, f), np.uint16)
    ovf_rows = _c(p["ovf_rows"][: p["n_ovf"]], np.int32)
    g_ovf = _c(p["g_ovf"][: p["n_ovf"]], np.uint16)
    if ovf_rows.size == 0:
        ovf_rows = np.zeros(1, np.int32)
        g_ovf = np.zeros((1, f), np.uint16)
    lib().oracle_unpack(_c(p["count"], np.uint16), _c(p["val"], np.uint16), _c(p["col"], np.uint8),
                        _c(p["row_ovf"], np.uint8), ovf_rows, p["n_ovf"], g_ovf, M, f, T_n, K, G)
    return G


def ffn_fwd(X, W_g, b_g, W_u, W_d, rows=None, mask=None, round_g: bool = False, gmat=None) -> np.ndarray:
    """Y = (ReLU(X W_g^T + b_g) * (X W_u^T)) W_d^T in float64 (rows subset optional).

    mask [nrows, f] replaces the z > 0 test; gmat [nrows, f] (bf16 bits) gives g
    itself (active where nonzero); round_g uses bf16(z) for g."""
    X, W_g, b_g, W_u, W_d = (_c(a, np.uint16) for a in (X, W_g, b_g, W_u, W_d))
    M, d = X.shape
    f = W_g.shape[0]
    r = None if rows is None else _c(rows, np.int32)
    n = M if r is None else r.size
    m = None if mask is None else _c(mask, np.uint8)
    if m is not None and m.shape != (n, f):
        raise ValueError("mask must be [nrows, d_ff]")
    gm = None if gmat is None else _c(gmat, np.uint16)
    if gm is not None and gm.shape != (n, f):
        raise ValueError("gmat must be [nrows, d_ff]")
    Y = np.empty((n, d), np.float64)
    if lib().oracle_ffn_fwd(X, W_g, b_g, W_u, W_d, M, d, f, _ptr(r), n, _ptr(m), int(round_g), _ptr(gm), Y):
        raise MemoryError("oracle_ffn_fwd")
    return Y


def ffn_fwd_hybrid(X, W_u, W_d, p: dict, T_n: int, K: int) -> np.ndarray:
    """Y computed from a packed hybrid representation (ELL rows + dense rows)."""
    X, W_u, W_d = (_c(a, np.uint16) for a in (X, W_u, W_d))
    M, d = X.shape
    f = W_u.shape[0]
    n_ovf = p["n_ovf"]
    ovf_rows = _c(p["ovf_rows"][:n_ovf], np.int32)
    g_ovf = _c(p["g_ovf"][:n_ovf], np.uint16)
    if n_ovf == 0:
        ovf_rows = np.zeros(1, np.int32)
        g_ovf = np.zeros((1, f), np.uint16)
    Y = np.empty((M, d), np.float64)
    rc = lib().oracle_ffn_fwd_hybrid(X, W_u, W_d, _c(p["count"], np.uint16), _c(p["val"], np.uint16),
                                     _c(p["col"], np.uint8), _c(p["row_ovf"], np.uint8), ovf_rows, n_ovf,
                                     g_ovf, M, d, f, T_n, K, Y)
    if rc:
        raise MemoryError("oracle_ffn_fwd_hybrid")
    return Y


def ffn_bwd(X, W_g, b_g, W_u, W_d, dY, lam: float = 0.0, mask=None, round_g: bool = False, gmat=None) -> dict:
    """Gradients of sum(Y * dY) + lam * sum(ReLU(z)): dX, dW_g, dW_u, dW_d, db_g (float64).

    mask / gmat / round_g as in ffn_fwd ([M, f])."""
    X, W_g, b_g, W_u, W_d, dY = (_c(a, np.uint16) for a in (X, W_g, b_g, W_u, W_d, dY))
    M, d = X.shape
    f = W_g.shape[0]
    m = None if mask is None else _c(mask, np.uint8)
    if m is not None and m.shape != (M, f):
        raise ValueError("mask must be [M, d_ff]")
    gm = None if gmat is None else _c(gmat, np.uint16)
    if gm is not None and gm.shape != (M, f):
        raise ValueError("gmat must be [M, d_ff]")
    out = dict(dX=np.empty((M, d)), dW_g=np.empty((f, d)), dW_u=np.empty((f, d)), dW_d=np.empty((d, f)),
               db_g=np.empty(f))
    rc = lib().oracle_ffn_bwd(X, W_g, b_g, W_u, W_d, dY, float(lam), M, d, f, _ptr(m), int(round_g), _ptr(gm),
                              out["dX"], out["dW_g"], out["dW_u"], out["dW_d"], _ptr(out["db_g"]))
    if rc:
        raise MemoryError("oracle_ffn_bwd")
    return out


def ffn_bwd_units(X, W_u, W_d, dY, lam: float, units, gcols) -> dict:
    """The weight gradients of the listed hidden units only, for L = sum(Y * dY)
    + lam * sum(g) ("Sakana AI и NVIDIA представили TwELL", paragraph 2: the
    backward over the hybrid format; the formulas of ffn_bwd restricted to unit j):
        dW_u[j] = sum_i dU_ij x_i,  dW_g[j] = sum_i dZ_ij x_i,
        dW_d[:, j] = sum_i h_ij dY_i,  db_g[j] = sum_i dZ_ij,
    over the rows i where unit j is active, with g_ij given as the stored bf16
    value (gcols [M, len(units)] bit patterns; active iff nonzero, as ffn_bwd's
    gmat), u_ij = x_i . W_u[j], dH_ij = dY_i . W_d[:, j], dU = dH g,
    dZ = dH u + lam, h = g u. float64; numpy's matrix products as the sums.
    Returns dW_g, dW_u [n, d], dW_d [d, n] and db_g [n] for the n listed units."""
    X, W_u, W_d, dY = (_c(a, np.uint16) for a in (X, W_u, W_d, dY))
    units = np.asarray(units, np.int64)
    gcols = np.asarray(gcols, np.uint16)
    M, d = X.shape
    n = units.size
    if gcols.shape != (M, n):
        raise ValueError("gcols must be [M, len(units)]")
    out = dict(dW_g=np.zeros((n, d)), dW_u=np.zeros((n, d)), dW_d=np.zeros((d, n)), db_g=np.zeros(n))
    for k, j in enumerate(units):
        rows = np.nonzero(gcols[:, k])[0]
        if rows.size == 0:
            continue
        g = bf16_to_f64(gcols[rows, k])
        x = bf16_to_f64(X[rows])
        dy = bf16_to_f64(dY[rows])
        u = x @ bf16_to_f64(W_u[j])
        dh = dy @ bf16_to_f64(W_d[:, j])
        du = dh * g
        dz = dh * u + lam
        out["dW_u"][k] = du @ x
        out["dW_g"][k] = dz @ x
        out["dW_d"][:, k] = (g * u) @ dy
        out["db_g"][k] = dz.sum()
    return out
