"""TEST INFRASTRUCTURE -- the CPU oracle of the WHA layer, not part of the product.

A ctypes wrapper around ``qwha_oracle.cpp`` (plain C++17, double precision,
std::thread over independent output rows). Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. It shares nothing with the CUDA library in
``walsh_hadamard_sparse_b200``; the two only meet on the seeded inputs from
``workloads``.

Each wrapper takes numpy arrays, converts them to the C types (float64 values,
int32 indices), and returns numpy arrays. Parity status of every function is
listed in the header of ``qwha_oracle.cpp``; all of them are pinned by
``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qwha_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source when missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            sig = {
                "oracle_set_threads": [ctypes.c_int],
                "oracle_hadamard": [i32, P],
                "oracle_transform_dense": [P, i64, i32, i32, P],
                "oracle_fwht": [P, i64, i32, i32, i32, P],
                "oracle_dequant": [i32, i32, i32, i32, P, P, P, P],
                "oracle_delta_w": [i32, i32, i32, P, P, P, P],
                "oracle_adapter_fwd": [i32, i32, i32, P, P, P, P, P, i64, f64, P, P],
                "oracle_adapter_fwd_sparse": [i32, i32, i32, P, P, P, P, i64, f64, P],
                "oracle_adapter_bwd_dx": [i32, i32, i32, P, P, P, P, P, i64, f64, P],
                "oracle_adapter_bwd_dc": [i32, i32, i32, P, P, i64, f64, i64, P, P, P],
                "oracle_init_alloc": [P, i32, i32, i32, i64, i32, i32, P, P, P, P, P],
                "oracle_init_norms": [P, i32, i32, P],
                "oracle_init_budgets": [P, i32, i32, i64, i32, i32, P, P],
                "oracle_init_select": [P, i32, i32, i32, P, P, P, P],
                "oracle_init_select_global": [P, i32, i32, i32, i64, i32, ctypes.c_uint64, P, P, P, P],
                "oracle_refine_values": [P, i32, i32, i32, P, f64, P, P, i32, P, P],
                "oracle_plan_build": [i32, i32, i64, P, P, P, P, P],
                "oracle_pattern_stats": [i32, i32, i64, P, P, P, P],
                "oracle_energy_stats": [P, i32, i32, i32, i64, P],
            }
            for name, args in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def set_threads(n: int) -> int:
    """Threads used by the oracle (0 = all hardware threads); returns the count in use."""
    return _load().oracle_set_threads(int(n))


def hadamard(n: int) -> np.ndarray:
    """Dense orthonormal Sylvester H_n."""
    H = np.empty((n, n), dtype=np.float64)
    _check(_load().oracle_hadamard(n, _p(H)), "hadamard")
    return H


def transform_dense(X, n: int) -> np.ndarray:
    """X @ blockdiag(H_n, ...) by the definition of the product."""
    X = _f64(X)
    Z = np.empty_like(X)
    _check(_load().oracle_transform_dense(_p(X), X.shape[0], X.shape[1], n, _p(Z)), "transform_dense")
    return Z


def fwht(X, n: int, normalize: bool = True) -> np.ndarray:
    """Row-wise fast Walsh-Hadamard transform per block of n (textbook stage order)."""
    X = _f64(X)
    Z = np.empty_like(X)
    _check(_load().oracle_fwht(_p(X), X.shape[0], X.shape[1], n, int(normalize), _p(Z)), "fwht")
    return Z


def dequant(qweight, scales, zeros, bits: int, group: int, d_out: int, d_in: int) -> np.ndarray:
    """W_Q from the packed codes, group scales and zero points (float32 products, as float64)."""
    qw = np.ascontiguousarray(qweight, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.float32)
    z = np.ascontiguousarray(zeros, dtype=np.uint8)
    W = np.empty((d_out, d_in), dtype=np.float64)
    _check(_load().oracle_dequant(bits, group, d_out, d_in, _p(qw), _p(s), _p(z), _p(W)), "dequant")
    return W


def delta_w(row_ptr, col_idx, coef, d_out: int, d_in: int, n: int) -> np.ndarray:
    """Dense dW = F H."""
    rp, ci, c = _i32(row_ptr), _i32(col_idx), _f64(coef)
    dW = np.empty((d_out, d_in), dtype=np.float64)
    _check(_load().oracle_delta_w(d_out, d_in, n, _p(rp), _p(ci), _p(c), _p(dW)), "delta_w")
    return dW


def adapter_fwd(row_ptr, col_idx, coef, X, d_out: int, n: int, alpha: float = 1.0, Wq=None, want_z=True):
    """(Z, Y): Z = X H, Y = X W_Q^T + alpha X (F H)^T. Z is None when want_z is False."""
    rp, ci, c, X = _i32(row_ptr), _i32(col_idx), _f64(coef), _f64(X)
    T, d_in = X.shape
    W = None if Wq is None else _f64(Wq)
    Z = np.empty_like(X) if want_z else None
    Y = np.empty((T, d_out), dtype=np.float64)
    rc = _load().oracle_adapter_fwd(d_out, d_in, n, _p(rp), _p(ci), _p(c), _p(W), _p(X), T, float(alpha), _p(Z), _p(Y))
    _check(rc, "adapter_fwd")
    return Z, Y


def adapter_fwd_sparse(row_ptr, col_idx, coef, X, d_out: int, n: int, alpha: float = 1.0):
    """Adapter output alpha (X H) F^T by the sparse route."""
    rp, ci, c, X = _i32(row_ptr), _i32(col_idx), _f64(coef), _f64(X)
    T, d_in = X.shape
    Y = np.empty((T, d_out), dtype=np.float64)
    rc = _load().oracle_adapter_fwd_sparse(d_out, d_in, n, _p(rp), _p(ci), _p(c), _p(X), T, float(alpha), _p(Y))
    _check(rc, "adapter_fwd_sparse")
    return Y


def adapter_bwd_dx(row_ptr, col_idx, coef, dY, d_in: int, n: int, alpha: float = 1.0, Wq=None):
    """dX = dY W_Q + alpha dY (F H)."""
    rp, ci, c, dY = _i32(row_ptr), _i32(col_idx), _f64(coef), _f64(dY)
    T, d_out = dY.shape
    W = None if Wq is None else _f64(Wq)
    dX = np.empty((T, d_in), dtype=np.float64)
    rc = _load().oracle_adapter_bwd_dx(d_out, d_in, n, _p(rp), _p(ci), _p(c), _p(W), _p(dY), T, float(alpha), _p(dX))
    _check(rc, "adapter_bwd_dx")
    return dX


def adapter_bwd_dc(X, dY, rows, cols, n: int, alpha: float = 1.0):
    """dc at positions (rows[j], cols[j]): alpha * sum_t dY[t, r] (X H)[t, k]."""
    X, dY = _f64(X), _f64(dY)
    r, k = _i32(rows), _i32(cols)
    T, d_in = X.shape
    d_out = dY.shape[1]
    assert dY.shape[0] == T and r.size == k.size
    dc = np.empty(r.size, dtype=np.float64)
    rc = _load().oracle_adapter_bwd_dc(d_out, d_in, n, _p(X), _p(dY), T, float(alpha), r.size, _p(r), _p(k), _p(dc))
    _check(rc, "adapter_bwd_dc")
    return dc


def csr_rows(row_ptr) -> np.ndarray:
    """Row index of every CSR position."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    return np.repeat(np.arange(rp.size - 1, dtype=np.int32), np.diff(rp))


def init_alloc(dWq, p: int, n: int, min_per_row: int = 2, mode: str = "fewest"):
    """AdaAlloc: dict(budgets, row_ptr, col_idx, coef, err_norm)."""
    w = np.ascontiguousarray(dWq, dtype=np.float32)
    d_out, d_in = w.shape
    b = np.empty(d_out, dtype=np.int32)
    rp = np.empty(d_out + 1, dtype=np.int32)
    ci = np.empty(p, dtype=np.int32)
    c = np.empty(p, dtype=np.float32)
    e = np.empty(d_out, dtype=np.float64)
    m = {"fewest": 0, "largest": 1}[mode]
    rc = _load().oracle_init_alloc(_p(w), d_out, d_in, n, int(p), int(min_per_row), m, _p(b), _p(rp), _p(ci), _p(c), _p(e))
    _check(rc, "init_alloc")
    return dict(budgets=b, row_ptr=rp, col_idx=ci, coef=c, err_norm=e)


def init_norms(dWq_rows):
    """AdaAlloc step 1 for a block of rows: e_i = ||dW_Q[i,:]||_2 (fp64)."""
    w = np.ascontiguousarray(dWq_rows, dtype=np.float32)
    rows, d_in = w.shape
    e = np.empty(rows, dtype=np.float64)
    _check(_load().oracle_init_norms(_p(w), rows, d_in, _p(e)), "init_norms")
    return e


def init_budgets(e, d_in: int, p: int, min_per_row: int = 2, mode: str = "fewest"):
    """AdaAlloc step 2 from all d_out norms: (budgets [d_out], row_ptr [d_out+1])."""
    e = _f64(e)
    d_out = e.size
    b = np.empty(d_out, dtype=np.int32)
    rp = np.empty(d_out + 1, dtype=np.int32)
    m = {"fewest": 0, "largest": 1}[mode]
    _check(_load().oracle_init_budgets(_p(e), d_out, d_in, int(p), int(min_per_row), m, _p(b), _p(rp)), "init_budgets")
    return b, rp


def init_select(dWq_rows, n: int, budgets, row_ptr):
    """AdaAlloc step 3 for a block of rows given its slices of budgets and row_ptr: (col_idx, coef)."""
    w = np.ascontiguousarray(dWq_rows, dtype=np.float32)
    rows, d_in = w.shape
    b, rp = _i32(budgets), _i32(row_ptr)
    cnt = int(rp[-1] - rp[0]) if rows else 0
    ci = np.empty(cnt, dtype=np.int32)
    c = np.empty(cnt, dtype=np.float32)
    _check(_load().oracle_init_select(_p(w), rows, d_in, n, _p(b), _p(rp), _p(ci), _p(c)), "init_select")
    return ci, c


def init_select_global(dWq, p: int, n: int, sel: str = "magnitude", seed: int = 0):
    """E over the whole matrix (the pages' alternatives to AdaAlloc): "magnitude" = the p largest |V| (ties to the
    lower flat index), "random" = the p smallest SplitMix64 keys; dict(budgets, row_ptr, col_idx, coef)."""
    w = np.ascontiguousarray(dWq, dtype=np.float32)
    d_out, d_in = w.shape
    b = np.empty(d_out, dtype=np.int32)
    rp = np.empty(d_out + 1, dtype=np.int32)
    ci = np.empty(p, dtype=np.int32)
    c = np.empty(p, dtype=np.float32)
    s = {"magnitude": 0, "random": 1}[sel]
    rc = _load().oracle_init_select_global(_p(w), d_out, d_in, n, int(p), s, ctypes.c_uint64(seed & (2**64 - 1)),
                                           _p(b), _p(rp), _p(ci), _p(c))
    _check(rc, "init_select_global")
    return dict(budgets=b, row_ptr=rp, col_idx=ci, coef=c)


def refine_values(dWq, S, row_ptr, col_idx, n: int, damp: float = 0.0, rows=None):
    """Value Refinement: least-squares values at E for the calibration Hessian S = X^T X [d_in, d_in] (fp64),
    S damped by damp * mean(diag S). Returns coef [p] (float32); only the entries of `rows` (all when None) are
    computed, the others are NaN."""
    w = np.ascontiguousarray(dWq, dtype=np.float32)
    d_out, d_in = w.shape
    S = _f64(S)
    assert S.shape == (d_in, d_in)
    rp, ci = _i32(row_ptr), _i32(col_idx)
    c = np.full(ci.size, np.nan, dtype=np.float32)
    sel = None if rows is None else _i32(rows)
    rc = _load().oracle_refine_values(_p(w), d_out, d_in, n, _p(S), float(damp), _p(rp), _p(ci),
                                      0 if sel is None else sel.size, _p(sel), _p(c))
    if rc == 2:
        raise ValueError("refine_values: a system is not positive definite")
    _check(rc, "refine_values")
    return c


def plan_build(row_ptr, col_idx, d_in: int):
    """CSC view: (col_ptr [d_in+1], row_idx [p], perm [p])."""
    rp, ci = _i32(row_ptr), _i32(col_idx)
    d_out = rp.size - 1
    p = ci.size
    cp = np.empty(d_in + 1, dtype=np.int32)
    ri = np.empty(p, dtype=np.int32)
    pm = np.empty(p, dtype=np.int32)
    _check(_load().oracle_plan_build(d_out, d_in, p, _p(rp), _p(ci), _p(cp), _p(ri), _p(pm)), "plan_build")
    return cp, ri, pm


PATTERN_STATS = ("empty_rows", "empty_cols", "min_row", "max_row", "min_col", "max_col", "rank_bound", "half_rows")


def pattern_stats(row_ptr, col_idx, d_in: int) -> dict:
    """Counts of E by row and column (the rank argument of the pages): dict of PATTERN_STATS plus col_counts."""
    rp, ci = _i32(row_ptr), _i32(col_idx)
    d_out = rp.size - 1
    cc = np.empty(d_in, dtype=np.int32)
    st = np.empty(8, dtype=np.int64)
    _check(_load().oracle_pattern_stats(d_out, d_in, ci.size, _p(rp), _p(ci), _p(cc), _p(st)), "pattern_stats")
    out = {k: int(v) for k, v in zip(PATTERN_STATS, st)}
    out["col_counts"] = cc
    return out


def numerical_rank(row_ptr, col_idx, coef, d_in: int) -> int:
    """rank(F) of F = Scatter(c, E) [d_out, d_in] in fp64 (numpy's SVD-based matrix_rank with its default
    tolerance); for the small shapes of the tests."""
    rp, ci = _i32(row_ptr), _i32(col_idx)
    d_out = rp.size - 1
    F = np.zeros((d_out, d_in), dtype=np.float64)
    F[np.repeat(np.arange(d_out), np.diff(rp)), ci] = _f64(coef)
    return int(np.linalg.matrix_rank(F))


def energy_stats(dWq, k: int, n: int) -> dict:
    """Hill exponent eta and cumulative energy of the k largest transform coefficients |dW_Q H| (see
    oracle_energy_stats): dict(eta, energy, threshold, total)."""
    w = np.ascontiguousarray(dWq, dtype=np.float32)
    d_out, d_in = w.shape
    out = np.empty(4, dtype=np.float64)
    _check(_load().oracle_energy_stats(_p(w), d_out, d_in, n, int(k), _p(out)), "energy_stats")
    return dict(eta=float(out[0]), energy=float(out[1]), threshold=float(out[2]), total=float(out[3]))
