"""Float64 CPU oracle for online log-domain Sinkhorn -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library in
``log_domain_sinkhorn_online_b200``) never does, and this package imports
nothing from it.

The arithmetic lives in ``sinkhorn_oracle.c`` (plain C, float64, OpenMP over
rows); this module compiles it with gcc on first use and wraps each entry
point with ctypes + numpy. Every function states what it computes and the
page it follows; see the C file's header for the readings taken where the
pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sinkhorn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

SCALE_NONE, SCALE_MEAN, SCALE_MAX_COST, SCALE_VALUE = 0, 1, 2, 3
_SCALE_NAMES = {"none": SCALE_NONE, "mean": SCALE_MEAN, "max_cost": SCALE_MAX_COST}


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, no fast-math, OpenMP) into oracle/_build."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32, D = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.orc_num_threads.restype = I32
            lib.orc_inv_scale_cost.argtypes = [P, P, I64, I64, I32, I32, D]
            lib.orc_inv_scale_cost.restype = D
            lib.orc_f_step.argtypes = [P, P, P, P, I64, I64, I32, D, D, P, I64, P]
            lib.orc_g_step.argtypes = [P, P, P, P, I64, I64, I32, D, D, P, I64, P]
            lib.orc_marginal_residual.argtypes = [P, P, P, P, P, P, I64, I64, I32, D, D,
                                                  P, P, P, P]
            lib.orc_sinkhorn.argtypes = [P, P, P, P, I64, I64, I32, D, D, I32, D, P, P, P]
            lib.orc_sinkhorn.restype = I32
            lib.orc_sinkhorn_anneal.argtypes = [P, P, P, P, I64, I64, I32, D, D, D, D, I32,
                                                P, P, P]
            lib.orc_sinkhorn_anneal.restype = I32
            lib.orc_materialize_rows.argtypes = [P, P, P, P, I64, I64, I32, D, D, P, I64, P]
            lib.orc_dense_plan.argtypes = [P, P, P, P, I64, I64, I32, D, D, P]
            lib.orc_min_row.argtypes = [P, P, P, P, P, I64, I64, I32, D, D, I64, P, P, P, P]
            lib.orc_min_row.restype = I64
            lib.orc_sparsify_csr.argtypes = [P, P, P, P, P, I64, I64, I32, D, D, D, P, P, P, I64]
            lib.orc_lr_rows.argtypes = [P, P, P, I64, I64, I32, P, I64, P]
            lib.orc_lrc_rows.argtypes = [P, P, P, P, I64, I64, I32, D, D, D, P, I64, P]
            lib.orc_sparsify_csr.restype = I64
            lib.orc_morton_codes.argtypes = [P, I64, I32, P, P, P]
            lib.orc_morton_order.argtypes = [P, I64, I32, P, P, P]
            lib.orc_block_mask.argtypes = [P, P, P, P, P, P, I64, I64, I32, D, D, I64, D, I32,
                                           P, P, P, P, P]
            lib.orc_block_mask.restype = I64
            lib.orc_sparse_f_step.argtypes = [P, P, P, P, I64, I64, I32, D, D, I64, P, P]
            lib.orc_sparse_g_step.argtypes = [P, P, P, P, I64, I64, I32, D, D, I64, P, P]
            lib.orc_sparse_row_residual.argtypes = [P, P, P, P, P, I64, I64, I32, D, D, I64, P]
            lib.orc_sparse_row_residual.restype = D
            lib.orc_sinkhorn_sparse.argtypes = [P, P, P, P, I64, I64, I32, D, D, I32, D, I64, D,
                                                I32, D, P, P, P, P]
            lib.orc_sinkhorn_sparse.restype = I32
            _lib = lib
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _pts(x, y):
    x, y = _f32(x), _f32(y)
    if x.ndim == 1:
        x = x[:, None]
    if y.ndim == 1:
        y = y[:, None]
    assert x.shape[1] == y.shape[1]
    return x, y, x.shape[0], y.shape[0], x.shape[1]


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().orc_num_threads())


def inv_scale_cost(x, y, scale="none", value=None) -> float:
    """c such that the cost used is C_ij = c * ||x_i - y_j||^2.

    "none" -> 1; "mean" -> 1 / mean over all n*m pairs (brute force);
    "max_cost" -> 1 / max over all pairs; a number v -> 1 / v. The parent
    problem's c is resolved once and reused for every row subset (moscot
    PR #846, section "Fix").
    """
    x, y, n, m, d = _pts(x, y)
    if isinstance(scale, str):
        mode, val = _SCALE_NAMES[scale], 0.0
    else:
        mode, val = SCALE_VALUE, float(scale if value is None else value)
    return float(_load().orc_inv_scale_cost(_ptr(x), _ptr(y), n, m, d, mode, val))


def f_step(x, y, a, g, c, eps, rows=None):
    """f_i = eps ln a_i - eps LSE_j((g_j - C_ij)/eps) (FlashSinkhorn 2, section 2.1).

    rows: optional int64 indices; then only those rows are returned.
    """
    x, y, n, m, d = _pts(x, y)
    a, g = _f64(a), _f64(g)
    if rows is None:
        out = np.empty(n)
        _load().orc_f_step(_ptr(x), _ptr(y), _ptr(a), _ptr(g), n, m, d, c, eps, None, 0,
                           _ptr(out))
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty(rows.shape[0])
        _load().orc_f_step(_ptr(x), _ptr(y), _ptr(a), _ptr(g), n, m, d, c, eps, _ptr(rows),
                           rows.shape[0], _ptr(out))
    return out


def g_step(x, y, b, f, c, eps, cols=None):
    """g_j = eps ln b_j - eps LSE_i((f_i - C_ij)/eps) (FlashSinkhorn 2, section 2.1)."""
    x, y, n, m, d = _pts(x, y)
    b, f = _f64(b), _f64(f)
    if cols is None:
        out = np.empty(m)
        _load().orc_g_step(_ptr(x), _ptr(y), _ptr(b), _ptr(f), n, m, d, c, eps, None, 0,
                           _ptr(out))
    else:
        cols = np.ascontiguousarray(cols, dtype=np.int64)
        out = np.empty(cols.shape[0])
        _load().orc_g_step(_ptr(x), _ptr(y), _ptr(b), _ptr(f), n, m, d, c, eps, _ptr(cols),
                           cols.shape[0], _ptr(out))
    return out


def sinkhorn(x, y, a, b, c, eps, n_iters, tol=0.0, f0=None, g0=None):
    """Alternating f/g updates from f=g=0 (or f0/g0).

    Returns (f, g, iterations, row_residual_of_returned_state). With tol > 0
    it stops after the first iteration whose ||T1 - a||_1 <= tol.
    """
    x, y, n, m, d = _pts(x, y)
    a, b = _f64(a), _f64(b)
    f = np.zeros(n) if f0 is None else _f64(f0).copy()
    g = np.zeros(m) if g0 is None else _f64(g0).copy()
    r = ctypes.c_double(0.0)
    it = _load().orc_sinkhorn(_ptr(x), _ptr(y), _ptr(a), _ptr(b), n, m, d, c, eps,
                              int(n_iters), float(tol), _ptr(f), _ptr(g), ctypes.byref(r))
    return f, g, int(it), float(r.value)


def sinkhorn_anneal(x, y, a, b, c, eps_target, eps_init=1.0, decay=0.7, iters_per_stage=20,
                    f0=None, g0=None):
    """eps-annealing: stage k at max(eps_target, eps_init*decay**k), carried potentials.

    Returns (f, g, stages, row_residual).
    """
    x, y, n, m, d = _pts(x, y)
    a, b = _f64(a), _f64(b)
    f = np.zeros(n) if f0 is None else _f64(f0).copy()
    g = np.zeros(m) if g0 is None else _f64(g0).copy()
    r = ctypes.c_double(0.0)
    k = _load().orc_sinkhorn_anneal(_ptr(x), _ptr(y), _ptr(a), _ptr(b), n, m, d, c,
                                    float(eps_target), float(eps_init), float(decay),
                                    int(iters_per_stage), _ptr(f), _ptr(g), ctypes.byref(r))
    return f, g, int(k), float(r.value)


def marginal_residual(x, y, a, b, f, g, c, eps, return_sums=False):
    """(||T1 - a||_1, ||T^T 1 - b||_1) with T_ij = exp((f_i+g_j-C_ij)/eps)."""
    x, y, n, m, d = _pts(x, y)
    a, b, f, g = _f64(a), _f64(b), _f64(f), _f64(g)
    r, q = ctypes.c_double(), ctypes.c_double()
    rs, cs = (np.empty(n), np.empty(m)) if return_sums else (None, None)
    _load().orc_marginal_residual(_ptr(x), _ptr(y), _ptr(a), _ptr(b), _ptr(f), _ptr(g), n, m,
                                  d, c, eps, ctypes.byref(r), ctypes.byref(q), _ptr(rs),
                                  _ptr(cs))
    if return_sums:
        return float(r.value), float(q.value), rs, cs
    return float(r.value), float(q.value)


def materialize_rows(x, y, f, g, c, eps, row_idx):
    """T[row_idx, :] with T_ij = exp((f_i + g_j - C_ij)/eps) (moscot PR #846, "Fix")."""
    x, y, n, m, d = _pts(x, y)
    f, g = _f64(f), _f64(g)
    row_idx = np.ascontiguousarray(row_idx, dtype=np.int64)
    out = np.empty((row_idx.shape[0], m))
    _load().orc_materialize_rows(_ptr(x), _ptr(y), _ptr(f), _ptr(g), n, m, d, c, eps,
                                 _ptr(row_idx), row_idx.shape[0], _ptr(out))
    return out


def dense_plan(x, y, f, g, c, eps):
    """The full n x m plan (small inputs only)."""
    x, y, n, m, d = _pts(x, y)
    f, g = _f64(f), _f64(g)
    T = np.empty((n, m))
    _load().orc_dense_plan(_ptr(x), _ptr(y), _ptr(f), _ptr(g), n, m, d, c, eps, _ptr(T))
    return T


def sparsify_csr(x, y, a, f, g, c, eps, thr):
    """The thresholded plan (T_ij >= thr, massful rows) in compressed-row form
    (moscot PR #846, "Behavioural changes"). Returns (row_ptr, col_idx, vals)."""
    x, y, n, m, d = _pts(x, y)
    a, f, g = _f64(a), _f64(f), _f64(g)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    L = _load()
    # first call with no room only sizes the result
    nnz = L.orc_sparsify_csr(_ptr(x), _ptr(y), _ptr(a), _ptr(f), _ptr(g), n, m, d, c, eps, float(thr),
                             _ptr(row_ptr), None, None, ctypes.c_int64(-1))
    assert nnz == -1
    total = int(row_ptr[n])
    col_idx = np.empty(max(total, 1), dtype=np.int64)
    vals = np.empty(max(total, 1), dtype=np.float64)
    nnz = L.orc_sparsify_csr(_ptr(x), _ptr(y), _ptr(a), _ptr(f), _ptr(g), n, m, d, c, eps, float(thr),
                             _ptr(row_ptr), _ptr(col_idx), _ptr(vals), ctypes.c_int64(total))
    assert nnz == total
    return row_ptr, col_idx[:total], vals[:total]


def lr_rows(Q, R, g, rows):
    """Rows of the low-rank coupling Q diag(1/g) R^T (moscot PR #846, "Fix")."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    R = np.ascontiguousarray(R, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n, r = Q.shape
    m = R.shape[0]
    out = np.empty((len(rows), m), dtype=np.float64)
    _load().orc_lr_rows(_ptr(Q), _ptr(R), _ptr(g), n, m, r, _ptr(rows), len(rows), _ptr(out))
    return out


def lrc_rows(cost1, cost2, f, g, bias, c, eps, rows):
    """Entropic rows exp((f_i + g_j - c (cost1[i].cost2[j] + bias))/eps) on a
    low-rank cost geometry (moscot PR #846, "Fix")."""
    cost1 = np.ascontiguousarray(cost1, dtype=np.float32)
    cost2 = np.ascontiguousarray(cost2, dtype=np.float32)
    f, g = _f64(f), _f64(g)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n, r = cost1.shape
    m = cost2.shape[0]
    out = np.empty((len(rows), m), dtype=np.float64)
    _load().orc_lrc_rows(_ptr(cost1), _ptr(cost2), _ptr(f), _ptr(g), n, m, r, float(bias), float(c),
                         float(eps), _ptr(rows), len(rows), _ptr(out))
    return out


def min_row(x, y, a, f, g, c, eps, block_rows=0):
    """Exact min_row threshold (moscot PR #846, "Behavioural changes").

    Returns dict(thr, argmin, counts[n], nnz, n_massless).
    """
    x, y, n, m, d = _pts(x, y)
    a, f, g = _f64(a), _f64(f), _f64(g)
    thr, arg, nnz = ctypes.c_double(), ctypes.c_int64(), ctypes.c_int64()
    counts = np.empty(n, dtype=np.int64)
    nm = _load().orc_min_row(_ptr(x), _ptr(y), _ptr(a), _ptr(f), _ptr(g), n, m, d, c, eps,
                             int(block_rows), ctypes.byref(thr), ctypes.byref(arg),
                             _ptr(counts), ctypes.byref(nnz))
    return dict(thr=float(thr.value), argmin=int(arg.value), counts=counts,
                nnz=int(nnz.value), n_massless=int(nm))


# ------------------------------------------------------- block-sparse updates
# "FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", sections 3, 3.2,
# A.3, B.1 and B.3; the readings are spelled out in sinkhorn_oracle.c.

def joint_box(x, y):
    """(lo, hi) per coordinate over both clouds, float64."""
    x, y, n, m, d = _pts(x, y)
    both = np.concatenate([x, y]).astype(np.float64)
    return both.min(0), both.max(0)


def morton_codes(x, lo, hi):
    """Morton codes (bits = 30/d per coordinate over the box [lo, hi])."""
    x = _f32(x)
    if x.ndim == 1:
        x = x[:, None]
    n, d = x.shape
    lo, hi = _f64(lo), _f64(hi)
    out = np.empty(n, dtype=np.uint64)
    _load().orc_morton_codes(_ptr(x), n, d, _ptr(lo), _ptr(hi), _ptr(out))
    return out


def morton_order(x, lo, hi):
    """perm with x[perm] in Morton order, ties by index (section 3)."""
    x = _f32(x)
    if x.ndim == 1:
        x = x[:, None]
    n, d = x.shape
    lo, hi = _f64(lo), _f64(hi)
    perm = np.empty(n, dtype=np.int64)
    _load().orc_morton_order(_ptr(x), n, d, _ptr(lo), _ptr(hi), _ptr(perm))
    return perm


def block_mask(x, y, a, b, f, g, c, eps, B, delta, verify=True):
    """Block-pair mask at (f, g) for points already in block order.

    Returns dict(cand, adm: [NB, MB] bool, screen_margin, mass_margin: [NB, MB]
    natural-log margins over the threshold, n_cand, n_adm).
    """
    x, y, n, m, d = _pts(x, y)
    a, b, f, g = _f64(a), _f64(b), _f64(f), _f64(g)
    NB, MB = -(-n // B), -(-m // B)
    cand = np.empty((NB, MB), dtype=np.uint8)
    adm = np.empty((NB, MB), dtype=np.uint8)
    sm = np.empty((NB, MB))
    mm = np.empty((NB, MB))
    nc = ctypes.c_int64()
    na = _load().orc_block_mask(_ptr(x), _ptr(y), _ptr(a), _ptr(b), _ptr(f), _ptr(g), n, m, d,
                                float(c), float(eps), int(B), float(delta), int(bool(verify)),
                                _ptr(cand), _ptr(adm), _ptr(sm), _ptr(mm), ctypes.byref(nc))
    return dict(cand=cand.astype(bool), adm=adm.astype(bool), screen_margin=sm,
                mass_margin=mm, n_cand=int(nc.value), n_adm=int(na))


def sparse_f_step(x, y, a, g, c, eps, B, adm):
    """f-update over the admitted tiles of each row block (all columns for a
    block without one), points in block order."""
    x, y, n, m, d = _pts(x, y)
    a, g = _f64(a), _f64(g)
    adm = np.ascontiguousarray(adm, dtype=np.uint8)
    out = np.empty(n)
    _load().orc_sparse_f_step(_ptr(x), _ptr(y), _ptr(a), _ptr(g), n, m, d, float(c), float(eps),
                              int(B), _ptr(adm), _ptr(out))
    return out


def sparse_g_step(x, y, b, f, c, eps, B, adm):
    """g-update over the admitted tiles of each column block (the mask read by columns)."""
    x, y, n, m, d = _pts(x, y)
    b, f = _f64(b), _f64(f)
    adm = np.ascontiguousarray(adm, dtype=np.uint8)
    out = np.empty(m)
    _load().orc_sparse_g_step(_ptr(x), _ptr(y), _ptr(b), _ptr(f), n, m, d, float(c), float(eps),
                              int(B), _ptr(adm), _ptr(out))
    return out


def sparse_row_residual(x, y, a, f, g, c, eps, B, adm):
    """sum_i |sum over admitted j of T_ij - a_i| (the stop test of a sparse iteration)."""
    x, y, n, m, d = _pts(x, y)
    a, f, g = _f64(a), _f64(f), _f64(g)
    adm = np.ascontiguousarray(adm, dtype=np.uint8)
    return float(_load().orc_sparse_row_residual(_ptr(x), _ptr(y), _ptr(a), _ptr(f), _ptr(g), n,
                                                 m, d, float(c), float(eps), int(B), _ptr(adm)))


def sinkhorn_sparse(x, y, a, b, c, eps, n_iters, tol=0.0, B=128, delta=0.0, verify=True,
                    dense_frac=0.5, f0=None, g0=None):
    """Block-sparse fine iterations in Morton order, potentials in the caller's order.

    Returns (f, g, iterations, residual, stats) with stats = (sparse
    iterations, dense iterations, candidates, admitted tiles of the last mask).
    """
    x, y, n, m, d = _pts(x, y)
    a, b = _f64(a), _f64(b)
    f = np.zeros(n) if f0 is None else _f64(f0).copy()
    g = np.zeros(m) if g0 is None else _f64(g0).copy()
    r = ctypes.c_double(0.0)
    st = np.zeros(4, dtype=np.int64)
    it = _load().orc_sinkhorn_sparse(_ptr(x), _ptr(y), _ptr(a), _ptr(b), n, m, d, float(c),
                                     float(eps), int(n_iters), float(tol), int(B), float(delta),
                                     int(bool(verify)), float(dense_frac), _ptr(f), _ptr(g),
                                     ctypes.byref(r), _ptr(st))
    if it < 0:
        raise ValueError("bad arguments (block size, sizes, or delta <= 0 with tol <= 0)")
    return f, g, int(it), float(r.value), tuple(int(v) for v in st)
