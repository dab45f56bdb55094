"""ctypes binding of ``include/ot_sinkhorn.h`` -- argument marshalling only.

Each function has the name of the C entry point it calls and takes raw device
pointers (ints), sizes and a stream handle (int, 0 = legacy default stream).
No arithmetic of the method happens here. Loading fails loudly when the
compiled library is missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libot_sinkhorn.so")
_lock = threading.Lock()
_lib = None

OT_OK = 0
OT_WARN_MASSLESS_ROWS = 1
OT_ERR_INVALID_ARG = -1
OT_ERR_OVERFLOW = -2
OT_ERR_CUDA = -3
OT_ERR_OOM = -4
OT_ERR_NONFINITE = -5
OT_ERR_UNSUPPORTED = -6

OT_SCALE_NONE, OT_SCALE_MEAN, OT_SCALE_MAX_COST, OT_SCALE_VALUE = 0, 1, 2, 3

# every symbol the header declares (checked by the CPU test suite)
EXPORTED = ("ot_version", "ot_last_error_string", "ot_options_default", "ot_sinkhorn_pointcloud",
            "ot_sinkhorn_pointcloud_host", "ot_marginal_residual", "ot_materialize_rows",
            "ot_sparsify_min_row", "ot_plan_destroy", "ot_marginal_residual_noalloc", "ot_trim_cache",
            "ot_sparsify_csr", "ot_materialize_rows_lowrank", "ot_materialize_rows_lrcost",
            "ot_testing_fail_device_allocs", "ot_testing_wait_fault", "ot_max_sqdist",
            "ot_shard_plan_create", "ot_shard_half_step", "ot_marginal_residual_range",
            "ot_min_row_range", "ot_kept_counts_range", "ot_row_pass_stats")
OT_NOALLOC_MAX_POINTS = 1 << 20


class OtOptions(ctypes.Structure):
    _fields_ = [("warm_start", ctypes.c_int32), ("check_every", ctypes.c_int32),
                ("use_graphs", ctypes.c_int32), ("iters_per_stage", ctypes.c_int32),
                ("scale_value", ctypes.c_double), ("eps_init", ctypes.c_double),
                ("eps_decay", ctypes.c_double), ("timing", ctypes.c_int32),
                ("col_splits", ctypes.c_int32), ("rows_per_thread", ctypes.c_int32),
                ("tensor_cores", ctypes.c_int32), ("device_loop", ctypes.c_int32),
                ("reserved1", ctypes.c_int32), ("block_sparse", ctypes.c_int32),
                ("sparse_block", ctypes.c_int32), ("sparse_verify", ctypes.c_int32),
                ("reserved2", ctypes.c_int32), ("sparse_delta", ctypes.c_double),
                ("sparse_dense_frac", ctypes.c_double), ("resid_history", ctypes.c_void_p),
                ("resid_history_len", ctypes.c_int64), ("sparse_mask_out", ctypes.c_void_p),
                ("sparse_mask_len", ctypes.c_int64)]


class OtInfo(ctypes.Structure):
    _fields_ = [("iterations", ctypes.c_int32), ("converged", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("col_splits", ctypes.c_int32),
                ("residual", ctypes.c_double), ("inv_scale_cost", ctypes.c_double),
                ("eps", ctypes.c_double), ("n_massless_rows", ctypes.c_int64),
                ("n_massless_cols", ctypes.c_int64), ("half_steps", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int64), ("loop_ms", ctypes.c_double),
                ("sparse_iterations", ctypes.c_int64), ("dense_iterations", ctypes.c_int64),
                ("tiles_candidate", ctypes.c_int64), ("tiles_admitted", ctypes.c_int64), ("tiles_exact", ctypes.c_int64),
                ("tiles_total", ctypes.c_int64), ("omitted_bound", ctypes.c_double),
                ("verify_ms", ctypes.c_double), ("sparse_hs_ms", ctypes.c_double),
                ("sparse_hs_launches", ctypes.c_int64)]


class OTError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"status {status}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m log_domain_sinkhorn_online_b200.build` (there is no CPU fallback)")
            L = ctypes.CDLL(_LIB_PATH)
            P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            L.ot_version.restype = ctypes.c_int
            L.ot_last_error_string.restype = ctypes.c_char_p
            L.ot_options_default.argtypes = [ctypes.POINTER(OtOptions)]
            L.ot_options_default.restype = None
            L.ot_sinkhorn_pointcloud.argtypes = [P, P, P, P, I64, I64, I32, ctypes.c_double, ctypes.c_int,
                                                 I32, ctypes.c_double, P, P, P,
                                                 ctypes.POINTER(OtOptions), ctypes.POINTER(P),
                                                 ctypes.POINTER(OtInfo)]
            L.ot_sinkhorn_pointcloud.restype = ctypes.c_int
            L.ot_sinkhorn_pointcloud_host.argtypes = L.ot_sinkhorn_pointcloud.argtypes
            L.ot_sinkhorn_pointcloud_host.restype = ctypes.c_int
            L.ot_max_sqdist.argtypes = [P, P, I64, I64, I32, I64, I64, ctypes.POINTER(ctypes.c_float), P]
            L.ot_max_sqdist.restype = ctypes.c_int
            L.ot_shard_plan_create.argtypes = [P, P, P, P, I64, I64, I32, D, ctypes.c_int, I64, I64, I64, I64,
                                               P, ctypes.POINTER(OtOptions), ctypes.POINTER(P),
                                               ctypes.POINTER(OtInfo)]
            L.ot_shard_plan_create.restype = ctypes.c_int
            L.ot_shard_half_step.argtypes = [P, I32, P, P, P, ctypes.POINTER(D), P]
            L.ot_shard_half_step.restype = ctypes.c_int
            L.ot_testing_fail_device_allocs.argtypes = [ctypes.c_int]
            L.ot_testing_fail_device_allocs.restype = None
            L.ot_testing_wait_fault.argtypes = [ctypes.c_int]
            L.ot_testing_wait_fault.restype = None
            L.ot_marginal_residual.argtypes = [P, ctypes.POINTER(D), ctypes.POINTER(D), P]
            L.ot_marginal_residual.restype = ctypes.c_int
            L.ot_materialize_rows.argtypes = [P, P, I64, P, P]
            L.ot_materialize_rows.restype = ctypes.c_int
            L.ot_sparsify_min_row.argtypes = [P, I64, ctypes.POINTER(ctypes.c_float), P,
                                              ctypes.POINTER(I64), ctypes.POINTER(I64),
                                              ctypes.POINTER(I64), P]
            L.ot_sparsify_min_row.restype = ctypes.c_int
            L.ot_sparsify_csr.argtypes = [P, I64, ctypes.c_float, P, P, P, I64, ctypes.POINTER(I64), P]
            L.ot_sparsify_csr.restype = ctypes.c_int
            L.ot_materialize_rows_lowrank.argtypes = [P, P, P, I64, I64, I32, P, I64, P, P]
            L.ot_materialize_rows_lowrank.restype = ctypes.c_int
            L.ot_materialize_rows_lrcost.argtypes = [P, P, P, P, I64, I64, I32, D, D, D, P, I64, P, P]
            L.ot_materialize_rows_lrcost.restype = ctypes.c_int
            L.ot_marginal_residual_noalloc.argtypes = [P, P, P, P, P, P, I64, I64, I32, D, D,
                                                       ctypes.POINTER(D), ctypes.POINTER(D), P]
            L.ot_marginal_residual_noalloc.restype = ctypes.c_int
            L.ot_marginal_residual_range.argtypes = [P, I64, I64, I64, I64, ctypes.POINTER(D),
                                                     ctypes.POINTER(D), P]
            L.ot_marginal_residual_range.restype = ctypes.c_int
            L.ot_min_row_range.argtypes = [P, I64, I64, I64, ctypes.POINTER(ctypes.c_float),
                                           ctypes.POINTER(I64), ctypes.POINTER(I64), P]
            L.ot_min_row_range.restype = ctypes.c_int
            L.ot_kept_counts_range.argtypes = [P, I64, I64, I64, ctypes.c_float, P, ctypes.POINTER(I64), P]
            L.ot_kept_counts_range.restype = ctypes.c_int
            L.ot_row_pass_stats.argtypes = [P, ctypes.POINTER(I64), ctypes.POINTER(I64)]
            L.ot_row_pass_stats.restype = ctypes.c_int
            L.ot_trim_cache.argtypes = []
            L.ot_trim_cache.restype = None
            L.ot_plan_destroy.argtypes = [P]
            L.ot_plan_destroy.restype = None
            _lib = L
    return _lib


def _check(status: int) -> int:
    if status < 0:
        raise OTError(status, ot_last_error_string())
    return status


def ot_version() -> int:
    return int(lib().ot_version())


def ot_last_error_string() -> str:
    return lib().ot_last_error_string().decode()


def ot_options_default() -> OtOptions:
    o = OtOptions()
    lib().ot_options_default(ctypes.byref(o))
    return o


def ot_sinkhorn_pointcloud(x, y, a, b, n, m, d, eps, scale_cost, n_iters, tol, f, g, stream,
                           opt: OtOptions | None = None, want_plan: bool = True):
    """Returns (status, plan handle or None, OtInfo); raises OTError on errors."""
    plan = ctypes.c_void_p()
    info = OtInfo()
    st = lib().ot_sinkhorn_pointcloud(x, y, a, b, n, m, d, eps, int(scale_cost), n_iters, tol, f, g,
                                      stream, ctypes.byref(opt) if opt is not None else None,
                                      ctypes.byref(plan) if want_plan else None,
                                      ctypes.byref(info))
    _check(st)
    return st, (plan.value if want_plan else None), info


def ot_sinkhorn_pointcloud_host(x, y, a, b, n, m, d, eps, scale_cost, n_iters, tol, f, g, stream,
                                opt: OtOptions | None = None, want_plan: bool = False):
    """As ot_sinkhorn_pointcloud with HOST pointers for x, y, a, b, f, g (the
    library copies them in and f, g back). Returns (status, plan or None, OtInfo)."""
    plan = ctypes.c_void_p()
    info = OtInfo()
    st = lib().ot_sinkhorn_pointcloud_host(x, y, a, b, n, m, d, eps, int(scale_cost), n_iters, tol, f, g,
                                           stream, ctypes.byref(opt) if opt is not None else None,
                                           ctypes.byref(plan) if want_plan else None,
                                           ctypes.byref(info))
    _check(st)
    return st, (plan.value if want_plan else None), info


def ot_max_sqdist(x, y, n, m, d, x_lo, x_hi, stream) -> float:
    """max over i in [x_lo, x_hi), all j of ||x_i - y_j||^2 (the max_cost pass's value)."""
    out = ctypes.c_float()
    _check(lib().ot_max_sqdist(x, y, n, m, d, x_lo, x_hi, ctypes.byref(out), stream))
    return out.value


def ot_shard_plan_create(x, y, a, b, n, m, d, eps, scale_cost, x_lo, x_hi, y_lo, y_hi, stream,
                         opt: OtOptions | None = None):
    """Returns (plan handle, OtInfo) of a plan for the given row ranges."""
    plan = ctypes.c_void_p()
    info = OtInfo()
    _check(lib().ot_shard_plan_create(x, y, a, b, n, m, d, eps, int(scale_cost), x_lo, x_hi, y_lo, y_hi,
                                      stream, ctypes.byref(opt) if opt is not None else None,
                                      ctypes.byref(plan), ctypes.byref(info)))
    return plan.value, info


def ot_shard_half_step(plan, side, other, cur, out, stream, want_resid=True):
    """One half-step over the plan's rows; returns the range's residual part (or None)."""
    r = ctypes.c_double()
    _check(lib().ot_shard_half_step(plan, side, other, cur, out, ctypes.byref(r) if want_resid else None,
                                    stream))
    return r.value if want_resid else None


def ot_testing_fail_device_allocs(after: int) -> None:
    """Failure tests only: the device allocation after `after` more fails (see the testing header)."""
    lib().ot_testing_fail_device_allocs(int(after))


def ot_testing_wait_fault(mode: int) -> None:
    """Failure tests only: make one bounded device wait give up (see the testing header)."""
    lib().ot_testing_wait_fault(int(mode))


def ot_marginal_residual(plan, stream):
    """Returns (status, row_l1, col_l1)."""
    r, c = ctypes.c_double(), ctypes.c_double()
    st = _check(lib().ot_marginal_residual(plan, ctypes.byref(r), ctypes.byref(c), stream))
    return st, r.value, c.value


def ot_materialize_rows(plan, row_idx, k, out, stream) -> int:
    return _check(lib().ot_materialize_rows(plan, row_idx, k, out, stream))


def ot_materialize_rows_lowrank(Q, R, g, n, m, r, row_idx, k, out, stream):
    return _check(lib().ot_materialize_rows_lowrank(Q, R, g, n, m, r, row_idx, k, out, stream))


def ot_materialize_rows_lrcost(cost1, cost2, f, g, n, m, r, bias, inv_scale_cost, eps, row_idx, k,
                               out, stream):
    return _check(lib().ot_materialize_rows_lrcost(cost1, cost2, f, g, n, m, r, bias, inv_scale_cost,
                                                   eps, row_idx, k, out, stream))


def ot_sparsify_csr(plan, block_rows, thr, row_ptr, col_idx, vals, capacity, stream):
    """Returns (status, nnz); row_ptr / col_idx / vals: device pointers."""
    nnz = ctypes.c_int64()
    st = lib().ot_sparsify_csr(plan, block_rows, thr, row_ptr, col_idx or None, vals or None,
                               capacity, ctypes.byref(nnz), stream)
    if st != OT_ERR_OVERFLOW:
        _check(st)
    return st, nnz.value


def ot_sparsify_min_row(plan, block_rows, row_counts, stream):
    """Returns (status, thr, nnz, n_massless, argmin); row_counts: device int64 [n] or 0."""
    thr = ctypes.c_float()
    nnz, nm, arg = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    st = _check(lib().ot_sparsify_min_row(plan, block_rows, ctypes.byref(thr), row_counts or None,
                                          ctypes.byref(nnz), ctypes.byref(nm), ctypes.byref(arg),
                                          stream))
    return st, thr.value, nnz.value, nm.value, arg.value


def ot_marginal_residual_range(plan, row_lo, row_hi, col_lo, col_hi, stream):
    """Returns (row_part, col_part) over rows [row_lo, row_hi) and columns [col_lo, col_hi)."""
    r, c = ctypes.c_double(), ctypes.c_double()
    _check(lib().ot_marginal_residual_range(plan, row_lo, row_hi, col_lo, col_hi, ctypes.byref(r),
                                            ctypes.byref(c), stream))
    return r.value, c.value


def ot_min_row_range(plan, row_lo, row_hi, block_rows, stream):
    """Returns (thr, argmin, n_massless) of rows [row_lo, row_hi)."""
    thr = ctypes.c_float()
    arg, nm = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ot_min_row_range(plan, row_lo, row_hi, block_rows, ctypes.byref(thr), ctypes.byref(arg),
                                  ctypes.byref(nm), stream))
    return thr.value, arg.value, nm.value


def ot_kept_counts_range(plan, row_lo, row_hi, block_rows, thr, row_counts, stream):
    """Returns nnz of rows [row_lo, row_hi) at thr; row_counts: device int64 [row_hi - row_lo] or 0."""
    nnz = ctypes.c_int64()
    _check(lib().ot_kept_counts_range(plan, row_lo, row_hi, block_rows, thr, row_counts or None,
                                      ctypes.byref(nnz), stream))
    return nnz.value


def ot_row_pass_stats(plan):
    """Returns (tiles evaluated, tiles of a full visit) of the plan's last row call."""
    v, t = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ot_row_pass_stats(plan, ctypes.byref(v), ctypes.byref(t)))
    return v.value, t.value


def ot_marginal_residual_noalloc(x, y, a, b, f, g, n, m, d, eps, inv_scale_cost, stream):
    """Returns (status, row_l1, col_l1); allocates nothing (see the header)."""
    r, c = ctypes.c_double(), ctypes.c_double()
    st = _check(lib().ot_marginal_residual_noalloc(x, y, a, b, f, g, n, m, d, eps, inv_scale_cost,
                                                   ctypes.byref(r), ctypes.byref(c), stream))
    return st, r.value, c.value


def ot_trim_cache() -> None:
    lib().ot_trim_cache()


def ot_plan_destroy(plan) -> None:
    if plan:
        lib().ot_plan_destroy(plan)
