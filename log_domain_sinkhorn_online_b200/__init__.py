"""Online log-domain Sinkhorn for point clouds on NVIDIA B200 (sm_100a).

Entropic OT between x[n,d] and y[m,d] under squared-Euclidean cost, computed
by hand-written CUDA kernels behind the C ABI of ``include/ot_sinkhorn.h``
("FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", section 2.1, for
the streaming log-sum-exp half-steps; moscot PR #846, section Fix, for the
plan rows and the captured scale). PyTorch only supplies device memory and
streams here: every step runs in the library's kernels.

    import torch, log_domain_sinkhorn_online_b200 as ot
    plan = ot.sinkhorn(x, y, a, b, eps=0.01, scale="mean", n_iters=2000, tol=1e-3)
    rows = plan.materialize_rows(torch.arange(16, device="cuda"))
    thr, counts, nnz = plan.sparsify_min_row(block_rows=1024)
"""
from __future__ import annotations

from . import _binding as B
from ._binding import OTError  # noqa: F401

_SCALES = {"none": B.OT_SCALE_NONE, "mean": B.OT_SCALE_MEAN, "max_cost": B.OT_SCALE_MAX_COST}


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t, dtype, name):
    import torch
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Plan:
    """A solved problem: potentials f, g and the captured eps / scale (owns the C plan)."""

    def __init__(self, handle, x, y, a, b, f, g, info, status):
        self._h = handle
        self._keep = (x, y, a, b)
        self.f, self.g, self.info, self.status = f, g, info, status

    def close(self):
        if self._h:
            B.ot_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def marginal_residual(self, stream=None):
        _, r, c = B.ot_marginal_residual(self._h, _stream(stream))
        return r, c

    def row_pass_stats(self):
        """(tiles evaluated, tiles of a full visit) in the last row call (d <= 3)."""
        return B.ot_row_pass_stats(self._h)

    def materialize_rows(self, row_idx, out=None, stream=None):
        import torch
        row_idx = _dev(row_idx, torch.int64, "row_idx")
        k = row_idx.numel()
        if out is None:
            out = torch.empty((k, self.g.numel()), dtype=torch.float32, device=row_idx.device)
        _dev(out, torch.float32, "out")
        B.ot_materialize_rows(self._h, row_idx.data_ptr(), k, out.data_ptr(), _stream(stream))
        return out

    def sparsify_min_row(self, block_rows=0, counts=None, stream=None):
        """Returns dict(thr, counts, nnz, n_massless, argmin, status)."""
        import torch
        if counts is None:
            counts = torch.empty(self.f.numel(), dtype=torch.int64, device=self.f.device)
        _dev(counts, torch.int64, "counts")
        st, thr, nnz, nm, arg = B.ot_sparsify_min_row(self._h, int(block_rows), counts.data_ptr(),
                                                      _stream(stream))
        return dict(thr=thr, counts=counts, nnz=nnz, n_massless=nm, argmin=arg, status=st)

    def sparsify_csr(self, thr=None, block_rows=0, capacity=None, out=None, stream=None):
        """The plan thresholded at thr (default: the min_row threshold) in
        compressed-row form. Returns dict(row_ptr [n+1] int64, col_idx [nnz]
        int64, vals [nnz] float32, nnz, thr); torch.sparse_csr_tensor(row_ptr,
        col_idx, vals, (n, m)) turns it into a torch sparse matrix. out: an
        optional (row_ptr, col_idx, vals) of device tensors to write into (the
        capacity is col_idx's length)."""
        import torch
        dev = self.f.device
        n = self.f.numel()
        if thr is None:
            mr = self.sparsify_min_row(block_rows=block_rows, stream=stream)
            thr = mr["thr"]
            if capacity is None and out is None:
                capacity = mr["nnz"]
        if out is not None:
            row_ptr, col_idx, vals = out
            _dev(row_ptr, torch.int64, "row_ptr")
            _dev(col_idx, torch.int64, "col_idx")
            _dev(vals, torch.float32, "vals")
            if row_ptr.numel() != n + 1 or vals.numel() < col_idx.numel():
                raise ValueError("out: row_ptr needs n + 1 entries and vals as many as col_idx")
            capacity = col_idx.numel()
        else:
            row_ptr = torch.empty(n + 1, dtype=torch.int64, device=dev)
            if capacity is None:  # size it first: a call with no room only counts
                _, capacity = B.ot_sparsify_csr(self._h, int(block_rows), float(thr),
                                                row_ptr.data_ptr(), 0, 0, 0, _stream(stream))
            col_idx = torch.empty(max(int(capacity), 1), dtype=torch.int64, device=dev)
            vals = torch.empty(max(int(capacity), 1), dtype=torch.float32, device=dev)
        st, nnz = B.ot_sparsify_csr(self._h, int(block_rows), float(thr), row_ptr.data_ptr(),
                                    col_idx.data_ptr(), vals.data_ptr(), int(capacity), _stream(stream))
        if st == B.OT_ERR_OVERFLOW:
            raise B.OTError(st, B.ot_last_error_string())
        return dict(row_ptr=row_ptr, col_idx=col_idx[:nnz], vals=vals[:nnz], nnz=nnz, thr=thr)


def _rows_out(row_idx, m, out, dev):
    import torch
    row_idx = _dev(row_idx, torch.int64, "row_idx")
    if out is None:
        out = torch.empty((row_idx.numel(), m), dtype=torch.float32, device=dev)
    _dev(out, torch.float32, "out")
    if out.shape != (row_idx.numel(), m):
        raise ValueError("out must be [k, m]")
    return row_idx, out


def lowrank_rows(Q, R, g, row_idx, out=None, stream=None):
    """Rows (Q diag(1/g) R^T)[row_idx] of a low-rank coupling; Q [n, r], R [m, r],
    g [r] float32 CUDA tensors. Returns out [k, m] float32."""
    import torch
    Q, R, g = _dev(Q, torch.float32, "Q"), _dev(R, torch.float32, "R"), _dev(g, torch.float32, "g")
    n, r = Q.shape
    m = R.shape[0]
    if R.shape[1] != r or g.numel() != r:
        raise ValueError("Q [n, r], R [m, r] and g [r] must share r")
    row_idx, out = _rows_out(row_idx, m, out, Q.device)
    B.ot_materialize_rows_lowrank(Q.data_ptr(), R.data_ptr(), g.data_ptr(), n, m, r, row_idx.data_ptr(),
                                  row_idx.numel(), out.data_ptr(), _stream(stream))
    return out


def lrcost_rows(cost1, cost2, f, g, row_idx, eps, inv_scale_cost=1.0, bias=0.0, out=None, stream=None):
    """Entropic rows exp((f_i + g_j - c (cost1[i].cost2[j] + bias)) / eps) on a
    low-rank cost geometry; cost1 [n, r], cost2 [m, r], f [n], g [m] float32
    CUDA tensors. Returns out [k, m] float32."""
    import torch
    c1, c2 = _dev(cost1, torch.float32, "cost1"), _dev(cost2, torch.float32, "cost2")
    f, g = _dev(f, torch.float32, "f"), _dev(g, torch.float32, "g")
    n, r = c1.shape
    m = c2.shape[0]
    if c2.shape[1] != r or f.numel() != n or g.numel() != m:
        raise ValueError("cost1 [n, r], cost2 [m, r], f [n], g [m]")
    row_idx, out = _rows_out(row_idx, m, out, c1.device)
    B.ot_materialize_rows_lrcost(c1.data_ptr(), c2.data_ptr(), f.data_ptr(), g.data_ptr(), n, m, r,
                                 float(bias), float(inv_scale_cost), float(eps), row_idx.data_ptr(),
                                 row_idx.numel(), out.data_ptr(), _stream(stream))
    return out


def sinkhorn(x, y, a, b, eps, scale="none", n_iters=100, tol=0.0, f=None, g=None, warm_start=False,
             check_every=16, use_graphs=True, eps_init=0.0, eps_decay=0.7, iters_per_stage=20,
             timing=False, col_splits=0, rows_per_thread=0, tensor_cores=True,
             device_loop=-1, block_sparse=False, sparse_block=0, sparse_verify=True,
             sparse_delta=0.0, sparse_dense_frac=0.5, resid_history=None, sparse_mask_out=None,
             stream=None) -> Plan:
    """Solves on the GPU; x [n,d], y [m,d], a [n], b [m] float32 CUDA tensors.

    block_sparse (d <= 3): block-sparse fine iterations ("FlashSinkhorn 2",
    sections 3.2, A.3, B.3): Morton-ordered blocks of sparse_block points, a
    box screen and (sparse_verify) an exact-mass check of every block pair
    against delta * min weight (sparse_delta, 0 = tol / (4 max(NB, MB))), the
    half-steps over the admitted tiles only; an iteration whose candidates
    exceed sparse_dense_frac of all pairs runs dense. f and g come back in the
    caller's order.

    resid_history: optional float64 CUDA tensor; entry k - 1 receives the
    in-loop ||T1 - a||_1 after iteration k (NaN where none was measured).
    sparse_mask_out: optional uint8 CUDA tensor of at least NB * MB bytes; the
    block mask of the first fine update (at the starting potentials).
    """
    import torch
    x, y = _dev(x, torch.float32, "x"), _dev(y, torch.float32, "y")
    a, b = _dev(a, torch.float32, "a"), _dev(b, torch.float32, "b")
    n, d = x.shape
    m = y.shape[0]
    f = torch.empty(n, dtype=torch.float32, device=x.device) if f is None else _dev(f, torch.float32, "f")
    g = torch.empty(m, dtype=torch.float32, device=x.device) if g is None else _dev(g, torch.float32, "g")
    opt = B.ot_options_default()
    opt.warm_start = int(warm_start)
    opt.check_every = int(check_every)
    opt.use_graphs = int(use_graphs)
    opt.eps_init = float(eps_init)
    opt.eps_decay = float(eps_decay)
    opt.iters_per_stage = int(iters_per_stage)
    opt.timing = int(timing)
    opt.col_splits = int(col_splits)
    opt.rows_per_thread = int(rows_per_thread)
    opt.tensor_cores = int(bool(tensor_cores))
    opt.device_loop = int(device_loop)
    opt.block_sparse = int(bool(block_sparse))
    opt.sparse_block = int(sparse_block)
    opt.sparse_verify = int(bool(sparse_verify))
    opt.sparse_delta = float(sparse_delta)
    opt.sparse_dense_frac = float(sparse_dense_frac)
    if sparse_mask_out is not None:
        _dev(sparse_mask_out, torch.uint8, "sparse_mask_out")
        opt.sparse_mask_out = sparse_mask_out.data_ptr()
        opt.sparse_mask_len = sparse_mask_out.numel()
    if resid_history is not None:
        _dev(resid_history, torch.float64, "resid_history")
        opt.resid_history = resid_history.data_ptr()
        opt.resid_history_len = resid_history.numel()
    if isinstance(scale, str):
        sc = _SCALES[scale]
    else:
        sc = B.OT_SCALE_VALUE
        opt.scale_value = float(scale)
    st, h, info = B.ot_sinkhorn_pointcloud(x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(),
                                           n, m, d, float(eps), sc, int(n_iters), float(tol),
                                           f.data_ptr(), g.data_ptr(), _stream(stream), opt)
    return Plan(h, x, y, a, b, f, g, info, st)
