"""The row-split solve's host logic on CPU ranks (gloo, world sizes 2 and 3).

log_domain_sinkhorn_online_b200.sharded orders the half-steps of each rank's
row ranges and the collectives between them (an all-gather of the updated
potential after every half-step, an all-reduce of the residual parts for the
stopping test). Here every rank's half-step is the float64 oracle's f-/g-update
of its rows (a stand-in backend with the same contract as the library's
ot_shard_half_step), so the split solve must reproduce the oracle's unsplit
trajectory bit for bit -- each row's update depends only on the other side's
whole potential -- and stop after the same iteration with the same residual
(summed in another order: 1e-12 relative). CPU only; no GPU is touched.
"""
import datetime
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleShard:
    """The oracle's half-step over one rank's rows (float64, CPU tensors)."""

    def __init__(self, w, c, xr, yr, rank):
        import oracle
        self.orc, self.w, self.c = oracle, w, c
        self.xs = (xr.lo(rank), xr.hi(rank))
        self.ys = (yr.lo(rank), yr.hi(rank))

    def half_step(self, side, other, cur, out, want_resid):
        import torch
        w, orc = self.w, self.orc
        lo, hi = self.xs if side == 0 else self.ys
        if hi <= lo:
            return 0.0
        idx = np.arange(lo, hi, dtype=np.int64)
        if side == 0:
            new = orc.f_step(w.x, w.y, w.a, other[:w.m].numpy(), self.c, w.eps, rows=idx)
            wts = w.a[lo:hi].astype(np.float64)
        else:
            new = orc.g_step(w.x, w.y, w.b, other[:w.n].numpy(), self.c, w.eps, cols=idx)
            wts = w.b[lo:hi].astype(np.float64)
        old = cur[lo:hi].numpy().copy()
        out[lo:hi] = torch.from_numpy(new)
        if not want_resid:
            return None
        # the rows' sums at the state before the update: w_i exp((old_i - new_i)/eps)
        live = wts > 0
        return float(np.abs(wts[live] * np.exp((old[live] - new[live]) / w.eps) - wts[live]).sum())


def _rank(rank, world, port, q, n_iters, tol):
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from log_domain_sinkhorn_online_b200 import sharded as S
    from log_domain_sinkhorn_online_b200 import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="1")
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        w = workloads.w2(n=301, m=245)
        c = oracle.inv_scale_cost(w.x, w.y, w.scale)
        xr, yr = S.Ranges(w.n, world, align=8), S.Ranges(w.m, world, align=8)
        solver = S.ShardedSinkhorn(OracleShard(w, c, xr, yr, rank), xr, yr, rank, world,
                                   like=torch.zeros(1, dtype=torch.float64))
        done, resid = solver.solve(n_iters, tol)
        f, g = solver.potentials()
        q.put((rank, done, resid, f.numpy().copy(), g.numpy().copy(),
               [(xr.lo(r), xr.hi(r)) for r in range(world)]))
    finally:
        dist.destroy_process_group()


class OracleRows:
    """The oracle's row reductions over a range of rows (float64), the stand-in
    for the library's range calls: min_row and kept counts on the sub-cloud of
    the range's rows, the residual's parts from the oracle's row and column sums."""

    def __init__(self, w, c, f, g):
        import oracle
        self.orc, self.w, self.c, self.f, self.g = oracle, w, c, f, g

    def residual(self, row_lo, row_hi, col_lo, col_hi):
        w = self.w
        _, _, rs, cs = self.orc.marginal_residual(w.x, w.y, w.a, w.b, self.f, self.g, self.c, w.eps,
                                                  return_sums=True)
        a, b = w.a.astype(np.float64), w.b.astype(np.float64)
        return (float(np.abs(rs[row_lo:row_hi] - a[row_lo:row_hi]).sum()),
                float(np.abs(cs[col_lo:col_hi] - b[col_lo:col_hi]).sum()))

    def row_max(self, lo, hi, block_rows):
        if hi <= lo:
            return float("inf"), -1, 0
        w = self.w
        r = self.orc.min_row(w.x[lo:hi], w.y, w.a[lo:hi], self.f[lo:hi], self.g, self.c, w.eps)
        return r["thr"], (r["argmin"] + lo if r["argmin"] >= 0 else -1), r["n_massless"]

    def row_count(self, lo, hi, thr, block_rows):
        if hi <= lo:
            return np.zeros(0, dtype=np.int64), 0
        w = self.w
        row_ptr, _, _ = self.orc.sparsify_csr(w.x[lo:hi], w.y, w.a[lo:hi], self.f[lo:hi], self.g,
                                              self.c, w.eps, thr)
        return np.diff(row_ptr), int(row_ptr[-1])


def _rows_problem():
    """workload 2's recipe on 301 x 245 points with a few massless rows, at the
    oracle's potentials after 6 iterations."""
    import oracle
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=301, m=245)
    a = w.a.copy()
    a[[0, 77, 300]] = 0.0
    w.a = (a / a.sum()).astype(np.float32)
    c = oracle.inv_scale_cost(w.x, w.y, w.scale)
    f, g, _, _ = oracle.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 6)
    return w, c, f, g


def _rows_rank(rank, world, port, q, align):
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from log_domain_sinkhorn_online_b200 import sharded as S
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="1")
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        w, c, f, g = _rows_problem()
        xr, yr = S.Ranges(w.n, world, align=align), S.Ranges(w.m, world, align=align)
        rows = S.ShardedRows(OracleRows(w, c, f, g), xr, yr, rank, world)
        resid = rows.marginal_residual()
        mr = rows.min_row()
        q.put((rank, resid, mr["thr"], mr["argmin"], mr["n_massless"], mr["nnz"],
               np.asarray(mr["counts"]).copy(), (xr.lo(rank), xr.hi(rank))))
    finally:
        dist.destroy_process_group()


def _run(world, n_iters, tol, target=None, args=None):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    target = target or _rank
    args = (n_iters, tol) if args is None else args
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world", [2, 3])
def test_split_solve_reproduces_the_unsplit_trajectory(orc, world):
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=301, m=245)
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    res = _run(world, 12, 0.0)
    f_ref, g_ref, it, r_ref = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 12)
    ranges = res[0][5]
    assert len({hi - lo for lo, hi in ranges if hi > lo}) >= 1 and sum(hi - lo for lo, hi in ranges) == w.n
    for rank, done, resid, f, g, _ in res:
        assert done == 12
        np.testing.assert_array_equal(f, f_ref)   # every rank holds the whole state
        np.testing.assert_array_equal(g, g_ref)
        assert resid == pytest.approx(r_ref, rel=1e-12)
    assert len({r[2] for r in res}) == 1           # one all-reduced value on every rank


def test_split_solve_stops_where_the_oracle_stops(orc):
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=301, m=245)
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    # a tolerance the oracle meets after some iterations, not within rounding of it
    f_ref, g_ref, it, r_ref = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 400, tol=2e-2)
    assert 2 <= it < 400
    res = _run(2, 400, 2e-2)
    for rank, done, resid, f, g, _ in res:
        assert done == it
        assert resid == pytest.approx(r_ref, rel=1e-10)
        np.testing.assert_array_equal(f, f_ref)
        np.testing.assert_array_equal(g, g_ref)


def test_ranges_cover_the_points_once():
    from log_domain_sinkhorn_online_b200.sharded import Ranges
    for count, world, align in ((2_000_000, 8, 1024), (8000, 3, 256), (100, 4, 64), (5, 2, 8)):
        r = Ranges(count, world, align)
        spans = [(r.lo(k), r.hi(k)) for k in range(world)]
        covered = sorted(i for lo, hi in spans for i in range(lo, hi))
        assert covered == list(range(count))
        assert all(lo % align == 0 for lo, hi in spans) and r.padded >= count
        assert r.shard % align == 0


@pytest.mark.parametrize("world,align", [(2, 64), (3, 8), (4, 128)])
def test_split_row_calls_equal_the_whole_plan(orc, world, align):
    """min_row (thr, argmin, massless rows, counts, nnz) and the marginal
    residual with the rows split across gloo ranks equal the oracle's whole-plan
    values; (4, 128) leaves one rank without x rows and two without y rows."""
    w, c, f, g = _rows_problem()
    ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)
    r_ref = orc.marginal_residual(w.x, w.y, w.a, w.b, f, g, c, w.eps)
    assert ref["n_massless"] == 3
    res = _run(world, 0, 0.0, target=_rows_rank, args=(align,))
    counts = np.zeros(w.n, dtype=np.int64)
    for rank, resid, thr, arg, nm, nnz, cnt, (lo, hi) in res:
        assert thr == ref["thr"] and arg == ref["argmin"]
        assert nm == ref["n_massless"] and nnz == ref["nnz"]
        assert resid[0] == pytest.approx(r_ref[0], rel=1e-12)
        assert resid[1] == pytest.approx(r_ref[1], rel=1e-12)
        counts[lo:hi] = cnt
    np.testing.assert_array_equal(counts, ref["counts"])
