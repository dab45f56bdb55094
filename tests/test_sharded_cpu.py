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


def _run(world, n_iters, tol):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, n_iters, tol)) for r in range(world)]
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
