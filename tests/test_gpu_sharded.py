"""The row-split solve's device half on one GPU (-m gpu).

ot_shard_half_step updates one rank's range of rows; here the ranks of a split
are run one after the other on the same GPU, each writing its own range of the
shared potential buffers, which is exactly what every rank's buffer holds after
the all-gather. With tile-aligned ranges and the same column splits and rows
per thread, every row tile is computed as in the unsplit solve, so the split
solve's potentials must equal the unsplit ones bit for bit (d = 3 on the CUDA
cores, d = 24 on the tensor cores). The residual parts must sum to the unsplit
in-loop residual (another summation order), ot_max_sqdist over the ranges must
give the unsplit max_cost exactly, and the driver of the split solve
(log_domain_sinkhorn_online_b200.sharded) must give the same result at world
size 1.

The row calls over ranges (ot_marginal_residual_range, ot_min_row_range,
ot_kept_counts_range) combined over the ranks of a split as the all-reduces
combine them must give the whole-plan calls' values: thr, argmin, the massless
count, the counts and nnz exactly, the residual to 1e-12 (another summation
order).
"""
import numpy as np
import pytest

import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ot():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import log_domain_sinkhorn_online_b200 as pkg
    return pkg


def _emulated_split(ot, x, y, a, b, eps, scale, world, iters, align, **opts):
    import torch
    from log_domain_sinkhorn_online_b200 import sharded as S
    n, m = x.shape[0], y.shape[0]
    xr, yr = S.Ranges(n, world, align), S.Ranges(m, world, align)
    ranks = [S.CudaShard(x, y, a, b, eps, scale, xr, yr, r, **opts) for r in range(world)]
    f = [torch.zeros(xr.padded, device="cuda"), torch.zeros(xr.padded, device="cuda")]
    g = torch.zeros(yr.padded, device="cuda")
    k, resid = 0, None
    for it in range(iters + 1):
        parts = [sh.half_step(0, g, f[k], f[k ^ 1], True) for sh in ranks]
        resid = sum(parts)
        if it == iters:
            break  # the final f-update only measures the residual
        for sh in ranks:
            sh.half_step(1, f[k ^ 1], g, g, False)
        k ^= 1
    for sh in ranks:
        sh.close()
    return f[k][:n].cpu().numpy(), g[:m].cpu().numpy(), resid, ranks[0].info


@pytest.mark.parametrize("world", [2, 3])
def test_split_d3_equals_unsplit_bit_for_bit(ot, world):
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=3000, m=2600)
    x, y, a, b = H.to_dev(w)
    opts = dict(col_splits=4, rows_per_thread=2)
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=10, device_loop=0, **opts)
    fr, gr, rr = p.f.cpu().numpy(), p.g.cpu().numpy(), p.info.residual
    p.close()
    f, g, resid, info = _emulated_split(ot, x, y, a, b, w.eps, w.scale, world, 10, 1024, **opts)
    assert info.col_splits == 4
    np.testing.assert_array_equal(f, fr)
    np.testing.assert_array_equal(g, gr)
    assert resid == pytest.approx(rr, rel=1e-9)


def test_split_tensor_cores_equal_unsplit_bit_for_bit(ot):
    import torch
    rng = np.random.default_rng(11)
    n, m, d = 1000, 700, 24
    x = torch.from_numpy(rng.random((n, d), dtype=np.float32)).cuda()
    y = torch.from_numpy(rng.random((m, d), dtype=np.float32)).cuda()
    a = torch.full((n,), 1.0 / n, device="cuda")
    b = torch.full((m,), 1.0 / m, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=0.5, scale="mean", n_iters=6, col_splits=2)
    fr, gr = p.f.cpu().numpy(), p.g.cpu().numpy()
    p.close()
    f, g, _, _ = _emulated_split(ot, x, y, a, b, 0.5, "mean", 3, 6, 128, col_splits=2)
    np.testing.assert_array_equal(f, fr)
    np.testing.assert_array_equal(g, gr)


def test_max_sqdist_over_ranges_is_the_max_cost(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    from log_domain_sinkhorn_online_b200 import sharded as S
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w5(n=20000)
    x, y, a, b = H.to_dev(w)
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale="max_cost", n_iters=1)
    c = p.info.inv_scale_cost
    p.close()
    xr = S.Ranges(w.n, 3, 1024)
    s = torch.cuda.current_stream().cuda_stream
    vals = [B.ot_max_sqdist(x.data_ptr(), y.data_ptr(), w.n, w.m, 3, xr.lo(r), xr.hi(r), s) for r in range(3)]
    assert 1.0 / float(np.float32(max(vals))) == c
    assert B.ot_max_sqdist(x.data_ptr(), y.data_ptr(), w.n, w.m, 3, 0, 0, s) == 0.0


def test_driver_at_world_size_one(ot):
    from log_domain_sinkhorn_online_b200 import sharded as S
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w5(n=6000)
    x, y, a, b = H.to_dev(w)
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=8, device_loop=0, col_splits=6,
                    rows_per_thread=2)
    fr, gr, rr = p.f.cpu().numpy(), p.g.cpu().numpy(), p.info.residual
    p.close()
    xr, yr = S.Ranges(w.n, 1), S.Ranges(w.m, 1)
    scale = S.max_cost_value(x, y, xr, 0)
    sh = S.CudaShard(x, y, a, b, w.eps, scale, xr, yr, 0, col_splits=6, rows_per_thread=2)
    solver = S.ShardedSinkhorn(sh, xr, yr, 0, 1, like=x)
    done, resid = solver.solve(8)
    f, g = solver.potentials()
    sh.close()
    assert done == 8
    np.testing.assert_array_equal(f.cpu().numpy(), fr)
    np.testing.assert_array_equal(g.cpu().numpy(), gr)
    assert resid == pytest.approx(rr, rel=1e-9)


def test_shard_plan_argument_checks(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    x = torch.zeros((64, 3), device="cuda")
    a = torch.full((64,), 1.0 / 64, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for lo, hi in ((5, 20), (-8, 8), (16, 8), (0, 65)):
        with pytest.raises(B.OTError) as e:
            B.ot_shard_plan_create(x.data_ptr(), x.data_ptr(), a.data_ptr(), a.data_ptr(), 64, 64, 3, 0.1,
                                   B.OT_SCALE_NONE, lo, hi, 0, 64, s)
        assert e.value.status == B.OT_ERR_INVALID_ARG
    plan, _ = B.ot_shard_plan_create(x.data_ptr(), x.data_ptr(), a.data_ptr(), a.data_ptr(), 64, 64, 3, 0.1,
                                     B.OT_SCALE_NONE, 0, 64, 8, 40, s)
    out = torch.empty((1, 64), device="cuda")
    rows = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(B.OTError):  # row calls refuse a split plan
        B.ot_materialize_rows(plan, rows.data_ptr(), 1, out.data_ptr(), s)
    with pytest.raises(B.OTError):
        B.ot_shard_half_step(plan, 2, x.data_ptr(), a.data_ptr(), a.data_ptr(), s)
    B.ot_plan_destroy(plan)


def test_split_with_empty_ranges_and_massless_rows(ot):
    """Four ranks on 1500 x 1300 points with 1024-row ranges: two ranks own no rows;
    a few massless rows and columns (-inf potentials) pass through unchanged."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=1500, m=1300)
    a = w.a.copy()
    b = w.b.copy()
    a[::97] = 0.0
    b[5::131] = 0.0
    a = (a / a.sum()).astype(np.float32)
    b = (b / b.sum()).astype(np.float32)
    x, y = (torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in (w.x, w.y))
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    opts = dict(col_splits=3, rows_per_thread=2)
    p = ot.sinkhorn(x, y, at, bt, eps=w.eps, scale=w.scale, n_iters=7, device_loop=0, **opts)
    fr, gr = p.f.cpu().numpy(), p.g.cpu().numpy()
    p.close()
    f, g, _, _ = _emulated_split(ot, x, y, at, bt, w.eps, w.scale, 4, 7, 1024, **opts)
    assert np.isneginf(f[::97]).all() and np.isneginf(g[5::131]).all()
    np.testing.assert_array_equal(f, fr)
    np.testing.assert_array_equal(g, gr)


def _massless_problem(d, n, m, seed):
    import torch
    rng = np.random.default_rng(seed)
    x = rng.random((n, d), dtype=np.float32)
    y = rng.random((m, d), dtype=np.float32)
    a = rng.random(n).astype(np.float32) + 0.1
    a[::53] = 0.0
    a = (a / a.sum()).astype(np.float32)
    b = np.full(m, 1.0 / m, dtype=np.float32)
    return tuple(torch.from_numpy(v).cuda() for v in (x, y, a, b))


@pytest.mark.parametrize("d,world,block_rows", [(3, 2, 0), (3, 3, 64), (2, 4, 0), (5, 3, 0)])
def test_range_row_calls_combine_to_the_whole_plan(ot, d, world, block_rows):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    from log_domain_sinkhorn_online_b200 import sharded as S
    n, m = 2100, 1700
    x, y, a, b = _massless_problem(d, n, m, 40 + d)
    p = ot.sinkhorn(x, y, a, b, eps=0.02, scale="mean", n_iters=5)
    whole = p.sparsify_min_row(block_rows=block_rows)
    rw, cw = p.marginal_residual()
    s = torch.cuda.current_stream().cuda_stream
    xr, yr = S.Ranges(n, world, 256), S.Ranges(m, world, 256)
    thr, arg, nm, nnz, rr, cc = np.inf, -1, 0, 0, 0.0, 0.0
    cands = []
    counts = torch.full((n,), -1, dtype=torch.int64, device="cuda")
    for r in range(world):
        lo, hi = xr.lo(r), xr.hi(r)
        t, ar, k = B.ot_min_row_range(p.handle, lo, hi, block_rows, s)
        cands.append((t, ar))
        thr, nm = min(thr, t), nm + k
        part_r, part_c = B.ot_marginal_residual_range(p.handle, lo, hi, yr.lo(r), yr.hi(r), s)
        rr, cc = rr + part_r, cc + part_c
    arg = min((ar for t, ar in cands if t == thr and ar >= 0), default=-1)
    for r in range(world):
        lo, hi = xr.lo(r), xr.hi(r)
        nnz += B.ot_kept_counts_range(p.handle, lo, hi, block_rows, thr,
                                      counts[lo:].data_ptr() if hi > lo else 0, s)
    assert whole["n_massless"] == nm == len(range(0, n, 53))
    assert thr == whole["thr"] and arg == whole["argmin"] and nnz == whole["nnz"]
    assert torch.equal(counts, whole["counts"])
    assert rr == pytest.approx(rw, rel=1e-12) and cc == pytest.approx(cw, rel=1e-12)
    p.close()


def test_sharded_rows_driver_at_world_size_one(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import sharded as S
    n, m = 3000, 2500
    x, y, a, b = _massless_problem(3, n, m, 7)
    p = ot.sinkhorn(x, y, a, b, eps=0.01, scale="max_cost", n_iters=8)
    whole = p.sparsify_min_row()
    rw, cw = p.marginal_residual()
    rows = torch.arange(0, n, 7, device="cuda")
    T = p.materialize_rows(rows)
    from log_domain_sinkhorn_online_b200 import _binding as B
    vmax = B.ot_max_sqdist(x.data_ptr(), y.data_ptr(), n, m, 3, 0, n, torch.cuda.current_stream().cuda_stream)
    back = S.CudaRows(x, y, a, b, p.f, p.g, 0.01, vmax)
    # the max_cost value passed as a value resolves the same inv_scale_cost
    assert back.plan.info.inv_scale_cost == p.info.inv_scale_cost
    sr = S.ShardedRows(back, S.Ranges(n, 1), S.Ranges(m, 1), 0, 1, device=x.device)
    mr = sr.min_row()
    assert (mr["thr"], mr["argmin"], mr["n_massless"], mr["nnz"]) == \
        (whole["thr"], whole["argmin"], whole["n_massless"], whole["nnz"])
    assert torch.equal(mr["counts"], whole["counts"])
    assert sr.marginal_residual() == pytest.approx((rw, cw), rel=1e-12)
    lo, hi = S.share(rows.numel(), 0, 1)
    assert torch.equal(back.materialize(rows[lo:hi]), T)
    back.close()
    p.close()


def test_range_calls_check_their_ranges(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    x, y, a, b = _massless_problem(3, 300, 200, 3)
    p = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=2)
    s = torch.cuda.current_stream().cuda_stream
    for lo, hi in ((-1, 10), (20, 10), (0, 301)):
        for call in (lambda: B.ot_min_row_range(p.handle, lo, hi, 0, s),
                     lambda: B.ot_kept_counts_range(p.handle, lo, hi, 0, 0.5, 0, s),
                     lambda: B.ot_marginal_residual_range(p.handle, lo, hi, 0, 200, s)):
            with pytest.raises(B.OTError) as e:
                call()
            assert e.value.status == B.OT_ERR_INVALID_ARG
    with pytest.raises(B.OTError):
        B.ot_marginal_residual_range(p.handle, 0, 300, 0, 201, s)
    with pytest.raises(B.OTError):
        B.ot_kept_counts_range(p.handle, 0, 300, 0, float("nan"), 0, s)
    # empty ranges: nothing to reduce
    assert B.ot_min_row_range(p.handle, 5, 5, 0, s) == (float("inf"), -1, 0)
    assert B.ot_kept_counts_range(p.handle, 5, 5, 0, 0.5, 0, s) == 0
    assert B.ot_marginal_residual_range(p.handle, 5, 5, 7, 7, s) == (0.0, 0.0)
    p.close()
