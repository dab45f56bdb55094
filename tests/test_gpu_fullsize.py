"""Full-size workloads on the GPU, checked against the float64 oracle (-m gpu).

A full oracle trajectory is out of reach beyond the 8000-point workload, so each
test runs the GPU at the workload's real size and launch shape and checks:
 - teacher-forced steps: one GPU iteration from the GPU's own state, against the
   oracle's f-update on sampled rows (from the same g) and g-update on sampled
   columns (from the GPU's new f) -- the sampled checks of "FlashSinkhorn 2",
   sections 3.1 and B.2, used as a verifier;
 - plan entries, residuals and min_row at the GPU's potentials, in full where the
   oracle can afford it (8000 x 8000), on sampled rows otherwise;
 - the captured scale: exact for "mean" (closed form) and for "max_cost" (the
   farthest point of y from any x is a vertex of y's convex hull).
"""
import numpy as np
import pytest

import helpers as H

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
SAMPLE = 512


@pytest.fixture(scope="module")
def ot():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import log_domain_sinkhorn_online_b200 as pkg
    return pkg


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _max_sqdist_hull(x, y):
    """max_ij ||x_i - y_j||^2 exactly: only vertices of y's hull can be farthest."""
    from scipy.spatial import ConvexHull
    yd = np.asarray(y, np.float64)
    yv = yd[ConvexHull(yd).vertices]
    best = 0.0
    for i0 in range(0, x.shape[0], 65536):
        xb = np.asarray(x[i0:i0 + 65536], np.float64)
        best = max(best, float(((xb[:, None, :] - yv[None]) ** 2).sum(-1).max()))
    return best


def _teacher_forced(ot, orc, w, x, y, a, b, f0, g0, c, maxc, seed, **kw):
    """One GPU iteration from (f0, g0) vs the oracle on sampled rows/columns."""
    import torch
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=1, f=f0.clone(), g=g0.clone(),
                    warm_start=True, **kw)
    torch.cuda.synchronize()
    assert p.info.inv_scale_cost == pytest.approx(c, rel=1e-6)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(w.n, size=min(SAMPLE, w.n), replace=False))
    cols = np.sort(rng.choice(w.m, size=min(SAMPLE, w.m), replace=False))
    g0n = g0.double().cpu().numpy()
    f1 = p.f.double().cpu().numpy()
    g1 = p.g.double().cpu().numpy()
    f_ref = orc.f_step(w.x, w.y, w.a, g0n, c, w.eps, rows=rows)
    g_ref = orc.g_step(w.x, w.y, w.b, f1, c, w.eps, cols=cols)
    ef = H.assert_potentials(f1[rows], f_ref, maxc, what="f (teacher-forced)")
    eg = H.assert_potentials(g1[cols], g_ref, maxc, what="g (teacher-forced)")
    p.close()
    return ef, eg


def test_w2_8000_full_path(ot, orc):
    """The benchmarked workload, in the bench's launch shape: solve to tol / cap,
    then the full oracle residual, min_row and rows at the GPU's potentials."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=w.n_iters, tol=w.tol)
    c = plan.info.inv_scale_cost
    xd, yd = w.x.astype(np.float64), w.y.astype(np.float64)
    mean = (xd ** 2).sum(1).mean() + (yd ** 2).sum(1).mean() - 2 * xd.mean(0) @ yd.mean(0)
    assert c == pytest.approx(1.0 / mean, rel=1e-9)
    maxc = H.max_cost(w.x, w.y, c)
    _teacher_forced(ot, orc, w, x, y, a, b, plan.f, plan.g, c, maxc, seed=1)
    f, g = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    r = plan.marginal_residual()
    r_ref = orc.marginal_residual(w.x, w.y, w.a, w.b, f, g, c, w.eps)
    assert abs(r[0] - r_ref[0]) <= H.RES_TOL and abs(r[1] - r_ref[1]) <= H.RES_TOL
    # the in-loop residual (float32 LSE) agrees with the float64 one
    assert plan.info.residual == pytest.approx(r_ref[0], rel=1e-3)
    mr = plan.sparsify_min_row(block_rows=w.block_rows)
    ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps, block_rows=w.block_rows)
    H.assert_min_row(mr, ref)
    # kept counts agree except entries inside the tie band around thr
    assert abs(mr["nnz"] - ref["nnz"]) <= max(2, ref["nnz"] // 10000)
    rows = torch.arange(3 * 1024, 4 * 1024, device="cuda")
    T = plan.materialize_rows(rows).double().cpu().numpy()
    H.assert_entries(T[::16], orc.materialize_rows(w.x, w.y, f, g, c, w.eps, rows.cpu().numpy()[::16]))
    # compressed-row sparsify in the same row blocks: min_row's counts, and on
    # sampled rows the oracle's kept entries (outside the tie band) and values
    csr = plan.sparsify_csr(block_rows=w.block_rows)
    assert csr["thr"] == mr["thr"] and csr["nnz"] == mr["nnz"]
    row_ptr = csr["row_ptr"].cpu().numpy()
    np.testing.assert_array_equal(np.diff(row_ptr), mr["counts"].cpu().numpy())
    col_idx, vals = csr["col_idx"].cpu().numpy(), csr["vals"].cpu().numpy()
    pick = np.arange(0, w.n, 397)
    Tref = orc.materialize_rows(w.x, w.y, f, g, c, w.eps, pick)
    ref_ptr = np.concatenate([[0], np.cumsum((Tref >= csr["thr"]).sum(1))])
    ref_cols = np.concatenate([np.nonzero(r >= csr["thr"])[0] for r in Tref])
    ref_vals = np.concatenate([r[r >= csr["thr"]] for r in Tref])
    got_ptr = np.concatenate([[0], np.cumsum([row_ptr[i + 1] - row_ptr[i] for i in pick])])
    got_cols = np.concatenate([col_idx[row_ptr[i]:row_ptr[i + 1]] for i in pick])
    got_vals = np.concatenate([vals[row_ptr[i]:row_ptr[i + 1]] for i in pick])
    H.assert_csr((got_ptr, got_cols, got_vals), (ref_ptr, ref_cols, ref_vals), csr["thr"])


def test_w3_tensor_core_full_size(ot, orc):
    """40000 x 50000, d = 50 on the tcgen05 path: 500 iterations, then a
    teacher-forced step and sampled rows at the GPU's potentials."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w3()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=w.n_iters)
    c = plan.info.inv_scale_cost
    f, g = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    assert np.isfinite(f).all() and np.isfinite(g).all()
    maxc = H.max_cost(w.x, w.y, c)
    _teacher_forced(ot, orc, w, x, y, a, b, plan.f, plan.g, c, maxc, seed=3)
    rows = np.sort(np.random.default_rng(5).choice(w.n, 16, replace=False)).astype(np.int64)
    T = plan.materialize_rows(torch.from_numpy(rows).cuda()).double().cpu().numpy()
    H.assert_entries(T, orc.materialize_rows(w.x, w.y, f, g, c, w.eps, rows))


def test_w4_million_points_step(ot, orc):
    """10^6 x 10^6 uniform vs 64 clusters at the final eps: two GPU iterations
    from zero, then a teacher-forced step (sampled rows and columns)."""
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w4()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=2)
    maxc = _max_sqdist_hull(w.x, w.y)
    _teacher_forced(ot, orc, w, x, y, a, b, plan.f, plan.g, 1.0, maxc, seed=4)


def test_w5_two_million_points_step_and_rows(ot, orc):
    """2*10^6 spirals, scale max_cost (checked exactly), eps 1e-3: a teacher-forced
    step, then one 4096-row block of the 65,536 rows (32.8 GB) and sampled rows."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w5()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=2)
    mx = _max_sqdist_hull(w.x, w.y)
    c = plan.info.inv_scale_cost
    # the pass runs in float32 on shifted coordinates: ~1e-7 relative
    assert c == pytest.approx(1.0 / mx, rel=1e-6)
    _teacher_forced(ot, orc, w, x, y, a, b, plan.f, plan.g, c, 1.0, seed=5)
    f, g = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    rows = torch.from_numpy(w.rows[:w.block_rows]).cuda()
    out = torch.empty((w.block_rows, w.m), dtype=torch.float32, device="cuda")
    plan.materialize_rows(rows, out=out)
    pick = np.arange(0, w.block_rows, 128)
    T = out[torch.from_numpy(pick).cuda()].double().cpu().numpy()
    del out
    H.assert_entries(T, orc.materialize_rows(w.x, w.y, f, g, c, w.eps, w.rows[pick]))
