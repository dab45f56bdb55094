"""Full-size workloads on the GPU, checked against the float64 oracle (-m gpu).

A full oracle trajectory is out of reach beyond the 8000-point workload, so each
test runs the GPU at the workload's real size and launch shape and checks:
 - single steps from a seeded state: one GPU f-update from a g drawn by the test,
   against the oracle's f-update on sampled rows from the same g, and the same for
   the g-update with the clouds' roles exchanged -- the sampled checks of
   "FlashSinkhorn 2", sections 3.1 and B.2, used as a verifier;
 - plan entries, residuals and min_row of a plan built at potentials that come
   from the oracle (in full where the oracle can afford it, 8000 x 8000) or, at
   the larger sizes, at sampled rows whose potentials the oracle computed from a
   seeded g;
 - properties of the GPU's own full-size solve (finite potentials, the reported
   residual against the GPU's float64 one);
 - the captured scale: exact for "mean" (closed form) and for "max_cost" (the
   farthest point of y from any x is a vertex of y's convex hull).
No oracle input comes from the GPU.
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


def _seeded_g(w, seed, spread):
    """A potential on the columns drawn by the test (not a solution)."""
    return np.random.default_rng(seed).normal(0.0, spread, w.m).astype(np.float32).astype(np.float64)


def _single_steps(ot, orc, w, c, maxc, seed, **kw):
    """One GPU f-update from a seeded g against the oracle's f-update on sampled
    rows; then the same with the clouds exchanged (the g-update's arithmetic).
    Returns the oracle's potentials at the sampled rows and the seeded g."""
    import torch
    from dataclasses import replace
    rng = np.random.default_rng(seed)
    out = []
    for side, ws in (("f", w), ("g", replace(w, x=w.y, y=w.x, a=w.b, b=w.a))):
        g0 = _seeded_g(ws, seed + (side == "g"), 0.02 * maxc)
        x, y, a, b = H.to_dev(ws)
        p = ot.sinkhorn(x, y, a, b, eps=ws.eps, scale=ws.scale, n_iters=1,
                        f=torch.zeros(ws.n, dtype=torch.float32, device="cuda"),
                        g=torch.from_numpy(g0.astype(np.float32)).cuda(), warm_start=True, **kw)
        torch.cuda.synchronize()
        assert p.info.inv_scale_cost == pytest.approx(c, rel=1e-6)
        rows = np.sort(rng.choice(ws.n, size=min(SAMPLE, ws.n), replace=False))
        f1 = p.f.double().cpu().numpy()
        f_ref = orc.f_step(ws.x, ws.y, ws.a, g0, c, ws.eps, rows=rows)
        H.assert_potentials(f1[rows], f_ref, maxc, what=f"{side} (one step from a seeded state)")
        p.close()
        out.append((rows, f_ref, g0))
    return out[0]


def _plan_at_sampled_rows(ot, w, rows, f_rows, g0, **kw):
    """A plan whose sampled rows carry the oracle's potentials (0 elsewhere)."""
    f = np.zeros(w.n)
    f[rows] = f_rows
    return H.plan_at(ot, w, H.f32(f), H.f32(g0), **kw), H.f32(f)


def test_w2_8000_full_path(ot, orc):
    """The benchmarked workload, in the bench's launch shape: the GPU's solve to
    tol / cap (its in-loop residual against its own float64 residual), single
    steps from a seeded state, then the full oracle residual, min_row, rows and
    sparse plan of a plan at the oracle's potentials after 30 iterations."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2()
    x, y, a, b = H.to_dev(w)
    solved = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=w.n_iters, tol=w.tol)
    c = solved.info.inv_scale_cost
    xd, yd = w.x.astype(np.float64), w.y.astype(np.float64)
    mean = (xd ** 2).sum(1).mean() + (yd ** 2).sum(1).mean() - 2 * xd.mean(0) @ yd.mean(0)
    assert c == pytest.approx(1.0 / mean, rel=1e-9)
    # the in-loop residual (float32 LSE) agrees with the GPU's float64 one
    assert solved.info.residual == pytest.approx(solved.marginal_residual()[0], rel=1e-3)
    solved.close()
    maxc = H.max_cost(w.x, w.y, c)
    _single_steps(ot, orc, w, c, maxc, seed=1)
    f_o, g_o, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 30)
    f, g = H.f32(f_o), H.f32(g_o)
    plan = H.plan_at(ot, w, f, g)
    r = plan.marginal_residual()
    r_ref = orc.marginal_residual(w.x, w.y, w.a, w.b, f, g, c, w.eps)
    assert abs(r[0] - r_ref[0]) <= H.RES_TOL and abs(r[1] - r_ref[1]) <= H.RES_TOL
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
    thr_ref = ref["thr"]  # each side keeps what reaches its own min_row threshold
    Tref = orc.materialize_rows(w.x, w.y, f, g, c, w.eps, pick)
    ref_ptr = np.concatenate([[0], np.cumsum((Tref >= thr_ref).sum(1))])
    ref_cols = np.concatenate([np.nonzero(r >= thr_ref)[0] for r in Tref])
    ref_vals = np.concatenate([r[r >= thr_ref] for r in Tref])
    got_ptr = np.concatenate([[0], np.cumsum([row_ptr[i + 1] - row_ptr[i] for i in pick])])
    got_cols = np.concatenate([col_idx[row_ptr[i]:row_ptr[i + 1]] for i in pick])
    got_vals = np.concatenate([vals[row_ptr[i]:row_ptr[i + 1]] for i in pick])
    H.assert_csr((got_ptr, got_cols, got_vals), (ref_ptr, ref_cols, ref_vals), thr_ref,
                 band_tol=2 * H.ROW_TOL)
    plan.close()


def test_w3_tensor_core_full_size(ot, orc):
    """40000 x 50000, d = 50 on the tcgen05 path: the 500-iteration solve (finite),
    single steps from a seeded state, and sampled rows of a plan whose sampled
    rows carry the oracle's potentials."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w3()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=w.n_iters)
    c = plan.info.inv_scale_cost
    f, g = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    assert np.isfinite(f).all() and np.isfinite(g).all()
    plan.close()
    maxc = H.max_cost(w.x, w.y, c)
    rows, f_rows, g0 = _single_steps(ot, orc, w, c, maxc, seed=3)
    rows, f_rows = rows[:16], f_rows[:16]
    p, fs = _plan_at_sampled_rows(ot, w, rows, f_rows, g0)
    T = p.materialize_rows(torch.from_numpy(rows.astype(np.int64)).cuda()).double().cpu().numpy()
    H.assert_entries(T, orc.materialize_rows(w.x, w.y, fs, H.f32(g0), c, w.eps, rows))
    p.close()


def test_w4_million_points_step(ot, orc):
    """10^6 x 10^6 uniform vs 64 clusters at the final eps: two GPU iterations
    from zero (finite), then single steps from a seeded state (sampled rows, both
    directions)."""
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w4()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=2)
    assert np.isfinite(plan.f.cpu().numpy()).all()
    plan.close()
    maxc = _max_sqdist_hull(w.x, w.y)
    _single_steps(ot, orc, w, 1.0, maxc, seed=4)


def test_w5_two_million_points_step_and_rows(ot, orc):
    """2*10^6 spirals, scale max_cost (checked exactly), eps 1e-3: single steps from
    a seeded state, then one 4096-row block of the 65,536 rows (32.8 GB) and sampled rows."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w5()
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=2)
    mx = _max_sqdist_hull(w.x, w.y)
    c = plan.info.inv_scale_cost
    # the pass runs in float32 on shifted coordinates: ~1e-7 relative
    assert c == pytest.approx(1.0 / mx, rel=1e-6)
    plan.close()
    _single_steps(ot, orc, w, c, 1.0, seed=5)
    # one 4096-row block of the 65,536 rows; the sampled rows among them carry the
    # oracle's potentials (f-update from a seeded g), the others 0
    pick = np.arange(0, w.block_rows, 128)
    g0 = _seeded_g(w, 6, 0.02)
    f_rows = orc.f_step(w.x, w.y, w.a, g0, c, w.eps, rows=w.rows[pick])
    p, fs = _plan_at_sampled_rows(ot, w, w.rows[pick], f_rows, g0)
    rows = torch.from_numpy(w.rows[:w.block_rows]).cuda()
    out = torch.empty((w.block_rows, w.m), dtype=torch.float32, device="cuda")
    p.materialize_rows(rows, out=out)
    T = out[torch.from_numpy(pick).cuda()].double().cpu().numpy()
    del out
    H.assert_entries(T, orc.materialize_rows(w.x, w.y, fs, H.f32(g0), c, w.eps, w.rows[pick]))
    p.close()


def test_block_sparse_certificate_at_2_18(ot, orc):
    """Block-sparse fine iterations on workload 4's clouds at n = m = 2^18 (its eps
    rule), from a state annealed by block-sparse iterations: the stop test's
    admitted-plan residual and the GPU's float64 residual over every pair differ by
    at most the omitted-mass bound, the mask is far from full, and a rerun from the
    same state is bit-identical."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w4(n=262144)
    x, y, a, b = H.to_dev(w)
    tau = 5e-3
    delta = tau / (4 * 2048)
    kw = dict(eps=w.eps, scale="none", block_sparse=True, sparse_delta=delta)
    warm = ot.sinkhorn(x, y, a, b, n_iters=20, eps_init=16 * w.eps, eps_decay=0.7,
                       iters_per_stage=20, **kw)
    f0, g0 = warm.f.clone(), warm.g.clone()
    warm.close()
    runs = []
    for _ in range(2):
        p = ot.sinkhorn(x, y, a, b, n_iters=5, f=f0.clone(), g=g0.clone(), warm_start=True, **kw)
        torch.cuda.synchronize()
        runs.append((p.f.clone(), p.g.clone(), p.info.residual))
        info = p.info
        full_row, full_col = p.marginal_residual()
        assert info.sparse_iterations == 5 and info.tiles_admitted < 0.1 * info.tiles_total
        assert abs(full_row - info.residual) <= info.omitted_bound + 1e-5
        assert info.omitted_bound <= tau / 4 * (1 + 1e-6)
        p.close()
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
    assert runs[0][2] == runs[1][2]
