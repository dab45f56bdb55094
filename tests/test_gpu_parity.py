"""GPU parity against the float64 oracle on the same seeded inputs (-m gpu).

Every call goes through the C ABI (via the ctypes binding). Sizes are chosen
so the oracle finishes in seconds yet the kernels see several row tiles
(1024 rows), several column splits and ragged tails.
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


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def _solve_both(ot, orc, w, n_iters, tol=0.0, **kw):
    import torch
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=n_iters, tol=tol, **kw)
    torch.cuda.synchronize()
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    assert abs(plan.info.inv_scale_cost - c) <= 2e-7 * c
    f_ref, g_ref, it_ref, r_ref = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, n_iters, tol)
    return plan, c, f_ref, g_ref, it_ref, r_ref


def _pots(plan):
    return plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()


def _cloud(seed, n, m, d, scale="none", eps=0.05):
    from log_domain_sinkhorn_online_b200.workloads import Workload
    rng = np.random.default_rng(seed)
    x = rng.random((n, d)).astype(np.float32)
    y = (rng.random((m, d)) * 0.8 + 0.15).astype(np.float32)
    a = (rng.random(n) + 0.5)
    b = (rng.random(m) + 0.5)
    return Workload("cloud", x, y, (a / a.sum()).astype(np.float32), (b / b.sum()).astype(np.float32),
                    eps=eps, scale=scale, n_iters=30)


# --------------------------------------------------------------- trajectories
@pytest.mark.parametrize("d", [1, 2, 3])
@pytest.mark.parametrize("scale", ["none", "mean", "max_cost"])
def test_lowd_trajectory_ragged(ot, orc, d, scale):
    w = _cloud(10 + d, 2085, 1379, d, scale=scale, eps=0.02)
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 25)
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")
    assert plan.info.iterations == 25


@pytest.mark.parametrize("d,tc", [(4, False), (5, False), (15, False), (16, False), (16, True),
                                  (17, True), (33, True), (50, False), (50, True), (64, True)])
def test_generic_d_trajectory(ot, orc, d, tc):
    """3 < d <= 64: CUDA-core FMA kernel, or for d >= 16 the tcgen05 tensor-core
    kernel (bf16 splits, fp32 accumulation); ragged sizes over several tiles."""
    w = _cloud(30 + d, 611, 530, d, scale="mean", eps=0.05)
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 15, tensor_cores=tc)
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


def test_w1_full_workload(ot, orc):
    """512 x 512 uniform in 2-D, eps 0.05, exactly 200 iterations, all rows, min_row."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w1()
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, w.n_iters)
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")
    plan.close()
    # rows, min_row and residual at the oracle's potentials (given to both sides)
    f, g = H.f32(f_ref), H.f32(g_ref)
    plan = H.plan_at(ot, w, f, g)
    T = plan.materialize_rows(torch.arange(w.n, device="cuda")).double().cpu().numpy()
    T_ref = orc.dense_plan(w.x, w.y, f, g, c, w.eps)
    H.assert_entries(T, T_ref)
    mr = plan.sparsify_min_row()
    ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)
    H.assert_min_row(mr, ref)
    kept = T >= mr["thr"]
    kept_ref = T_ref >= ref["thr"]
    band = np.abs(T_ref - ref["thr"]) <= 1e-5 * ref["thr"]
    assert np.array_equal(kept[~band], kept_ref[~band])
    assert (kept.sum(1) >= 1).all()
    assert mr["nnz"] == int(kept.sum())
    r = plan.marginal_residual()
    r_ref = orc.marginal_residual(w.x, w.y, w.a, w.b, f, g, c, w.eps)
    assert abs(r[0] - r_ref[0]) <= H.RES_TOL and abs(r[1] - r_ref[1]) <= H.RES_TOL


def test_tol_stopping_counts(ot, orc):
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=1500, m=1400)
    plan, c, f_ref, g_ref, it_ref, r_ref = _solve_both(ot, orc, w, 2000, tol=w.tol)
    maxc = H.max_cost(w.x, w.y, c)
    assert plan.info.converged == 1 and it_ref < 2000
    if plan.info.iterations != it_ref:
        # the residual crossed tol within rounding: rerun both with the oracle's count
        assert abs(plan.info.iterations - it_ref) <= 2
        plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, it_ref)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")
    assert abs(plan.info.residual - r_ref) <= 1e-3 * max(r_ref, w.tol)


def test_massless_rows_and_columns(ot, orc):
    w = _cloud(5, 1500, 1100, 3, eps=0.03)
    w.a[[0, 7, 1024, 1499]] = 0.0
    w.b[[3, 1099]] = 0.0
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 20)
    assert plan.status == 1 and plan.info.n_massless_rows == 4 and plan.info.n_massless_cols == 2
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")
    plan.close()
    f, g = H.f32(f_ref), H.f32(g_ref)
    plan = H.plan_at(ot, w, f, g)
    mr = plan.sparsify_min_row(block_rows=333)
    ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)
    H.assert_min_row(mr, ref)
    counts = mr["counts"].cpu().numpy()
    assert (counts[[0, 7, 1024, 1499]] == 0).all() and (np.delete(counts, [0, 7, 1024, 1499]) >= 1).all()


@pytest.mark.parametrize("n,m", [(1, 1), (1, 37), (37, 1), (8, 8), (9, 1031), (1031, 9)])
def test_tiny_and_degenerate_sizes(ot, orc, n, m):
    w = _cloud(n * 7 + m, n, m, 3, eps=0.1)
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 10)
    maxc = max(H.max_cost(w.x, w.y, c), 1e-6)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


def test_no_graphs_same_result(ot, orc):
    import torch
    w = _cloud(77, 1200, 900, 3, eps=0.02)
    x, y, a, b = H.to_dev(w)
    p1 = ot.sinkhorn(x, y, a, b, eps=w.eps, n_iters=37, use_graphs=True, check_every=8)
    p2 = ot.sinkhorn(x, y, a, b, eps=w.eps, n_iters=37, use_graphs=False)
    torch.cuda.synchronize()
    assert torch.equal(p1.f, p2.f) and torch.equal(p1.g, p2.g)  # deterministic kernels


def test_rows_and_residual_at_given_potentials(ot, orc):
    """Rows, residuals and min_row (several block sizes) of a plan at the
    oracle's potentials after 60 iterations, against the oracle there."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=3001, m=2777)
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    f_ref, g_ref, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 60)
    f, g = H.f32(f_ref), H.f32(g_ref)
    plan = H.plan_at(ot, w, f, g)
    assert plan.info.inv_scale_cost == pytest.approx(c, rel=2e-7)
    rows = np.array([0, 1, 1023, 1024, 2047, 3000, 5, 5], dtype=np.int64)
    T = plan.materialize_rows(torch.from_numpy(rows).cuda()).double().cpu().numpy()
    H.assert_entries(T, orc.materialize_rows(w.x, w.y, f, g, c, w.eps, rows))
    r = plan.marginal_residual()
    r_ref = orc.marginal_residual(w.x, w.y, w.a, w.b, f, g, c, w.eps)
    assert abs(r[0] - r_ref[0]) <= H.RES_TOL and abs(r[1] - r_ref[1]) <= H.RES_TOL
    ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)
    outs = [plan.sparsify_min_row(block_rows=br) for br in (1, 64, 1024, 0)]
    for o in outs:
        H.assert_min_row(o, ref)
        assert o["thr"] == outs[0]["thr"] and o["nnz"] == outs[0]["nnz"]
        assert torch.equal(o["counts"], outs[0]["counts"])


def _csr_case(ot, orc):
    """A plan at the oracle's potentials (40 iterations), with massless rows."""
    w = _cloud(33, 517, 389, 2, scale="mean", eps=0.02)
    w.a = w.a.copy()
    w.a[[5, 100, 516]] = 0.0  # rows without mass keep nothing
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    f_ref, g_ref, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 40)
    f, g = H.f32(f_ref), H.f32(g_ref)
    return w, H.plan_at(ot, w, f, g), f, g, c


def test_sparsify_csr_matches_oracle(ot, orc):
    """Compressed-row sparsify against the oracle's thresholded plan, both at the
    oracle's potentials and each at its own min_row threshold: the same kept
    entries outside the tie band, values as plan entries, increasing columns;
    counts and nnz are min_row's."""
    w, plan, f, g, c = _csr_case(ot, orc)
    mr = plan.sparsify_min_row()
    csr = plan.sparsify_csr()
    assert csr["thr"] == mr["thr"] and csr["nnz"] == mr["nnz"]
    row_ptr = csr["row_ptr"].cpu().numpy()
    np.testing.assert_array_equal(np.diff(row_ptr), mr["counts"].cpu().numpy())
    assert all(row_ptr[i + 1] == row_ptr[i] for i in (5, 100, 516))
    thr_ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)["thr"]
    assert abs(csr["thr"] - thr_ref) <= H.ROW_TOL * thr_ref
    ref = orc.sparsify_csr(w.x, w.y, w.a, f, g, c, w.eps, thr_ref)
    # each side thresholds at its own thr (within 1e-5 of the other): band 2e-5
    band = H.assert_csr((row_ptr, csr["col_idx"].cpu().numpy(), csr["vals"].cpu().numpy()), ref,
                        thr_ref, band_tol=2 * H.ROW_TOL)
    assert band <= max(2, csr["nnz"] // 1000)
    plan.close()


def test_sparsify_csr_block_rows_and_threshold(ot, orc):
    """block_rows never changes the output (bit for bit); a lower threshold keeps
    a superset; a capacity below nnz is an overflow that reports nnz."""
    import torch
    w, plan, _, _, _ = _csr_case(ot, orc)
    outs = [plan.sparsify_csr(block_rows=br) for br in (0, 1, 7, 64)]
    for o in outs[1:]:
        for k in ("row_ptr", "col_idx", "vals"):
            assert torch.equal(o[k], outs[0][k])
    lo = plan.sparsify_csr(thr=outs[0]["thr"] * 0.5)
    assert lo["nnz"] >= outs[0]["nnz"]
    assert plan.sparsify_csr(thr=float("inf"))["nnz"] == 0
    from log_domain_sinkhorn_online_b200 import _binding as B
    with pytest.raises(B.OTError) as e:
        plan.sparsify_csr(thr=outs[0]["thr"], capacity=outs[0]["nnz"] - 1)
    assert e.value.status == B.OT_ERR_OVERFLOW
    plan.close()


@pytest.mark.parametrize("d,loop", [(3, 0), (8, 0), (24, 0)])
def test_dynamic_work_items_are_deterministic(ot, d, loop):
    """The per-launch kernels claim work items at run time; which block runs an
    item must not change a result: two solves agree bit for bit."""
    import torch
    w = _cloud(57, 3001, 2777, d, scale="mean", eps=0.03)
    x, y, a, b = H.to_dev(w)
    outs = []
    for _ in range(2):
        plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=15, device_loop=loop)
        outs.append((plan.f.clone(), plan.g.clone()))
        plan.close()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_sparsify_csr_generic_d(ot, orc):
    """The compressed-row sparsify on the generic-d entry path (d = 5)."""
    w = _cloud(61, 301, 257, 5, scale="max_cost", eps=0.03)
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    f_ref, g_ref, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 25)
    f, g = H.f32(f_ref), H.f32(g_ref)
    plan = H.plan_at(ot, w, f, g)
    csr = plan.sparsify_csr(block_rows=64)
    mr = plan.sparsify_min_row()
    assert csr["nnz"] == mr["nnz"]
    thr_ref = orc.min_row(w.x, w.y, w.a, f, g, c, w.eps)["thr"]
    assert abs(csr["thr"] - thr_ref) <= H.ROW_TOL * thr_ref
    ref = orc.sparsify_csr(w.x, w.y, w.a, f, g, c, w.eps, thr_ref)
    band = H.assert_csr((csr["row_ptr"].cpu().numpy(), csr["col_idx"].cpu().numpy(),
                         csr["vals"].cpu().numpy()), ref, thr_ref, band_tol=2 * H.ROW_TOL)
    assert band <= max(2, csr["nnz"] // 1000)
    plan.close()


@pytest.mark.parametrize("r", [1, 7, 32, 128])
def test_lowrank_coupling_rows_match_oracle(ot, orc, r):
    """(Q diag(1/g) R^T)[rows] against the oracle: nonnegative factors, a ragged
    column count, unsorted and repeated rows, rows past one launch tile."""
    import torch
    rng = np.random.default_rng(70 + r)
    n, m = 203, 1031
    Q = rng.random((n, r)).astype(np.float32)
    R = rng.random((m, r)).astype(np.float32)
    g = (rng.random(r) + 0.2).astype(np.float32)
    rows = np.concatenate([rng.integers(0, n, 90), [0, n - 1, 5, 5]]).astype(np.int64)
    got = ot.lowrank_rows(*(torch.from_numpy(v).cuda() for v in (Q, R, g, rows))).double().cpu().numpy()
    H.assert_entries(got, orc.lr_rows(Q, R, g, rows))


@pytest.mark.parametrize("r", [2, 16, 128])
def test_lowrank_cost_rows_match_oracle(ot, orc, r):
    """Entropic rows on a low-rank cost (signed factors, a bias, a massless row)
    against the oracle, float64 exponent like the point-cloud rows."""
    import torch
    rng = np.random.default_rng(90 + r)
    n, m = 150, 517
    c1 = (rng.standard_normal((n, r)) / np.sqrt(r)).astype(np.float32)
    c2 = (rng.standard_normal((m, r)) / np.sqrt(r)).astype(np.float32)
    f = rng.normal(0, 0.05, n).astype(np.float32)
    g = rng.normal(0, 0.05, m).astype(np.float32)
    f[7] = -np.inf
    rows = rng.integers(0, n, 70).astype(np.int64)
    rows[3] = 7
    eps, c, bias = 0.05, 0.8, 0.3
    dev = [torch.from_numpy(v).cuda() for v in (c1, c2, f, g, rows)]
    got = ot.lrcost_rows(*dev[:4], dev[4], eps=eps, inv_scale_cost=c, bias=bias).double().cpu().numpy()
    ref = orc.lrc_rows(c1, c2, f, g, bias, c, eps, rows)
    assert np.all(got[3] == 0.0)
    H.assert_entries(got, ref)


def test_lowrank_cost_rows_reproduce_point_cloud_rows(ot):
    """Squared Euclidean as a low-rank cost, [|x|^2, 1, -2x] . [1, |y|^2, y]: the
    low-rank-cost rows at a solved plan's potentials are that plan's rows."""
    import torch
    w = _cloud(71, 600, 450, 3, scale="mean", eps=0.05)
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=30)
    xd, yd = w.x.astype(np.float64), w.y.astype(np.float64)
    c1 = np.concatenate([(xd ** 2).sum(1, keepdims=True), np.ones((600, 1)), -2 * xd], 1).astype(np.float32)
    c2 = np.concatenate([np.ones((450, 1)), (yd ** 2).sum(1, keepdims=True), yd], 1).astype(np.float32)
    rows = torch.arange(0, 600, 7, device="cuda")
    want = plan.materialize_rows(rows).double().cpu().numpy()
    got = ot.lrcost_rows(torch.from_numpy(c1).cuda(), torch.from_numpy(c2).cuda(), plan.f, plan.g, rows,
                         eps=w.eps, inv_scale_cost=plan.info.inv_scale_cost).double().cpu().numpy()
    # the factors round |x|^2 and |y|^2 to float32: ~1e-7 of the cost, scaled by c / eps
    H.assert_entries(got, want, tol=2e-5)
    plan.close()


def test_lowrank_rows_report_bad_rows_and_rank(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    Q = torch.rand(10, 4, device="cuda")
    R = torch.rand(12, 4, device="cuda")
    g = torch.rand(4, device="cuda") + 0.5
    with pytest.raises(B.OTError) as e:
        ot.lowrank_rows(Q, R, g, torch.tensor([0, 10], device="cuda"))
    assert e.value.status == B.OT_ERR_INVALID_ARG
    big = torch.rand(10, 129, device="cuda")
    with pytest.raises(B.OTError) as e:
        ot.lowrank_rows(big, torch.rand(12, 129, device="cuda"), torch.rand(129, device="cuda") + 0.5,
                        torch.tensor([0], device="cuda"))
    assert e.value.status == B.OT_ERR_UNSUPPORTED


def test_bad_row_index_is_reported(ot):
    import torch
    w = _cloud(3, 300, 200, 2)
    x, y, a, b = H.to_dev(w)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, n_iters=3)
    with pytest.raises(ot.OTError) as e:
        plan.materialize_rows(torch.tensor([0, 300], device="cuda"))
    assert e.value.status == -1
    out = plan.materialize_rows(torch.tensor([299, 0], device="cuda"))
    assert torch.isfinite(out).all()


def test_nonfinite_input_is_reported(ot):
    w = _cloud(4, 100, 90, 3)
    w.x[5, 1] = np.nan
    x, y, a, b = H.to_dev(w)
    with pytest.raises(ot.OTError) as e:
        ot.sinkhorn(x, y, a, b, eps=w.eps, n_iters=3)
    assert e.value.status == -5


def test_annealing_matches_oracle(ot, orc):
    from log_domain_sinkhorn_online_b200 import workloads
    import torch
    w = workloads.w4(n=2000)
    x, y, a, b = H.to_dev(w)
    eps_t = 0.002
    plan = ot.sinkhorn(x, y, a, b, eps=eps_t, n_iters=10, eps_init=1.0, eps_decay=0.7,
                       iters_per_stage=10)
    torch.cuda.synchronize()
    f_ref, g_ref, stages, r_ref = orc.sinkhorn_anneal(w.x, w.y, w.a, w.b, 1.0, eps_t, 1.0, 0.7, 10)
    assert plan.info.stages == stages
    maxc = H.max_cost(w.x, w.y, 1.0)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


@pytest.mark.parametrize("n,m", [(1, 300), (129, 127), (2000, 3001)])
def test_tensor_core_path_ragged_and_massless(ot, orc, n, m):
    """tcgen05 path on sizes that are not multiples of the 128-row tile, with a
    massless row and column, against the oracle's trajectory."""
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w3(n=n, m=m)
    if n > 1:
        w.a[n // 2] = 0.0
    w.b[m // 3] = 0.0
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 12)
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


@pytest.mark.parametrize("loop", [0, 1])
@pytest.mark.parametrize("d", [1, 3])
def test_device_loop_and_launch_paths(ot, orc, loop, d):
    """The same solve through per-half-step launches (loop=0) and through the
    device-resident cooperative loop (loop=1): both against the oracle, with
    the tol stop inside the loop (the count is checked like the launch path's)."""
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w2(n=1777, m=1501)
    if d == 1:
        w.x, w.y = w.x[:, :1].copy(), w.y[:, :1].copy()
    plan, c, f_ref, g_ref, it_ref, r_ref = _solve_both(ot, orc, w, 300, tol=2e-3, device_loop=loop)
    maxc = H.max_cost(w.x, w.y, c)
    if plan.info.iterations != it_ref:
        assert abs(plan.info.iterations - it_ref) <= 2
        plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, it_ref, device_loop=loop)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


@pytest.mark.parametrize("loop,rpt", [(1, 1), (1, 2), (0, 1), (0, 2), (0, 4), (0, 8)])
def test_rows_per_thread_shapes(ot, orc, loop, rpt):
    """Every row layout of the d <= 3 kernels (tiles of 128 rpt rows) in both the
    device-resident loop and the per-launch path, on a ragged problem (neither
    side a multiple of a tile), against the oracle's trajectory."""
    w = _cloud(17, 1313, 1207, 3, scale="mean", eps=0.02)
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 40, device_loop=loop, rows_per_thread=rpt)
    assert plan.info.kernel_launches < 40 if loop else plan.info.kernel_launches >= 80
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


def test_device_loop_long_run_crosses_chunks(ot, orc):
    """600 iterations: three cooperative launches of the loop kernel."""
    w = _cloud(91, 900, 1100, 2, eps=0.03)
    plan, c, f_ref, g_ref, _, _ = _solve_both(ot, orc, w, 600, device_loop=1)
    assert plan.info.iterations == 600
    maxc = H.max_cost(w.x, w.y, c)
    f, g = _pots(plan)
    H.assert_potentials(f, f_ref, maxc, what="f")
    H.assert_potentials(g, g_ref, maxc, what="g")


def test_resource_cache_reuse_and_trim(ot):
    """Plans reuse cached workspaces (stale contents must not matter) and the
    cache can be emptied; every solve gives the same bits."""
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    w = _cloud(55, 3000, 2500, 3, eps=0.02)
    x, y, a, b = H.to_dev(w)
    outs = []
    for k in range(4):
        if k == 2:
            B.ot_trim_cache()
        p = ot.sinkhorn(x, y, a, b, eps=w.eps, n_iters=30)
        outs.append((p.f.clone(), p.g.clone()))
        p.close()
        # a different problem in between leaves other data in the cached buffers
        q = ot.sinkhorn(y, x, b, a, eps=0.05, n_iters=3)
        q.close()
    for f, g in outs[1:]:
        assert torch.equal(f, outs[0][0]) and torch.equal(g, outs[0][1])
