"""Block-sparse fine iterations on the GPU against the oracle's block-sparse solve
("FlashSinkhorn 2: Block-Sparse Entropic Optimal Transport", sections 3, 3.2,
A.3, B.3), through the C ABI (-m gpu).

Potentials are compared after the same iterations from the same start within
1e-4 of max C. The masks are compared through their tile counts: the GPU's
candidate and admitted counts of the last mask must equal the oracle's up to
the tiles whose oracle margin lies within a band of the threshold (the two
states differ by float32 rounding). The certificate is checked on the GPU
itself: after a sparse solve that met tol, the full float64 residual of the
returned potentials is <= tol.
"""
import numpy as np
import pytest

import helpers as H

pytestmark = pytest.mark.gpu

BAND = 0.1  # natural-log units around the threshold where the two masks may differ


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


def _clusters(seed, n, m, d, k=12, sigma=0.03, massless=False):
    from log_domain_sinkhorn_online_b200.workloads import Workload
    rng = np.random.default_rng(seed)
    cx = rng.random((k, d))
    x = np.clip(cx[rng.integers(0, k, n)] + sigma * rng.standard_normal((n, d)), 0, 1)
    y = np.clip(cx[rng.integers(0, k, m)] + 0.02 + sigma * rng.standard_normal((m, d)), 0, 1)
    a = rng.random(n) + 0.5
    b = rng.random(m) + 0.5
    if massless:
        a[rng.choice(n, n // 50, replace=False)] = 0.0
    a = (a / a.sum()).astype(np.float32)
    b = (b / b.sum()).astype(np.float32)
    return Workload("clusters", x.astype(np.float32), y.astype(np.float32), a, b, eps=1e-3,
                    scale="none", n_iters=10)


def _gpu(ot, w, n_iters, tol=0.0, f0=None, g0=None, **kw):
    import torch
    x, y, a, b = H.to_dev(w)
    extra = {}
    if f0 is not None:
        extra = dict(f=torch.from_numpy(f0.astype(np.float32)).cuda(),
                     g=torch.from_numpy(g0.astype(np.float32)).cuda(), warm_start=True)
    plan = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=n_iters, tol=tol,
                       block_sparse=True, **extra, **kw)
    torch.cuda.synchronize()
    return plan


def _band_counts(orc, w, f, g, B, delta, verify):
    """Oracle mask at the oracle's own final state: its counts and the number of
    tiles within BAND of the threshold (screen and verification)."""
    lo, hi = orc.joint_box(w.x, w.y)
    px, py = orc.morton_order(w.x, lo, hi), orc.morton_order(w.y, lo, hi)
    o = orc.block_mask(w.x[px], w.y[py], w.a[px].astype(np.float64), w.b[py].astype(np.float64),
                       f[px], g[py], 1.0, w.eps, B, delta, verify)
    near_s = int((np.abs(o["screen_margin"]) < BAND).sum())
    mm = o["mass_margin"]
    near_m = int((np.abs(mm[np.isfinite(mm)]) < BAND).sum())
    return o["n_cand"], o["n_adm"], near_s, near_s + near_m


def _compare(plan, orc_f, orc_g, w):
    maxc = H.max_cost(w.x, w.y, 1.0)
    fg, gg = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    ef = H.assert_potentials(fg, orc_f, maxc, what="f")
    eg = H.assert_potentials(gg, orc_g, maxc, what="g")
    return ef, eg


@pytest.mark.parametrize("d,B,verify,n,m", [
    (3, 128, True, 5000, 4100), (3, 256, True, 5000, 4100), (2, 128, False, 3000, 3333),
    (1, 128, True, 2000, 1500),
])
def test_sparse_trajectory_matches_the_oracle(ot, orc, d, B, verify, n, m):
    w = _clusters(10 + d, n, m, d)
    delta = 1e-6
    plan = _gpu(ot, w, 10, sparse_block=B, sparse_verify=verify, sparse_delta=delta,
                sparse_dense_frac=1.0)
    f, g, it, r, st = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 10, B=B, delta=delta,
                                          verify=verify, dense_frac=1.0)
    _compare(plan, f, g, w)
    info = plan.info
    assert info.iterations == 10 and info.sparse_iterations == 10 and info.dense_iterations == 0
    NB, MB = -(-n // B), -(-m // B)
    assert info.tiles_total == NB * MB
    cand, adm, near_s, near_all = _band_counts(orc, w, f, g, B, delta, verify)
    assert abs(info.tiles_candidate - cand) <= near_s, (info.tiles_candidate, cand, near_s)
    assert abs(info.tiles_admitted - adm) <= near_all, (info.tiles_admitted, adm, near_all)
    assert info.tiles_admitted < NB * MB  # the mask is not trivial here
    if verify:  # every admitted tile had its exact mass evaluated
        assert info.tiles_admitted <= info.tiles_exact <= info.tiles_candidate
    assert abs(info.residual - r) <= 1e-3 * max(r, 1e-3)
    plan.close()


def _uniform(seed, n, m, eps):
    from log_domain_sinkhorn_online_b200.workloads import Workload
    rng = np.random.default_rng(seed)
    x = rng.random((n, 3)).astype(np.float32)
    y = rng.random((m, 3)).astype(np.float32)
    return Workload("uniform", x, y, np.full(n, 1 / n, np.float32), np.full(m, 1 / m, np.float32),
                    eps=eps, scale="none", n_iters=10)


def test_sparse_stop_rule_certifies_the_full_residual(ot, orc):
    w = _uniform(21, 4000, 3900, 4e-3)  # converges in about 100 iterations
    tol = 1e-2
    plan = _gpu(ot, w, 300, tol=tol, sparse_dense_frac=1.0)
    info = plan.info
    assert info.converged == 1 and info.sparse_iterations == info.iterations
    assert 0.0 < info.omitted_bound <= tol / 4 * (1 + 1e-6)
    assert info.residual <= tol - info.omitted_bound
    full_row, _ = plan.marginal_residual()           # float64, every pair
    assert full_row <= tol
    assert abs(full_row - info.residual) <= info.omitted_bound + 1e-5
    f, g, it, r, st = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 300, tol=tol, B=128,
                                          dense_frac=1.0)
    assert abs(info.iterations - it) <= 1, (info.iterations, it)
    plan.close()


def test_full_mask_is_the_dense_solve(ot, orc):
    w = _clusters(22, 2600, 2100, 3)
    w.eps = 0.05  # every tile then holds far more than 1e-300 of mass
    plan = _gpu(ot, w, 8, sparse_delta=1e-300, sparse_dense_frac=1.0)
    assert plan.info.tiles_admitted == plan.info.tiles_total
    f, g, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, 1.0, w.eps, 8)
    _compare(plan, f, g, w)
    plan.close()


def test_candidate_fraction_policy_runs_dense_iterations(ot, orc):
    w = _clusters(23, 1500, 1700, 3)
    w.eps = 0.5                       # every tile survives the screen
    plan = _gpu(ot, w, 6, sparse_delta=1e-6, sparse_dense_frac=0.5)
    assert plan.info.dense_iterations == 6 and plan.info.sparse_iterations == 0
    f, g, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, 1.0, w.eps, 6)
    _compare(plan, f, g, w)
    plan.close()


def test_warm_start_with_massless_rows(ot, orc):
    w = _clusters(24, 3000, 2900, 3, massless=True)
    f0, g0, _, _ = orc.sinkhorn(w.x, w.y, w.a, w.b, 1.0, w.eps, 3)
    f0 = np.where(np.isneginf(f0), 0.0, f0).astype(np.float32).astype(np.float64)
    g0 = g0.astype(np.float32).astype(np.float64)
    plan = _gpu(ot, w, 6, f0=f0, g0=g0, sparse_delta=1e-6, sparse_dense_frac=1.0)
    f, g, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 6, B=128, delta=1e-6,
                                        dense_frac=1.0, f0=f0, g0=g0)
    _compare(plan, f, g, w)
    plan.close()


@pytest.mark.parametrize("n,m", [(1, 1), (50, 37), (129, 300), (300, 129)])
def test_sparse_small_and_single_block_problems(ot, orc, n, m):
    w = _clusters(25 + n, n, m, 3)
    w.eps = 0.01
    plan = _gpu(ot, w, 5, sparse_delta=1e-6, sparse_dense_frac=1.0)
    f, g, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 5, B=128, delta=1e-6,
                                        dense_frac=1.0)
    _compare(plan, f, g, w)
    plan.close()


def test_sparse_solve_is_deterministic(ot):
    w = _clusters(26, 6000, 5000, 3)
    p1 = _gpu(ot, w, 6, sparse_delta=1e-6, sparse_dense_frac=1.0)
    p2 = _gpu(ot, w, 6, sparse_delta=1e-6, sparse_dense_frac=1.0)
    assert np.array_equal(p1.f.cpu().numpy(), p2.f.cpu().numpy())
    assert np.array_equal(p1.g.cpu().numpy(), p2.g.cpu().numpy())
    assert p1.info.tiles_admitted == p2.info.tiles_admitted
    p1.close()
    p2.close()


def test_rows_after_a_sparse_solve_use_the_callers_order(ot, orc):
    # the plan keeps the caller's x, y, f, g: rows and residuals need no permutation
    w = _clusters(27, 2000, 1800, 3)
    plan = _gpu(ot, w, 5, sparse_delta=1e-6, sparse_dense_frac=1.0)
    fg, gg = plan.f.double().cpu().numpy(), plan.g.double().cpu().numpy()
    import torch
    rows = torch.tensor([0, 7, 1999], dtype=torch.int64, device="cuda")
    T = plan.materialize_rows(rows).double().cpu().numpy()
    f, g, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 5, B=128, delta=1e-6,
                                        dense_frac=1.0)
    T_ref = orc.materialize_rows(w.x, w.y, f, g, 1.0, w.eps, [0, 7, 1999])
    # entries agree to the potentials' tolerance: |dT/T| <= (|df| + |dg|) / eps
    rel = np.abs(T - T_ref) / np.maximum(T_ref, 1e-300)
    big = T_ref > 1e-20
    assert np.all(rel[big] <= 2 * H.POT_TOL * H.max_cost(w.x, w.y, 1.0) / w.eps * 1.01)
    plan.close()


def test_blocks_without_admitted_tiles_fall_back_to_every_column(ot, orc):
    """Warm start in which the columns of one cluster carry no mass (g = -50):
    the row blocks near that cluster keep no tile (their screen or verification
    rejects everything), so their f-update runs over every column, while the other
    row blocks stay sparse -- against the oracle's block-sparse solve."""
    from log_domain_sinkhorn_online_b200.workloads import Workload
    rng = np.random.default_rng(31)
    n, m = 3000, 2600
    x = rng.random((n, 3)).astype(np.float32)
    y = np.concatenate([rng.random((m // 2, 3)) * 0.2, 0.8 + rng.random((m - m // 2, 3)) * 0.2])
    y = y.astype(np.float32)
    w = Workload("two_clusters", x, y, np.full(n, 1 / n, np.float32), np.full(m, 1 / m, np.float32),
                 eps=1e-3, scale="none", n_iters=2)
    f0 = np.zeros(n)
    g0 = np.where(np.arange(m) < m // 2, 0.0, -50.0)
    lo, hi = orc.joint_box(w.x, w.y)
    px, py = orc.morton_order(w.x, lo, hi), orc.morton_order(w.y, lo, hi)
    o = orc.block_mask(w.x[px], w.y[py], w.a[px].astype(np.float64), w.b[py].astype(np.float64),
                       f0[px], g0[py], 1.0, w.eps, 128, 1e-6)
    empty = ~o["adm"].any(1)
    assert empty.any() and not empty.all()  # the case the test is about
    plan = _gpu(ot, w, 2, f0=f0, g0=g0, sparse_delta=1e-6, sparse_dense_frac=1.0)
    f, g, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 2, B=128, delta=1e-6,
                                        dense_frac=1.0, f0=f0, g0=g0)
    _compare(plan, f, g, w)
    plan.close()


def test_annealed_block_sparse_solve_matches_the_oracle(ot, orc):
    """eps-annealing with block-sparse iterations in every stage, against the
    oracle's block-sparse solve run stage by stage with the same schedule."""
    w = _clusters(41, 2500, 2300, 3)
    eps_t, eps0, decay, per_stage = 1e-3, 8e-3, 0.5, 4
    plan = _gpu(ot, w, 5, eps_init=eps0, eps_decay=decay, iters_per_stage=per_stage,
                sparse_delta=1e-6, sparse_dense_frac=1.0)
    f = np.zeros(w.n)
    g = np.zeros(w.m)
    k, stages = 0, 0
    while True:
        ek = max(eps_t, eps0 * decay ** k)
        its = 5 if ek == eps_t else per_stage
        f, g, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, ek, its, B=128, delta=1e-6,
                                            dense_frac=1.0, f0=f, g0=g)
        stages += 1
        if ek == eps_t:
            break
        k += 1
    assert plan.info.stages == stages == 4
    _compare(plan, f, g, w)
    plan.close()


@pytest.mark.parametrize("scale,B,verify", [("mean", 128, True), ("max_cost", 256, False)])
def test_scaled_costs_and_massless_columns(ot, orc, scale, B, verify):
    """Block-sparse iterations on a scaled cost with massless rows and columns and
    m much larger than n, against the oracle's block-sparse solve at the same c."""
    w = _clusters(51, 1200, 4100, 3, massless=True)
    w.b = w.b.copy()
    w.b[[0, 77, 4099]] = 0.0
    w.scale, w.eps = scale, 2e-3
    c = orc.inv_scale_cost(w.x, w.y, scale)
    plan = _gpu(ot, w, 6, sparse_block=B, sparse_verify=verify, sparse_delta=1e-6,
                sparse_dense_frac=1.0)
    assert plan.info.inv_scale_cost == pytest.approx(c, rel=2e-7)
    f, g, _, _, st = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, c, w.eps, 6, B=B, delta=1e-6,
                                         verify=verify, dense_frac=1.0)
    maxc = H.max_cost(w.x, w.y, c)
    H.assert_potentials(plan.f.double().cpu().numpy(), f, maxc, what="f")
    H.assert_potentials(plan.g.double().cpu().numpy(), g, maxc, what="g")
    assert plan.info.sparse_iterations == 6 and 0 < st[3] < plan.info.tiles_total
    plan.close()


@pytest.mark.parametrize("d,B,verify,n,m", [
    (3, 128, True, 5000, 4100), (3, 256, True, 5000, 4100), (2, 128, True, 3000, 3333),
    (1, 128, True, 2000, 1500), (3, 128, False, 4000, 3000),
])
def test_first_mask_matches_the_oracle_tile_by_tile(ot, orc, d, B, verify, n, m):
    """The block mask built at given potentials (the oracle's after 6 block-sparse
    iterations, rounded to float32) against the oracle's mask at the same
    potentials, tile by tile: every tile whose oracle margin lies outside BAND of
    the threshold (the screen's, and the exact mass's where it was evaluated)
    takes the same decision ("FlashSinkhorn 2", sections 3.2 and A.3)."""
    import torch
    w = _clusters(20 + d, n, m, d)
    delta = 1e-6
    f6, g6, _, _, _ = orc.sinkhorn_sparse(w.x, w.y, w.a, w.b, 1.0, w.eps, 6, B=B, delta=delta,
                                          verify=verify, dense_frac=1.0)
    f0, g0 = H.f32(f6), H.f32(g6)
    NB, MB = -(-n // B), -(-m // B)
    mask = torch.full((NB * MB,), 7, dtype=torch.uint8, device="cuda")
    plan = _gpu(ot, w, 1, f0=f0, g0=g0, sparse_block=B, sparse_verify=verify, sparse_delta=delta,
                sparse_dense_frac=1.0, sparse_mask_out=mask)
    plan.close()
    got = mask.cpu().numpy().reshape(NB, MB)
    assert set(np.unique(got)) <= {0, 1}
    lo, hi = orc.joint_box(w.x, w.y)
    px, py = orc.morton_order(w.x, lo, hi), orc.morton_order(w.y, lo, hi)
    o = orc.block_mask(w.x[px], w.y[py], w.a[px].astype(np.float64), w.b[py].astype(np.float64),
                       f0[px], g0[py], 1.0, w.eps, B, delta, verify)
    ref = o["adm"] if verify else o["cand"]
    sm, mm = o["screen_margin"], o["mass_margin"]
    clear = np.abs(sm) > BAND
    if verify:
        clear &= ~np.isfinite(mm) | (np.abs(mm) > BAND)
    assert clear.mean() > 0.9, clear.mean()
    bad = np.argwhere(clear & (got.astype(bool) != ref))
    assert bad.size == 0, (bad[:5], int(got.sum()), int(ref.sum()))
    assert 0 < int(ref.sum()) < NB * MB  # neither empty nor full
