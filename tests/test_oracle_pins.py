"""Pins for the float64 oracle against what the mathematics and the pages fix.

None of these re-types the oracle's formulas: each checks a property that a
dropped term, a wrong sign, a transposed index or a wrong scale would break
(marginal identities, closed forms, brute-force exact OT, limits, invariances,
the min_row contract of moscot PR #846 "Behavioural changes").
"""
import itertools
import math

import numpy as np
import pytest


def _cloud(seed, n, m, d, lo=0.0, hi=1.0):
    rng = np.random.default_rng(seed)
    x = rng.uniform(lo, hi, (n, d)).astype(np.float32)
    y = rng.uniform(lo, hi, (m, d)).astype(np.float32)
    return x, y


def _sqd(x, y):
    # squared distances by broadcasting (float64), used only to build reference
    # quantities such as exact-OT costs
    xd, yd = np.asarray(x, np.float64), np.asarray(y, np.float64)
    return ((xd[:, None, :] - yd[None, :, :]) ** 2).sum(-1)


# ---------------------------------------------------------------- half-steps
def test_f_step_makes_row_marginals_exact(orc):
    x, y = _cloud(1, 37, 29, 3)
    rng = np.random.default_rng(5)
    a = rng.random(37) + 0.1
    a /= a.sum()
    g = rng.normal(0, 0.3, 29)
    eps, c = 0.07, 1.3
    f = orc.f_step(x, y, a, g, c, eps)
    T = orc.dense_plan(x, y, f, g, c, eps)
    np.testing.assert_allclose(T.sum(1), a, rtol=1e-13, atol=0)


def test_g_step_makes_col_marginals_exact(orc):
    x, y = _cloud(2, 31, 41, 2)
    rng = np.random.default_rng(6)
    b = rng.random(41) + 0.1
    b /= b.sum()
    f = rng.normal(0, 0.3, 31)
    eps, c = 0.05, 0.8
    g = orc.g_step(x, y, b, f, c, eps)
    T = orc.dense_plan(x, y, f, g, c, eps)
    np.testing.assert_allclose(T.sum(0), b, rtol=1e-13, atol=0)


def test_sampled_rows_match_full_step(orc):
    x, y = _cloud(3, 50, 40, 3)
    a = np.full(50, 1 / 50)
    g = np.random.default_rng(1).normal(0, 0.1, 40)
    full = orc.f_step(x, y, a, g, 1.0, 0.1)
    rows = np.array([0, 7, 49, 3], dtype=np.int64)
    np.testing.assert_array_equal(orc.f_step(x, y, a, g, 1.0, 0.1, rows=rows), full[rows])


# ------------------------------------------------------------- closed forms
@pytest.mark.parametrize("eps", [1.0, 0.3, 0.1, 0.03])
def test_two_point_symmetric_closed_form(orc, eps):
    # x = y = {0, 1}, uniform weights: converged plan has T11 = 1/(2(1+e^{-1/eps}))
    x = np.array([[0.0], [1.0]], np.float32)
    a = np.array([0.5, 0.5])
    f, g, it, r = orc.sinkhorn(x, x, a, a, 1.0, eps, 5000, tol=1e-15)
    T = orc.dense_plan(x, x, f, g, 1.0, eps)
    p = 1.0 / (2.0 * (1.0 + math.exp(-1.0 / eps)))
    np.testing.assert_allclose(T, [[p, 0.5 - p], [0.5 - p, p]], rtol=1e-10, atol=1e-14)


def test_cross_ratio_of_any_plan(orc):
    # For T = exp((f+g-C)/eps), T11 T22 / (T12 T21) = exp((C12+C21-C11-C22)/eps)
    # whatever f, g are: pins the sign, the eps scaling and the index order of C.
    x, y = _cloud(11, 2, 2, 3)
    rng = np.random.default_rng(3)
    f, g = rng.normal(0, 0.2, 2), rng.normal(0, 0.2, 2)
    c, eps = 1.7, 0.2
    T = orc.dense_plan(x, y, f, g, c, eps)
    C = c * _sqd(x, y)
    lhs = T[0, 0] * T[1, 1] / (T[0, 1] * T[1, 0])
    assert lhs == pytest.approx(math.exp((C[0, 1] + C[1, 0] - C[0, 0] - C[1, 1]) / eps),
                                rel=1e-12)


def test_two_by_two_weighted_closed_form(orc):
    # converged 2x2 plan with marginals a, b is fixed by the cross ratio K:
    # p (1 - a1 - b1 + p) = K (a1 - p)(b1 - p), p = T11 in (max(0,a1+b1-1), min(a1,b1))
    x, y = _cloud(12, 2, 2, 2)
    a = np.array([0.3, 0.7])
    b = np.array([0.6, 0.4])
    c, eps = 1.0, 0.15
    f, g, it, r = orc.sinkhorn(x, y, a, b, c, eps, 20000, tol=1e-15)
    C = c * _sqd(x, y)
    K = math.exp((C[0, 1] + C[1, 0] - C[0, 0] - C[1, 1]) / eps)
    a1, b1 = a[0], b[0]
    # (1-K) p^2 + (1 - a1 - b1 + K(a1 + b1)) p - K a1 b1 = 0
    A, B, Cq = 1.0 - K, 1.0 - a1 - b1 + K * (a1 + b1), -K * a1 * b1
    roots = np.roots([A, B, Cq]) if abs(A) > 1e-15 else np.array([-Cq / B])
    lo, hi = max(0.0, a1 + b1 - 1.0), min(a1, b1)
    p = [float(np.real(z)) for z in roots if lo - 1e-12 <= np.real(z) <= hi + 1e-12][0]
    T = orc.dense_plan(x, y, f, g, c, eps)
    np.testing.assert_allclose(T, [[p, a1 - p], [b1 - p, 1 - a1 - b1 + p]], rtol=1e-9,
                               atol=1e-13)


def test_trivial_sizes(orc):
    # m = 1: after one f-step T_i1 = a_i; n = m = 1: T = a then b.
    x, y = _cloud(4, 9, 1, 2)
    a = np.random.default_rng(2).random(9)
    f = orc.f_step(x, y, a, np.array([0.37]), 1.0, 0.05)
    T = orc.dense_plan(x, y, f, [0.37], 1.0, 0.05)
    np.testing.assert_allclose(T[:, 0], a, rtol=1e-13)
    x1, y1 = _cloud(5, 1, 1, 3)
    f = orc.f_step(x1, y1, [0.4], [0.0], 1.0, 0.01)
    assert orc.dense_plan(x1, y1, f, [0.0], 1.0, 0.01)[0, 0] == pytest.approx(0.4, rel=1e-13)
    g = orc.g_step(x1, y1, [0.9], f, 1.0, 0.01)
    assert orc.dense_plan(x1, y1, f, g, 1.0, 0.01)[0, 0] == pytest.approx(0.9, rel=1e-13)


# ------------------------------------------------------------ exact OT limits
def test_brute_force_exact_ot_as_eps_to_zero(orc):
    # uniform weights, n = m: exact OT is attained at a permutation (Birkhoff);
    # entropic cost satisfies 0 <= <C,T_eps> - OT <= eps * ln(n) at convergence.
    n = 6
    x, y = _cloud(21, n, n, 2)
    C = _sqd(x, y)
    ot = min(sum(C[i, s[i]] for i in range(n)) for s in itertools.permutations(range(n))) / n
    a = np.full(n, 1.0 / n)
    gaps = []
    for eps in [0.05, 0.01, 0.002]:
        f, g, it, r = orc.sinkhorn(x, y, a, a, 1.0, eps, 200000, tol=1e-13)
        assert r <= 1e-13
        T = orc.dense_plan(x, y, f, g, 1.0, eps)
        gap = float((C * T).sum() - ot)
        assert -1e-12 <= gap <= eps * math.log(n) + 1e-12
        gaps.append(gap)
    assert gaps[-1] < gaps[0]


def test_one_d_sorted_matching(orc):
    # d = 1: the optimal coupling of equal-size uniform measures is the sorted matching
    n = 100
    rng = np.random.default_rng(7)
    x = rng.random((n, 1)).astype(np.float32)
    y = (rng.random((n, 1)) ** 2).astype(np.float32)
    ot = float(np.mean((np.sort(x[:, 0].astype(np.float64)) - np.sort(y[:, 0].astype(np.float64))) ** 2))
    a = np.full(n, 1.0 / n)
    eps = 1e-4
    f, g, it, r = orc.sinkhorn(x, y, a, a, 1.0, eps, 20000, tol=1e-9)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    gap = float((_sqd(x, y) * T).sum() - ot)
    assert -1e-8 <= gap <= eps * math.log(n) + 1e-8


def test_assignment_library_routine(orc):
    from scipy.optimize import linear_sum_assignment
    n = 40
    x, y = _cloud(8, n, n, 2)
    C = _sqd(x, y)
    r_, c_ = linear_sum_assignment(C)
    ot = C[r_, c_].sum() / n
    a = np.full(n, 1.0 / n)
    eps = 2e-4
    f, g, it, r = orc.sinkhorn(x, y, a, a, 1.0, eps, 50000, tol=1e-9)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    gap = float((C * T).sum() - ot)
    assert -1e-8 <= gap <= eps * math.log(n) + 1e-8


def test_identical_point_sets_give_identity(orc):
    h = 1.0 / 7
    g1 = np.arange(8) * h
    x = np.stack(np.meshgrid(g1, g1), -1).reshape(-1, 2).astype(np.float32)
    n = x.shape[0]
    a = np.full(n, 1.0 / n)
    eps = h * h / 20
    f, g, it, r = orc.sinkhorn(x, x, a, a, 1.0, eps, 2000, tol=1e-13)
    T = orc.dense_plan(x, x, f, g, 1.0, eps)
    off = T.sum() - np.trace(T)
    assert off <= n * math.exp(-20)
    np.testing.assert_allclose(np.diag(T), a, rtol=4 * math.exp(-20) * 1e2)


def test_large_eps_gives_product_coupling(orc):
    x, y = _cloud(9, 20, 30, 3)
    rng = np.random.default_rng(4)
    a = rng.random(20); a /= a.sum()
    b = rng.random(30); b /= b.sum()
    maxc = _sqd(x, y).max()
    errs = []
    for eps in [1e3, 1e5]:
        f, g, it, r = orc.sinkhorn(x, y, a, b, 1.0, eps, 500, tol=1e-15)
        T = orc.dense_plan(x, y, f, g, 1.0, eps)
        rel = np.abs(T / np.outer(a, b) - 1.0).max()
        assert rel <= 2.0 * maxc / eps  # O(max C / eps)
        errs.append(rel)
    assert errs[1] < 2e-2 * errs[0]


def test_primal_dual_gap_vanishes(orc):
    x, y = _cloud(10, 25, 35, 3)
    a = np.full(25, 1 / 25)
    b = np.full(35, 1 / 35)
    eps = 0.05
    f, g, it, r = orc.sinkhorn(x, y, a, b, 1.0, eps, 100000, tol=1e-14)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    C = _sqd(x, y)
    P = (C * T).sum() + eps * (T * (np.log(T) - 1)).sum()
    D = f @ a + g @ b - eps * T.sum()
    assert abs(P - D) <= 1e-10


# ------------------------------------------------------------- invariances
def test_gauge_shift_invariance(orc):
    x, y = _cloud(13, 30, 20, 3)
    a = np.full(30, 1 / 30)
    b = np.full(20, 1 / 20)
    c, eps, k = 1.0, 0.03, 0.37
    f, g, it, r = orc.sinkhorn(x, y, a, b, c, eps, 50)
    T1 = orc.dense_plan(x, y, f, g, c, eps)
    T2 = orc.dense_plan(x, y, f + k, g - k, c, eps)
    np.testing.assert_allclose(T2, T1, rtol=1e-12)
    m1, m2 = orc.min_row(x, y, a, f, g, c, eps), orc.min_row(x, y, a, f + k, g - k, c, eps)
    assert m2["thr"] == pytest.approx(m1["thr"], rel=1e-12)
    np.testing.assert_array_equal(m1["counts"], m2["counts"])
    r1, r2 = orc.marginal_residual(x, y, a, b, f, g, c, eps), orc.marginal_residual(
        x, y, a, b, f + k, g - k, c, eps)
    np.testing.assert_allclose(r2, r1, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(orc.f_step(x, y, a, g - k, c, eps),
                               orc.f_step(x, y, a, g, c, eps) + k, rtol=1e-12, atol=1e-14)


# ------------------------------------------------- materializer and min_row
def test_rows_equal_dense_plan_bit_for_bit(orc):
    # moscot PR #846, "Results": reconstruction is bit-exact (rel_err = 0.0)
    x, y = _cloud(14, 40, 33, 3)
    a = np.full(40, 1 / 40)
    b = np.full(33, 1 / 33)
    f, g, _, _ = orc.sinkhorn(x, y, a, b, 1.0, 0.02, 30)
    T = orc.dense_plan(x, y, f, g, 1.0, 0.02)
    rows = np.array([39, 0, 5, 5, 17], dtype=np.int64)
    assert np.array_equal(orc.materialize_rows(x, y, f, g, 1.0, 0.02, rows), T[rows])


def test_min_row_contract(orc):
    # moscot PR #846, "Behavioural changes": thr = min over massful rows of the row
    # max; every massful row keeps >= 1 entry; independent of the row block size;
    # massless rows keep nothing and do not take part.
    x, y = _cloud(15, 64, 50, 2)
    a = np.full(64, 1 / 60)
    a[[3, 17, 40, 41]] = 0.0
    b = np.full(50, 1 / 50)
    f, g, _, _ = orc.sinkhorn(x, y, a, b, 1.0, 0.01, 40)
    T = orc.dense_plan(x, y, f, g, 1.0, 0.01)
    massful = a > 0
    want = T[massful].max(1).min()
    outs = [orc.min_row(x, y, a, f, g, 1.0, 0.01, block_rows=br) for br in [1, 7, 64, 0]]
    for o in outs:
        assert o["thr"] == want
        assert o["n_massless"] == 4
        assert (o["counts"][massful] >= 1).all()
        assert (o["counts"][~massful] == 0).all()
        np.testing.assert_array_equal(o["counts"], outs[0]["counts"])
        assert o["nnz"] == int((T[massful] >= want).sum())
        assert T[o["argmin"]].max() == want and a[o["argmin"]] > 0


@pytest.mark.parametrize("eps", [0.3, 0.1])
def test_sparsify_two_point_keeps_the_diagonal(orc, eps):
    # x = y = {0, 1}, uniform weights: the converged plan is [[p, q], [q, p]] with
    # p = 1/(2(1+e^{-1/eps})) > q, so thr = p and thresholding keeps exactly the
    # diagonal (moscot PR #846, "Behavioural changes").
    x = np.array([[0.0], [1.0]], np.float32)
    a = np.array([0.5, 0.5])
    f, g, _, _ = orc.sinkhorn(x, x, a, a, 1.0, eps, 5000, tol=1e-15)
    mr = orc.min_row(x, x, a, f, g, 1.0, eps)
    p = 1.0 / (2.0 * (1.0 + math.exp(-1.0 / eps)))
    assert mr["thr"] == pytest.approx(p, rel=1e-10)
    row_ptr, col_idx, vals = orc.sparsify_csr(x, x, a, f, g, 1.0, eps, mr["thr"])
    assert row_ptr.tolist() == [0, 1, 2] and col_idx.tolist() == [0, 1]
    np.testing.assert_allclose(vals, [p, p], rtol=1e-10)


def test_sparsify_csr_is_the_thresholded_plan(orc):
    # The CSR lists, row by row in increasing column order, exactly the entries of
    # the dense plan with T_ij >= thr in rows with mass; every massful row keeps
    # at least its maximum; the per-row counts are min_row's.
    x, y = _cloud(21, 40, 33, 3)
    a = np.full(40, 1 / 37)
    a[[0, 11, 39]] = 0.0
    b = np.full(33, 1 / 33)
    f, g, _, _ = orc.sinkhorn(x, y, a, b, 1.0, 0.02, 30)
    T = orc.dense_plan(x, y, f, g, 1.0, 0.02)
    mr = orc.min_row(x, y, a, f, g, 1.0, 0.02)
    row_ptr, col_idx, vals = orc.sparsify_csr(x, y, a, f, g, 1.0, 0.02, mr["thr"])
    assert row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0) and row_ptr[-1] == len(col_idx) == mr["nnz"]
    np.testing.assert_array_equal(np.diff(row_ptr), mr["counts"])
    dense = np.zeros_like(T)
    for i in range(40):
        cols = col_idx[row_ptr[i]:row_ptr[i + 1]]
        assert np.all(np.diff(cols) > 0)
        dense[i, cols] = vals[row_ptr[i]:row_ptr[i + 1]]
        if a[i] == 0.0:
            assert len(cols) == 0
        else:
            assert int(np.argmax(T[i])) in cols.tolist()
    mask = (T >= mr["thr"]) & (a[:, None] > 0)
    np.testing.assert_array_equal(dense != 0, mask)
    np.testing.assert_array_equal(dense[mask], T[mask])


def test_lr_rows_separable_factors_give_the_product_coupling(orc):
    # Q = a g^T, R = b g^T with sum(g) = 1: Q diag(1/g) R^T = a b^T sum(g) = a b^T
    # (moscot PR #846, "Fix": low-rank rows are (Q diag(1/g) R^T)[rows]).
    rng = np.random.default_rng(3)
    a = rng.random(9); a /= a.sum()
    b = rng.random(6); b /= b.sum()
    g = rng.random(4) + 0.3; g /= g.sum()
    T = orc.lr_rows(np.outer(a, g), np.outer(b, g), g, np.arange(9))
    np.testing.assert_allclose(T, np.outer(a, b), rtol=1e-6)


def test_lr_rows_marginal_and_rank(orc):
    # If R^T 1 = g then T 1 = Q 1; T = Q diag(1/g) R^T has rank <= r; rows in any
    # order and repeated come out as the same rows.
    rng = np.random.default_rng(4)
    n, m, r = 30, 25, 3
    g = (rng.random(r) + 0.5).astype(np.float32)
    R = rng.random((m, r)).astype(np.float64)
    R = (R / R.sum(0) * g.astype(np.float64)).astype(np.float32)
    Q = rng.random((n, r)).astype(np.float32)
    T = orc.lr_rows(Q, R, g, np.arange(n))
    want = Q.astype(np.float64).sum(1)
    np.testing.assert_allclose(T.sum(1), want, rtol=2e-6)
    sv = np.linalg.svd(T, compute_uv=False)
    assert sv[r] <= 1e-12 * sv[0]
    rows = np.array([7, 0, 7, 29])
    np.testing.assert_array_equal(orc.lr_rows(Q, R, g, rows), T[rows])


def test_lrc_rows_squared_euclidean_factorisation(orc):
    # ||x - y||^2 = [|x|^2, 1, -2x] . [1, |y|^2, y]: the low-rank-cost rows with these
    # factors are the point-cloud plan rows (moscot PR #846, "Fix", cost rows of an
    # LRCGeometry); a bias b multiplies every entry by exp(-c b / eps).
    x, y = _cloud(23, 12, 10, 3)
    f = np.random.default_rng(5).normal(0, 0.1, 12)
    g = np.random.default_rng(6).normal(0, 0.1, 10)
    xd, yd = x.astype(np.float64), y.astype(np.float64)
    c1 = np.concatenate([(xd ** 2).sum(1, keepdims=True), np.ones((12, 1)), -2 * xd], 1)
    c2 = np.concatenate([np.ones((10, 1)), (yd ** 2).sum(1, keepdims=True), yd], 1)
    rows = np.array([0, 5, 11])
    eps, c = 0.1, 0.7
    ref = orc.materialize_rows(x, y, f, g, c, eps, rows)
    got = orc.lrc_rows(c1, c2, f, g, 0.0, c, eps, rows)
    np.testing.assert_allclose(got, ref, rtol=1e-5)
    biased = orc.lrc_rows(c1, c2, f, g, 0.25, c, eps, rows)
    np.testing.assert_allclose(biased, got * np.exp(-c * 0.25 / eps), rtol=1e-12)
    # one factor each, by hand: C = c (2 * 3 + bias)
    one = orc.lrc_rows(np.array([[2.0]]), np.array([[3.0]]), [0.4], [-0.1], 1.0, 0.5, 0.2, [0])
    assert one[0, 0] == pytest.approx(math.exp((0.4 - 0.1 - 0.5 * (6.0 + 1.0)) / 0.2), rel=1e-12)


def test_min_row_all_massless(orc):
    x, y = _cloud(16, 5, 4, 2)
    o = orc.min_row(x, y, np.zeros(5), np.full(5, -np.inf), np.zeros(4), 1.0, 0.1)
    assert o["thr"] == np.inf and o["nnz"] == 0 and o["n_massless"] == 5 and o["argmin"] == -1


def test_scale_capture_subset(orc):
    # moscot PR #846, "Fix": rows of a subset use the parent's resolved scale; a
    # subset-derived scale gives different values.
    x, y = _cloud(17, 60, 45, 3)
    a = np.full(60, 1 / 60)
    b = np.full(45, 1 / 45)
    c = orc.inv_scale_cost(x, y, "mean")
    f, g, _, _ = orc.sinkhorn(x, y, a, b, c, 0.05, 50)
    rows = np.arange(0, 60, 7, dtype=np.int64)
    T = orc.dense_plan(x, y, f, g, c, 0.05)
    assert np.array_equal(orc.materialize_rows(x, y, f, g, c, 0.05, rows), T[rows])
    c_sub = orc.inv_scale_cost(x[rows], y, "mean")
    assert c_sub != c
    bad = orc.materialize_rows(x, y, f, g, c_sub, 0.05, rows)
    assert np.abs(bad - T[rows]).max() > 1e-3 * T[rows].max()


def test_scale_mean_closed_form_and_max(orc):
    x, y = _cloud(18, 70, 55, 3)
    xd, yd = x.astype(np.float64), y.astype(np.float64)
    mean = (xd ** 2).sum(1).mean() + (yd ** 2).sum(1).mean() - 2 * xd.mean(0) @ yd.mean(0)
    assert 1.0 / orc.inv_scale_cost(x, y, "mean") == pytest.approx(mean, rel=1e-12)
    assert 1.0 / orc.inv_scale_cost(x, y, "max_cost") == pytest.approx(_sqd(x, y).max(), rel=1e-14)
    assert orc.inv_scale_cost(x, y, "none") == 1.0
    assert orc.inv_scale_cost(x, y, 4.0) == 0.25


# ------------------------------------------------------- log-domain corners
def test_massless_rows_and_all_neg_inf_lse(orc):
    x, y = _cloud(19, 10, 8, 2)
    a = np.full(10, 0.1)
    a[2] = 0.0
    f = orc.f_step(x, y, a, np.zeros(8), 1.0, 0.05)
    assert f[2] == -np.inf and np.isfinite(np.delete(f, 2)).all()
    g = orc.g_step(x, y, np.full(8, 1 / 8), f, 1.0, 0.05)
    assert np.isfinite(g).all()
    # POT PR #868: LSE over an all -inf row is -inf, so f = eps ln a - eps(-inf) = +inf
    f2 = orc.f_step(x, y, a, np.full(8, -np.inf), 1.0, 0.05)
    assert (f2[a > 0] == np.inf).all()


def test_small_eps_stays_finite(orc):
    # POT PR #868: a single global shift underflows at small regularisation where
    # the exact per-row reduction stays finite.
    x, y = _cloud(20, 30, 30, 3)
    a = np.full(30, 1 / 30)
    f, g, it, r = orc.sinkhorn(x, y, a, a, 1.0, 1e-5, 30)
    assert np.isfinite(f).all() and np.isfinite(g).all()


# ------------------------------------------------------------------ drivers
def test_stopping_rule_counts_iterations(orc):
    x, y = _cloud(22, 40, 40, 3)
    a = np.full(40, 1 / 40)
    tol = 1e-4
    f, g, k, r = orc.sinkhorn(x, y, a, a, 1.0, 0.02, 5000, tol=tol)
    assert 1 < k < 5000 and r <= tol
    _, _, k2, r2 = orc.sinkhorn(x, y, a, a, 1.0, 0.02, k - 1, tol=0.0)
    assert k2 == k - 1 and r2 > tol
    f3, g3, k3, r3 = orc.sinkhorn(x, y, a, a, 1.0, 0.02, k, tol=0.0)
    assert np.array_equal(f3, f) and np.array_equal(g3, g) and r3 == r


def test_annealing_schedule(orc):
    x, y = _cloud(23, 30, 30, 3)
    a = np.full(30, 1 / 30)
    eps_t = 0.01
    f, g, stages, r = orc.sinkhorn_anneal(x, y, a, a, 1.0, eps_t, 1.0, 0.7, 5)
    assert stages == math.ceil(math.log(eps_t) / math.log(0.7)) + 1
    # same potentials as running the stages one by one
    f2, g2 = np.zeros(30), np.zeros(30)
    for k in range(stages):
        ek = max(eps_t, 0.7 ** k)
        f2, g2, _, _ = orc.sinkhorn(x, y, a, a, 1.0, ek, 5, f0=f2, g0=g2)
    np.testing.assert_array_equal(f, f2)
    np.testing.assert_array_equal(g, g2)
