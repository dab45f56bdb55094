"""Pins of the oracle's block-sparse fine updates ("FlashSinkhorn 2: Block-Sparse
Entropic Optimal Transport", sections 3, 3.2, A.3, B.1, B.3) against what the
mathematics fixes: the Z-order of small grids, the screen and the verification
against tile masses summed from the dense plan (itself pinned in
test_oracle_pins.py), the per-tile omitted-mass bound, the marginals that a masked
update must reproduce exactly, the invariance of the mask under (f + k, g - k),
permutation equivariance, the full mask reducing to the dense solve, and the
certified full residual of a converged solve. CPU only.
"""
import itertools

import numpy as np
import pytest

import oracle as orc


def _problem(n, m, d=3, seed=0, massless=False):
    rng = np.random.default_rng(seed)
    x = rng.random((n, d)).astype(np.float32)
    y = rng.random((m, d)).astype(np.float32)
    a = rng.random(n) + 0.2
    b = rng.random(m) + 0.2
    if massless:
        a[::17] = 0.0
    return x, y, a / a.sum(), b / b.sum()


def _sorted(x, y, a, b):
    lo, hi = orc.joint_box(x, y)
    px, py = orc.morton_order(x, lo, hi), orc.morton_order(y, lo, hi)
    return x[px], y[py], a[px], b[py], px, py


def _tile_sums(T, B):
    n, m = T.shape
    NB, MB = -(-n // B), -(-m // B)
    out = np.zeros((NB, MB))
    for p in range(NB):
        for q in range(MB):
            out[p, q] = T[p * B:(p + 1) * B, q * B:(q + 1) * B].sum()
    return out


def _rho(a, b, B, delta):
    NB, MB = -(-len(a) // B), -(-len(b) // B)
    amin = np.array([a[p * B:(p + 1) * B][a[p * B:(p + 1) * B] > 0].min(initial=np.inf) for p in range(NB)])
    bmin = np.array([b[q * B:(q + 1) * B][b[q * B:(q + 1) * B] > 0].min(initial=np.inf) for q in range(MB)])
    return delta * np.minimum(amin[:, None], bmin[None, :])


def _state(x, y, a, b, eps, iters=15):
    f, g, _, _ = orc.sinkhorn(x, y, a, b, 1.0, eps, iters)
    return f, g


# ------------------------------------------------------------------ Morton --
def test_morton_z_order_of_a_4x4_grid():
    # Z-curve with coordinate 0 the more significant bit of each pair (hand-listed)
    pts = np.array([(i / 3, j / 3) for i in range(4) for j in range(4)], np.float32)
    expect = [(0, 0), (0, 1), (1, 0), (1, 1), (0, 2), (0, 3), (1, 2), (1, 3),
              (2, 0), (2, 1), (3, 0), (3, 1), (2, 2), (2, 3), (3, 2), (3, 3)]
    perm = orc.morton_order(pts, np.zeros(2), np.ones(2))
    got = [(int(round(pts[k, 0] * 3)), int(round(pts[k, 1] * 3))) for k in perm]
    assert got == expect


def test_morton_octants_count_in_binary():
    pts = np.array(list(itertools.product([1.0, 0.0], repeat=3)), np.float32)  # reversed listing
    perm = orc.morton_order(pts, np.zeros(3), np.ones(3))
    assert [tuple(int(v) for v in pts[k]) for k in perm] == list(itertools.product([0, 1], repeat=3))


def test_morton_in_one_dimension_is_a_stable_argsort():
    rng = np.random.default_rng(3)
    x = rng.permutation(np.arange(500, dtype=np.float32) / 499.0)
    x = np.concatenate([x, x[:40]])  # repeated values: ties go by index
    perm = orc.morton_order(x[:, None], np.zeros(1), np.ones(1))
    assert np.array_equal(perm, np.argsort(x, kind="stable"))


def test_morton_code_of_the_far_corner_sets_every_bit():
    code = orc.morton_codes(np.ones((1, 3), np.float32), np.zeros(3), np.ones(3))
    assert int(code[0]) == (1 << 30) - 1


# ----------------------------------------------------------- screen/verify --
def test_screen_with_single_point_blocks_is_the_entry_test():
    # B = 1: the box distance is the point distance, so U_pq = T_pq exactly
    x, y, a, b = _problem(40, 30, d=2, seed=1)
    eps, delta = 0.02, 1e-3
    f, g = _state(x, y, a, b, eps)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    rho = _rho(a, b, 1, delta)
    o = orc.block_mask(x, y, a, b, f, g, 1.0, eps, 1, delta, verify=False)
    margin = np.log(T) - np.log(rho)
    assert np.allclose(o["screen_margin"], margin, atol=1e-9)
    clear = np.abs(margin) > 1e-9
    assert np.array_equal(o["cand"][clear], (T > rho)[clear])
    assert 0 < o["n_cand"] < T.size


def test_screen_bound_is_tight_for_blocks_of_coincident_points():
    # every block repeats one point and holds one potential value, so
    # M_pq = |I||J| exp((F_p + G_q - c D_pq)/eps) = U_pq exactly
    rng = np.random.default_rng(2)
    B, NB, MB, eps, delta, c = 4, 5, 4, 0.05, 1e-3, 1.7
    x = np.repeat(rng.random((NB, 3)), B, axis=0).astype(np.float32)[:NB * B - 1]  # ragged
    y = np.repeat(rng.random((MB, 3)), B, axis=0).astype(np.float32)
    f = np.repeat(rng.normal(0, 0.05, NB), B)[:NB * B - 1]
    g = np.repeat(rng.normal(0, 0.05, MB), B)
    a, b = rng.random(NB * B - 1) + 0.1, rng.random(MB * B) + 0.1
    M = _tile_sums(orc.dense_plan(x, y, f, g, c, eps), B)
    o = orc.block_mask(x, y, a, b, f, g, c, eps, B, delta)
    assert np.allclose(o["screen_margin"], np.log(M / _rho(a, b, B, delta)), rtol=0, atol=1e-9)
    assert np.allclose(o["mass_margin"][o["cand"]], o["screen_margin"][o["cand"]], atol=1e-9)


@pytest.mark.parametrize("B,seed", [(4, 0), (8, 1), (16, 2)])
def test_screen_bound_dominates_every_tile_mass(B, seed):
    x, y, a, b = _problem(150, 121, seed=seed)
    x, y, a, b, _, _ = _sorted(x, y, a, b)
    eps, delta = 0.004, 1e-4
    f, g = _state(x, y, a, b, eps)
    M = _tile_sums(orc.dense_plan(x, y, f, g, 1.0, eps), B)
    rho = _rho(a, b, B, delta)
    o = orc.block_mask(x, y, a, b, f, g, 1.0, eps, B, delta)
    # ln U - ln rho >= ln M - ln rho for every tile; a rejected tile carries <= rho
    assert np.all(o["screen_margin"] >= np.log(M / rho) - 1e-9)
    assert np.all(M[~o["cand"]] <= rho[~o["cand"]] * (1 + 1e-12))
    # the screen is not trivial here: it rejects some tiles and keeps others
    assert 0 < o["n_cand"] < M.size


@pytest.mark.parametrize("B", [4, 16])
def test_verification_admits_exactly_the_tiles_above_the_threshold(B):
    x, y, a, b = _problem(130, 170, seed=4)
    x, y, a, b, _, _ = _sorted(x, y, a, b)
    eps, delta = 0.004, 1e-4
    f, g = _state(x, y, a, b, eps)
    M = _tile_sums(orc.dense_plan(x, y, f, g, 1.0, eps), B)
    rho = _rho(a, b, B, delta)
    o = orc.block_mask(x, y, a, b, f, g, 1.0, eps, B, delta)
    assert np.allclose(o["mass_margin"][o["cand"]], np.log(M / rho)[o["cand"]], atol=1e-9)
    clear = np.abs(np.log(M / rho)) > 1e-9
    assert np.array_equal(o["adm"][clear], (o["cand"] & (M > rho))[clear])
    assert o["n_adm"] == int(o["adm"].sum()) < o["n_cand"]


def test_omitted_tiles_respect_the_per_row_and_per_column_bound():
    # an omitted tile adds at most delta a_i to row i and delta b_j to column j
    x, y, a, b = _problem(200, 160, seed=5, massless=True)
    x, y, a, b, _, _ = _sorted(x, y, a, b)
    eps, delta, B = 0.003, 1e-3, 16
    f, g = _state(x, y, a, b, eps)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    o = orc.block_mask(x, y, a, b, f, g, 1.0, eps, B, delta)
    NB, MB = o["adm"].shape
    for p in range(NB):
        for q in range(MB):
            if o["adm"][p, q]:
                continue
            tile = T[p * B:(p + 1) * B, q * B:(q + 1) * B]
            assert np.all(tile.sum(1) <= delta * a[p * B:(p + 1) * B] * (1 + 1e-12))
            assert np.all(tile.sum(0) <= delta * b[q * B:(q + 1) * B] * (1 + 1e-12))


def test_mask_is_invariant_under_opposite_potential_shifts():
    x, y, a, b = _problem(96, 80, seed=6)
    x, y, a, b, _, _ = _sorted(x, y, a, b)
    eps, delta, B = 0.004, 1e-4, 8
    f, g = _state(x, y, a, b, eps)
    f, g = np.round(f * 1024) / 1024, np.round(g * 1024) / 1024  # dyadic: sums stay exact
    o1 = orc.block_mask(x, y, a, b, f, g, 1.0, eps, B, delta)
    o2 = orc.block_mask(x, y, a, b, f + 0.25, g - 0.25, 1.0, eps, B, delta)
    assert np.array_equal(o1["cand"], o2["cand"]) and np.array_equal(o1["adm"], o2["adm"])


# ----------------------------------------------------------- masked updates --
def _mask_with_empty_blocks(NB, MB, seed):
    rng = np.random.default_rng(seed)
    adm = rng.random((NB, MB)) < 0.4
    adm[1, :] = False      # a row block with no admitted tile
    adm[:, 2] = False      # a column block with no admitted tile
    return adm


def test_masked_updates_reproduce_the_admitted_marginals():
    x, y, a, b = _problem(90, 75, seed=7, massless=True)
    eps, B = 0.01, 8
    g = np.random.default_rng(8).normal(0, 0.01, 75)
    adm = _mask_with_empty_blocks(-(-90 // B), -(-75 // B), 9)
    cols = np.repeat(adm, B, axis=1)[:, :75]
    rows_mask = np.repeat(cols, B, axis=0)[:90]  # [n, m] admitted pairs
    rows_mask[8:16, :] = True                    # row block 1 reduces over everything
    f = orc.sparse_f_step(x, y, a, g, 1.0, eps, B, adm)
    T = orc.dense_plan(x, y, f, g, 1.0, eps)
    assert np.allclose((T * rows_mask).sum(1), a, rtol=1e-12, atol=0)
    g2 = orc.sparse_g_step(x, y, b, f, 1.0, eps, B, adm)
    T = orc.dense_plan(x, y, f, g2, 1.0, eps)
    cmask = np.repeat(np.repeat(adm, B, axis=0)[:90], B, axis=1)[:, :75]
    cmask[:, 16:24] = True                       # column block 2 reduces over everything
    assert np.allclose((T * cmask).sum(0), b, rtol=1e-12, atol=0)
    assert np.isclose(orc.sparse_row_residual(x, y, a, f, g, 1.0, eps, B, adm), 0.0, atol=1e-14)


def test_full_mask_gives_the_dense_updates():
    x, y, a, b = _problem(70, 66, seed=10)
    eps, B = 0.02, 16
    g = np.random.default_rng(11).normal(0, 0.02, 66)
    adm = np.ones((-(-70 // B), -(-66 // B)), dtype=bool)
    f = orc.sparse_f_step(x, y, a, g, 1.0, eps, B, adm)
    assert np.allclose(f, orc.f_step(x, y, a, g, 1.0, eps), rtol=0, atol=1e-14)
    assert np.allclose(orc.sparse_g_step(x, y, b, f, 1.0, eps, B, adm),
                       orc.g_step(x, y, b, f, 1.0, eps), rtol=0, atol=1e-14)


# ----------------------------------------------------------------- driver --
def test_sparse_solve_with_every_tile_admitted_is_the_dense_solve():
    x, y, a, b = _problem(120, 100, seed=12)
    eps = 0.01
    fd, gd, _, _ = orc.sinkhorn(x, y, a, b, 1.0, eps, 30)
    fs, gs, it, _, st = orc.sinkhorn_sparse(x, y, a, b, 1.0, eps, 30, B=16, delta=1e-300,
                                            dense_frac=1.0)
    assert it == 30 and st[0] == 30 and st[1] == 0
    assert np.allclose(fs, fd, rtol=0, atol=1e-13) and np.allclose(gs, gd, rtol=0, atol=1e-13)


def test_sparse_solve_certifies_the_full_residual():
    x, y, a, b = _problem(600, 500, seed=13)
    eps, tol = 1.5e-3, 1e-2
    f, g, it, r, st = orc.sinkhorn_sparse(x, y, a, b, 1.0, eps, 400, tol=tol, B=32,
                                          dense_frac=1.0)
    NB, MB = -(-600 // 32), -(-500 // 32)
    assert st[0] == it and st[3] < NB * MB           # sparse iterations on a real mask
    omitted = MB * (tol / (4 * max(NB, MB))) * a.sum()  # bound on the mass the mask omits
    assert r <= tol - omitted
    full, _ = orc.marginal_residual(x, y, a, b, f, g, 1.0, eps)
    assert full <= tol and abs(full - r) <= omitted


def test_sparse_solve_is_permutation_equivariant():
    x, y, a, b = _problem(150, 140, seed=14)
    perm_x = np.random.default_rng(15).permutation(150)
    perm_y = np.random.default_rng(16).permutation(140)
    kw = dict(B=16, delta=1e-5, dense_frac=1.0)
    f1, g1, _, _, _ = orc.sinkhorn_sparse(x, y, a, b, 1.0, 0.004, 12, **kw)
    f2, g2, _, _, _ = orc.sinkhorn_sparse(x[perm_x], y[perm_y], a[perm_x], b[perm_y], 1.0, 0.004,
                                          12, **kw)
    assert np.array_equal(f2, f1[perm_x]) and np.array_equal(g2, g1[perm_y])


def test_candidate_fraction_policy_switches_to_dense_iterations():
    x, y, a, b = _problem(100, 90, seed=17)
    f, g, it, _, st = orc.sinkhorn_sparse(x, y, a, b, 1.0, 0.5, 5, B=16, delta=1e-6,
                                          dense_frac=0.5)
    assert st == (0, 5, 42, 42)  # large eps: every tile survives, so every iteration is dense
    fd, gd, _, _ = orc.sinkhorn(x, y, a, b, 1.0, 0.5, 5)
    assert np.allclose(f, fd, atol=1e-13) and np.allclose(g, gd, atol=1e-13)
