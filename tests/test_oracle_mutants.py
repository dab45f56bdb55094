"""The oracle's pins catch plausible mistakes: each test plants one mistake in a
temporary copy of the oracle's C source (a flipped sign, a dropped factor, a max
for a min, ...), builds it, and checks that the pin battery below fails on it
while passing on the real oracle. Nothing here touches the real oracle's files.
"""
import importlib.util
import math
import os
import shutil
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle")

MUTANTS = {
    "cost_sign_in_f_step": ("(g[j] - cost(x, y, i, j, d, c)) / eps", "(g[j] + cost(x, y, i, j, d, c)) / eps"),
    "dropped_eps_on_log_weight": ("out = eps * log(a[i]) - eps * lse(v, m);", "out = log(a[i]) - eps * lse(v, m);"),
    "plan_sign_of_g": ("exp((f[i] + g[j] - cost(x, y, i, j, d, c)) / eps)", "exp((f[i] - g[j] - cost(x, y, i, j, d, c)) / eps)"),
    "plan_missing_eps": ("exp((f[i] + g[j] - cost(x, y, i, j, d, c)) / eps)", "exp((f[i] + g[j] - cost(x, y, i, j, d, c)))"),
    "min_row_takes_max": ("if (rowmax[i] < thr) { thr = rowmax[i]; arg = i; }", "if (rowmax[i] > thr || thr == INFINITY) { thr = rowmax[i]; arg = i; }"),
    "residual_wrong_sign": ("for (int64_t i = 0; i < n; ++i) r += fabs(rs[i] - a[i]);", "for (int64_t i = 0; i < n; ++i) r += fabs(rs[i] + a[i]);"),
    "mean_scale_wrong_count": ("if (mode == 1) r /= ((double)n * (double)m);", "if (mode == 1) r /= ((double)n * (double)n);"),
    "lse_no_shift_back": ("return mx + log(s);", "return log(s);"),
    "g_step_uses_a_weight": ("out = eps * log(b[j]) - eps * lse(v, n);", "out = eps * log(b[0]) - eps * lse(v, n);"),
    "csr_strict_threshold": ("            if (t >= thr) {\n                col_idx[k] = j;", "            if (t > thr) {\n                col_idx[k] = j;"),
    "csr_drops_the_column_order": ("                col_idx[k] = j;", "                col_idx[k] = m - 1 - j;"),
    "lr_multiplies_by_g": ("(double)R[j * r + q] / (double)g[q];", "(double)R[j * r + q] * (double)g[q];"),
    "lrc_drops_the_bias": ("const double C = c * (dot + bias);", "const double C = c * dot;"),
    "morton_bit_order": ("cd |= (uint64_t)1 << (t * d + (d - 1 - k));", "cd |= (uint64_t)1 << (t * d + k);"),
    "screen_drops_tile_size": ("log((double)ni * (double)mj) + (sp[0]", "(sp[0]"),
    "screen_gap_one_sided": ("if (sq[2 + k] - sp[2 + d + k] > gap) gap = sq[2 + k] - sp[2 + d + k];", ""),
    "threshold_takes_the_larger_weight": ("log(sp[1] < sq[1] ? sp[1] : sq[1])", "log(sp[1] > sq[1] ? sp[1] : sq[1])"),
    "sparse_f_without_fallback": ("if (all || adm[p * MB + j / B]) v[len++]", "if (adm[p * MB + j / B]) v[len++]"),
    "sparse_residual_counts_all_columns": ("if (all || adm[p * MB + j / B]) s +=", "s +="),
    "sparse_stop_ignores_the_omitted_mass": ("const double tol_eff = tol - (double)MB * delta * asum;",
                                             "const double tol_eff = tol;"),
    "sparse_g_step_without_fallback": ("if (all || adm[(i / B) * MB + q]) v[len++]", "if (adm[(i / B) * MB + q]) v[len++]"),
}


def _load_variant(tmp_path, name, old=None, new=None):
    dst = tmp_path / f"oracle_{name}"
    shutil.copytree(SRC, dst, ignore=shutil.ignore_patterns("_build", "__pycache__"))
    if old is not None:
        c = (dst / "sinkhorn_oracle.c").read_text()
        assert old in c, f"mutation site for {name} not found"
        (dst / "sinkhorn_oracle.c").write_text(c.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", dst / "__init__.py",
                                                  submodule_search_locations=[str(dst)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _sqd(x, y):
    xd, yd = np.asarray(x, np.float64), np.asarray(y, np.float64)
    return ((xd[:, None, :] - yd[None]) ** 2).sum(-1)


def _battery(orc):
    """Returns the names of the pins that fail for this oracle build."""
    failed = []
    rng = np.random.default_rng(0)
    x = rng.random((9, 2)).astype(np.float32)
    y = rng.random((7, 2)).astype(np.float32)
    a = rng.random(9) + 0.1
    a /= a.sum()
    b = rng.random(7) + 0.1
    b /= b.sum()
    g = rng.normal(0, 0.2, 7)
    eps, c = 0.1, 1.3

    def check(name, fn):
        try:
            if not fn():
                failed.append(name)
        except Exception:
            failed.append(name)

    def row_marginals():
        f = orc.f_step(x, y, a, g, c, eps)
        return np.allclose(orc.dense_plan(x, y, f, g, c, eps).sum(1), a, rtol=1e-12)

    def col_marginals():
        f = orc.f_step(x, y, a, g, c, eps)
        g2 = orc.g_step(x, y, b, f, c, eps)
        return np.allclose(orc.dense_plan(x, y, f, g2, c, eps).sum(0), b, rtol=1e-12)

    def two_point():
        x2 = np.array([[0.0], [1.0]], np.float32)
        h = np.array([0.5, 0.5])
        f, gg, _, _ = orc.sinkhorn(x2, x2, h, h, 1.0, 0.3, 5000, tol=1e-15)
        p = 1.0 / (2.0 * (1.0 + math.exp(-1.0 / 0.3)))
        return abs(orc.dense_plan(x2, x2, f, gg, 1.0, 0.3)[0, 0] - p) < 1e-9

    def cross_ratio():
        f = rng.normal(0, 0.2, 9)
        T = orc.dense_plan(x, y, f, g, c, eps)
        C = c * _sqd(x, y)
        lhs = T[0, 0] * T[1, 1] / (T[0, 1] * T[1, 0])
        return abs(lhs / math.exp((C[0, 1] + C[1, 0] - C[0, 0] - C[1, 1]) / eps) - 1) < 1e-10

    def min_row_contract():
        f, gg, _, _ = orc.sinkhorn(x, y, a, b, c, eps, 20)
        T = orc.dense_plan(x, y, f, gg, c, eps)
        o = orc.min_row(x, y, a, f, gg, c, eps)
        return o["thr"] == T.max(1).min() and (o["counts"] >= 1).all()

    def residual():
        f, gg, _, _ = orc.sinkhorn(x, y, a, b, c, eps, 3)
        T = orc.dense_plan(x, y, f, gg, c, eps)
        r, q = orc.marginal_residual(x, y, a, b, f, gg, c, eps)
        return abs(r - np.abs(T.sum(1) - a).sum()) < 1e-12 and abs(q - np.abs(T.sum(0) - b).sum()) < 1e-12

    def csr():
        f, gg, _, _ = orc.sinkhorn(x, y, a, b, c, eps, 20)
        T = orc.dense_plan(x, y, f, gg, c, eps)
        thr = T.max(1).min()
        row_ptr, col_idx, vals = orc.sparsify_csr(x, y, a, f, gg, c, eps, thr)
        dense = np.zeros_like(T)
        for i in range(len(a)):
            dense[i, col_idx[row_ptr[i]:row_ptr[i + 1]]] = vals[row_ptr[i]:row_ptr[i + 1]]
        return np.array_equal(dense != 0, T >= thr) and np.array_equal(dense[T >= thr], T[T >= thr])

    def lowrank():
        g4 = np.array([0.2, 0.3, 0.5])
        Q = np.outer(a, g4)
        R = np.outer(b, g4)
        ok = np.allclose(orc.lr_rows(Q, R, g4, np.arange(len(a))), np.outer(a, b), rtol=1e-6)
        one = orc.lrc_rows(np.array([[2.0]]), np.array([[3.0]]), [0.4], [-0.1], 1.0, 0.5, 0.2, [0])
        return ok and abs(one[0, 0] / math.exp((0.4 - 0.1 - 0.5 * 7.0) / 0.2) - 1) < 1e-12

    def mean_scale():
        xd, yd = x.astype(np.float64), y.astype(np.float64)
        mean = (xd ** 2).sum(1).mean() + (yd ** 2).sum(1).mean() - 2 * xd.mean(0) @ yd.mean(0)
        return abs(1.0 / orc.inv_scale_cost(x, y, "mean") - mean) < 1e-12 * mean

    def block_sparse():
        # FlashSinkhorn 2, sections 3, 3.2, A.3: Z-order, screen, verification,
        # omitted-mass bound and the masked updates' marginals
        grid = np.array([(i / 3, j / 3) for i in range(4) for j in range(4)], np.float32)
        perm = orc.morton_order(grid, np.zeros(2), np.ones(2))
        z = [(0, 0), (0, 1), (1, 0), (1, 1), (0, 2), (0, 3), (1, 2), (1, 3),
             (2, 0), (2, 1), (3, 0), (3, 1), (2, 2), (2, 3), (3, 2), (3, 3)]
        if [(int(round(grid[k, 0] * 3)), int(round(grid[k, 1] * 3))) for k in perm] != z:
            return False
        r3 = np.random.default_rng(2)  # coincident points per block: the screen bound is exact
        xt = np.repeat(r3.random((5, 3)), 4, axis=0).astype(np.float32)[:19]
        yt = np.repeat(r3.random((4, 3)), 4, axis=0).astype(np.float32)
        ft, gt = np.repeat(r3.normal(0, 0.05, 5), 4)[:19], np.repeat(r3.normal(0, 0.05, 4), 4)
        at, bt = r3.random(19) + 0.1, r3.random(16) + 0.1
        Tt = orc.dense_plan(xt, yt, ft, gt, 1.7, 0.05)
        Mt = np.array([[Tt[p * 4:(p + 1) * 4, q * 4:(q + 1) * 4].sum() for q in range(4)] for p in range(5)])
        rt = 1e-3 * np.minimum(np.array([at[p * 4:(p + 1) * 4].min() for p in range(5)])[:, None],
                               np.array([bt[q * 4:(q + 1) * 4].min() for q in range(4)])[None, :])
        ot = orc.block_mask(xt, yt, at, bt, ft, gt, 1.7, 0.05, 4, 1e-3)
        if not np.allclose(ot["screen_margin"], np.log(Mt / rt), rtol=0, atol=1e-9):
            return False
        r2 = np.random.default_rng(5)
        xs, ys = r2.random((120, 3)).astype(np.float32), r2.random((100, 3)).astype(np.float32)
        lo, hi = orc.joint_box(xs, ys)
        xs, ys = xs[orc.morton_order(xs, lo, hi)], ys[orc.morton_order(ys, lo, hi)]
        aa, bb = r2.random(120) + 0.2, r2.random(100) + 0.2
        aa, bb = aa / aa.sum(), bb / bb.sum()
        e2, B, delta = 0.004, 8, 1e-3
        f2, g2, _, _ = orc.sinkhorn(xs, ys, aa, bb, 1.0, e2, 15)
        T = orc.dense_plan(xs, ys, f2, g2, 1.0, e2)
        NB, MB = 15, 13
        M = np.array([[T[p * B:(p + 1) * B, q * B:(q + 1) * B].sum() for q in range(MB)] for p in range(NB)])
        amin = np.array([aa[p * B:(p + 1) * B].min() for p in range(NB)])
        bmin = np.array([bb[q * B:(q + 1) * B].min() for q in range(MB)])
        rho = delta * np.minimum(amin[:, None], bmin[None, :])
        o = orc.block_mask(xs, ys, aa, bb, f2, g2, 1.0, e2, B, delta)
        if not np.all(o["screen_margin"] >= np.log(M / rho) - 1e-9):
            return False
        if not np.array_equal(o["adm"], o["cand"] & (M > rho)):
            return False
        for p in range(NB):
            for q in range(MB):
                if not o["adm"][p, q]:
                    t = T[p * B:(p + 1) * B, q * B:(q + 1) * B]
                    if np.any(t.sum(1) > delta * aa[p * B:(p + 1) * B] * (1 + 1e-12)):
                        return False
        adm = o["adm"].copy()
        adm[2, :] = False  # a row block that falls back to every column
        fs = orc.sparse_f_step(xs, ys, aa, g2, 1.0, e2, B, adm)
        rows = np.repeat(np.repeat(adm, B, axis=0), B, axis=1)[:120, :100]
        rows[16:24, :] = True
        T = orc.dense_plan(xs, ys, fs, g2, 1.0, e2)
        if not np.allclose((T * rows).sum(1), aa, rtol=1e-12, atol=0):
            return False
        if abs(orc.sparse_row_residual(xs, ys, aa, fs, g2, 1.0, e2, B, adm)) >= 1e-13:
            return False
        # the g-update with a column block that falls back to every row
        adm2 = o["adm"].copy()
        adm2[:, 3] = False
        gs = orc.sparse_g_step(xs, ys, bb, fs, 1.0, e2, B, adm2)
        cols = np.repeat(np.repeat(adm2, B, axis=0), B, axis=1)[:120, :100]
        cols[:, 24:32] = True
        T = orc.dense_plan(xs, ys, fs, gs, 1.0, e2)
        if not np.allclose((T * cols).sum(0), bb, rtol=1e-12, atol=0):
            return False
        # the certificate: the stop test leaves room for the omitted mass
        ux, uy = r2.random((400, 3)).astype(np.float32), r2.random((380, 3)).astype(np.float32)
        ua, ub = np.full(400, 1 / 400), np.full(380, 1 / 380)
        tol = 1e-2
        _, _, _, rr, _ = orc.sinkhorn_sparse(ux, uy, ua, ub, 1.0, 4e-3, 300, tol=tol, B=32, dense_frac=1.0)
        omitted = 12 * (tol / (4 * 13)) * ua.sum()
        return rr <= tol - omitted

    for name, fn in [("block_sparse", block_sparse), ("row_marginals", row_marginals), ("col_marginals", col_marginals),
                     ("two_point", two_point), ("cross_ratio", cross_ratio),
                     ("min_row_contract", min_row_contract), ("residual", residual), ("csr", csr),
                     ("lowrank", lowrank),
                     ("mean_scale", mean_scale)]:
        check(name, fn)
    return failed


def test_real_oracle_passes_the_battery(tmp_path):
    assert _battery(_load_variant(tmp_path, "real")) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    failed = _battery(_load_variant(tmp_path, name, old, new))
    assert failed, f"no pin caught the mutant {name}"
