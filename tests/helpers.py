"""Shared helpers for the GPU parity tests (comparison rules and device transfer).

Tolerances:
 - potentials: max |f - f_ref| and |g - g_ref| <= 1e-4 * max_ij C_ij (the cost
   as used, i.e. scaled), -inf at the same (massless) entries;
 - plan entries of a plan built at given potentials (the oracle's, rounded to
   float32, or seeded ones; never the GPU's): |T - T_ref| <= 1e-5 * T_ref where
   T_ref >= 1e-30, and T <= 1e-30 where T_ref < 1e-30;
 - marginal residual at the same given potentials: within 1e-5 (absolute; the
   residual of a unit-mass plan is at most 2);
 - min_row: thr within 1e-5 relative, the same argmin row, the same kept
   (i, j) entries except those within 1e-5 relative of thr (counted);
 - compressed-row sparsify: at the same thr, the same kept (i, j) except those
   within 1e-5 relative of thr, columns increasing in each row, values as plan
   entries.
"""
from __future__ import annotations

import numpy as np

POT_TOL = 1e-4
ROW_TOL = 1e-5
RES_TOL = 1e-5
TINY = 1e-30


def to_dev(w, dev="cuda"):
    import torch
    return tuple(torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (w.x, w.y, w.a, w.b))


def max_cost(x, y, c, block=4096):
    """max_ij c * ||x_i - y_j||^2 in float64 (expansion form, blockwise): only the
    normaliser of the potential tolerance, so 1e-12 relative is ample."""
    xd, yd = np.asarray(x, np.float64), np.asarray(y, np.float64)
    best = 0.0
    yy = (yd ** 2).sum(1)
    for i0 in range(0, xd.shape[0], block):
        xb = xd[i0:i0 + block]
        dist = (xb ** 2).sum(1)[:, None] + yy[None, :] - 2 * xb @ yd.T
        best = max(best, float(dist.max()))
    return c * best


def assert_potentials(got, ref, maxc, tol=POT_TOL, what="f"):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    ninf_g, ninf_r = np.isneginf(got), np.isneginf(ref)
    assert np.array_equal(ninf_g, ninf_r), f"{what}: -inf pattern differs"
    fin = ~ninf_r
    assert np.isfinite(got[fin]).all(), f"{what}: non-finite entries"
    err = np.abs(got[fin] - ref[fin]).max() / maxc if fin.any() else 0.0
    assert err <= tol, f"{what}: max err {err:.3e} of max C (tol {tol})"
    return err


def assert_entries(T, T_ref, tol=ROW_TOL):
    T, T_ref = np.asarray(T, np.float64), np.asarray(T_ref, np.float64)
    big = T_ref >= TINY
    rel = np.abs(T[big] - T_ref[big]) / T_ref[big]
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= tol, f"plan entries: max rel err {worst:.3e}"
    # below the floor both must be tiny; the floor itself carries the same
    # relative band, so rounding across exactly 1e-30 is not a failure
    small = T[~big]
    assert np.all(small <= TINY * (1.0 + tol)), (
        f"oracle entry below 1e-30 but {float(small.max()):.3e} here "
        f"(oracle {float(T_ref[~big][np.argmax(small)]):.3e})")
    return worst


def assert_min_row(got, ref, tol=ROW_TOL):
    assert got["n_massless"] == ref["n_massless"]
    if ref["argmin"] < 0:
        assert got["argmin"] == -1 and np.isinf(got["thr"])
        return 0
    assert abs(got["thr"] - ref["thr"]) <= tol * ref["thr"], (got["thr"], ref["thr"])
    assert got["argmin"] == ref["argmin"]
    return 0


def csr_rows(row_ptr, col_idx, vals):
    """{row: (columns, values)} from compressed-row arrays (numpy)."""
    out = {}
    for i in range(len(row_ptr) - 1):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        out[i] = (np.asarray(col_idx[a:b]), np.asarray(vals[a:b], np.float64))
    return out


def assert_csr(got, ref, thr, tol=ROW_TOL, band_tol=None):
    """got/ref: (row_ptr, col_idx, vals) as numpy arrays, thresholded at thr.
    The kept sets agree except entries within band_tol (relative, default tol) of
    thr; values of entries kept by both agree as plan entries (tol). Returns the
    tie-band count."""
    band_tol = tol if band_tol is None else band_tol
    g, r = csr_rows(*got), csr_rows(*ref)
    assert len(g) == len(r)
    band = 0
    for i in r:
        gc, gv = g[i]
        rc, rv = r[i]
        assert np.all(np.diff(gc) > 0), f"row {i}: columns not increasing"
        common, gi, ri = np.intersect1d(gc, rc, return_indices=True)
        if common.size:
            assert_entries(gv[gi], rv[ri], tol)
        only_g = np.setdiff1d(np.arange(len(gc)), gi)
        only_r = np.setdiff1d(np.arange(len(rc)), ri)
        for v in list(gv[only_g]) + list(rv[only_r]):
            assert abs(v - thr) <= band_tol * thr, f"row {i}: entry {v:.6e} kept by one side only, thr {thr:.6e}"
            band += 1
    return band


def f32(v):
    """float64 copy of v rounded to float32: the potentials both sides are given."""
    return np.asarray(v, np.float64).astype(np.float32).astype(np.float64)


def plan_at(ot, w, f, g, **kw):
    """A GPU plan at given potentials (warm start, no iteration), so that rows,
    residuals, min_row and sparsify are compared with the oracle at potentials
    that come from the oracle or from a seeded generator, never from the GPU."""
    import torch
    x, y, a, b = to_dev(w)
    ft = torch.from_numpy(np.asarray(f, np.float32).copy()).cuda()
    gt = torch.from_numpy(np.asarray(g, np.float32).copy()).cuda()
    kw.setdefault("eps", w.eps)
    kw.setdefault("scale", w.scale)
    return ot.sinkhorn(x, y, a, b, n_iters=0, f=ft, g=gt, warm_start=True, **kw)
