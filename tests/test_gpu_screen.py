"""The tile screen of the row passes against the materialized plan (-m gpu).

For d <= 3 the residual, min_row and count passes visit rows and columns in
Morton order and skip every (32-row, 256-column) tile whose bound on the
exponent,
    kappa max_I f + kappa max_J g - kappa c dist(box(x'_I), box(y'_J))^2,
lies below -127: all its entries are below 2^-126, where the entry function
returns exactly 0. The materializer visits every entry in the plain order, so
its rows are the reference the screen must reproduce exactly: thr (the min over
massful rows of the row maxima), its argmin and the kept counts bit for bit,
the residuals up to summation order. The problems are clustered clouds at a
small eps, where many entries vanish (the test checks that they do), with
massless rows and columns.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ot():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import log_domain_sinkhorn_online_b200 as pkg
    return pkg


def _clusters(rng, count, d, centres):
    k = rng.integers(0, len(centres), count)
    return np.clip(centres[k] + 0.02 * rng.standard_normal((count, d)), 0.0, 1.0).astype(np.float32)


def _problem(d, n, m, seed):
    import torch
    rng = np.random.default_rng(seed)
    centres = rng.random((24, d))
    x, y = _clusters(rng, n, d, centres), _clusters(rng, m, d, centres)
    a = rng.random(n).astype(np.float32) + 0.5
    b = rng.random(m).astype(np.float32) + 0.5
    a[7::101] = 0.0
    b[3::89] = 0.0
    a, b = (a / a.sum()).astype(np.float32), (b / b.sum()).astype(np.float32)
    return tuple(torch.from_numpy(v).cuda() for v in (x, y, a, b))


@pytest.mark.parametrize("d,eps", [(1, 1e-4), (2, 2e-4), (3, 3e-4)])
def test_screened_passes_equal_the_materialized_plan(ot, d, eps):
    import torch
    n, m = 3001, 2603
    x, y, a, b = _problem(d, n, m, 60 + d)
    p = ot.sinkhorn(x, y, a, b, eps=eps, scale="max_cost", n_iters=40)
    T = p.materialize_rows(torch.arange(n, device="cuda"))
    assert (T == 0).double().mean().item() > 0.3          # many entries vanish: the screen has work
    massful = a > 0
    rowmax = T.max(1).values
    thr_ref = rowmax[massful].min()
    argmin_ref = int(torch.nonzero(massful & (rowmax == thr_ref))[0])
    counts_ref = torch.where(massful, (T >= thr_ref).sum(1), torch.zeros_like(rowmax, dtype=torch.int64))
    for block_rows in (0, 1000):
        mr = p.sparsify_min_row(block_rows=block_rows)
        visited, total = p.row_pass_stats()
        assert total > 0 and 0 < visited < total              # the screen skipped tiles
        assert mr["thr"] == float(thr_ref) and mr["argmin"] == argmin_ref
        assert torch.equal(mr["counts"], counts_ref) and mr["nnz"] == int(counts_ref.sum())
        assert mr["n_massless"] == int((~massful).sum())
    # kept counts at a threshold below every entry but 0: the count pass may not skip
    # vanishing tiles there (they count at thr <= 0), and at a tiny positive thr it may
    from log_domain_sinkhorn_online_b200 import _binding as B
    s = torch.cuda.current_stream().cuda_stream
    c0 = torch.empty(n, dtype=torch.int64, device="cuda")
    assert B.ot_kept_counts_range(p.handle, 0, n, 0, 0.0, c0.data_ptr(), s) == int(massful.sum()) * m
    tiny = float(T[T > 0].min())
    c1 = torch.empty(n, dtype=torch.int64, device="cuda")
    nnz1 = B.ot_kept_counts_range(p.handle, 0, n, 0, tiny, c1.data_ptr(), s)
    ref1 = torch.where(massful, (T >= tiny).sum(1), torch.zeros_like(c1))
    assert torch.equal(c1, ref1) and nnz1 == int(ref1.sum())
    # residuals: the materialized rows and columns summed in float64
    Td = T.double()
    r_ref = (Td.sum(1) - a.double()).abs().sum().item()
    c_ref = (Td.sum(0) - b.double()).abs().sum().item()
    r, c = p.marginal_residual()
    assert abs(r - r_ref) <= 1e-6 and abs(c - c_ref) <= 1e-6
    visited, total = p.row_pass_stats()
    assert 0 < visited < total
    p.close()


def test_row_pass_stats_without_screen(ot):
    """d > 3 has no screen: the statistics are (0, 0)."""
    import torch
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.random((300, 5), dtype=np.float32)).cuda()
    y = torch.from_numpy(rng.random((200, 5), dtype=np.float32)).cuda()
    a = torch.full((300,), 1 / 300, device="cuda")
    b = torch.full((200,), 1 / 200, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=0.1, n_iters=3)
    p.marginal_residual()
    assert p.row_pass_stats() == (0, 0)
    p.close()


def test_screened_range_rows_equal_the_materialized_plan(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    n, m = 2500, 2200
    x, y, a, b = _problem(3, n, m, 77)
    p = ot.sinkhorn(x, y, a, b, eps=1e-3, scale="max_cost", n_iters=30)
    s = torch.cuda.current_stream().cuda_stream
    lo, hi = 611, 1899
    T = p.materialize_rows(torch.arange(lo, hi, device="cuda"))
    massful = a[lo:hi] > 0
    rowmax = T.max(1).values
    thr, arg, nm = B.ot_min_row_range(p.handle, lo, hi, 0, s)
    assert thr == float(rowmax[massful].min()) and nm == int((~massful).sum())
    assert arg == lo + int(torch.nonzero(massful & (rowmax == rowmax[massful].min()))[0])
    cnt = torch.empty(hi - lo, dtype=torch.int64, device="cuda")
    nnz = B.ot_kept_counts_range(p.handle, lo, hi, 0, thr, cnt.data_ptr(), s)
    ref = torch.where(massful, (T >= thr).sum(1), torch.zeros_like(cnt))
    assert torch.equal(cnt, ref) and nnz == int(ref.sum())
    r, _ = B.ot_marginal_residual_range(p.handle, lo, hi, 0, 0, s)
    assert abs(r - (T.double().sum(1) - a[lo:hi].double()).abs().sum().item()) <= 1e-6
    p.close()


def test_screen_over_several_windows_of_chunks(ot):
    """More than 8192 chunks of 256 columns (m = 2.2e6): the pass screens them a
    window at a time; rows 100, so the materialized plan is the reference."""
    import torch
    n, m = 100, 2_200_000
    x, y, a, b = _problem(3, n, m, 91)
    p = ot.sinkhorn(x, y, a, b, eps=3e-4, scale="max_cost", n_iters=3)
    T = p.materialize_rows(torch.arange(n, device="cuda"))
    massful = a > 0
    rowmax = T.max(1).values
    thr_ref = rowmax[massful].min()
    mr = p.sparsify_min_row()
    visited, total = p.row_pass_stats()
    assert 0 < visited < total
    assert mr["thr"] == float(thr_ref)
    counts_ref = torch.where(massful, (T >= thr_ref).sum(1), torch.zeros_like(mr["counts"]))
    assert torch.equal(mr["counts"], counts_ref)
    r, _ = p.marginal_residual()
    assert abs(r - (T.double().sum(1) - a.double()).abs().sum().item()) <= 1e-6
    p.close()


def test_screen_at_workload_5_full_size(ot):
    """Workload 5 at n = m = 2e6, in the launch shape the bench times, after 5
    iterations: min_row's thr, argmin and counts against sampled materialized rows
    (exactly: the argmin row's maximum is thr, every sampled massful row keeps
    its count of entries >= thr), and the residual's part of single-row ranges
    against the rows' float64 sums."""
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w5()
    x, y, a, b = (torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in (w.x, w.y, w.a, w.b))
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=5)
    mr = p.sparsify_min_row(block_rows=w.block_rows)
    visited, total = p.row_pass_stats()
    assert 0 < visited < 0.6 * total                      # the screen skips most tiles here
    arg = mr["argmin"]
    rows = np.unique(np.concatenate([[arg], np.linspace(0, w.n - 1, 63).astype(np.int64)]))
    rt = torch.from_numpy(rows).cuda()
    T = p.materialize_rows(rt)
    rowmax = T.max(1).values
    k = int(np.nonzero(rows == arg)[0][0])
    assert float(rowmax[k]) == mr["thr"]
    assert bool((rowmax >= mr["thr"]).all())
    assert torch.equal((T >= mr["thr"]).sum(1), mr["counts"][rt])
    s = torch.cuda.current_stream().cuda_stream
    sums = T.double().sum(1).cpu().numpy()
    for t, i in enumerate(rows[:16]):
        part, _ = B.ot_marginal_residual_range(p.handle, int(i), int(i) + 1, 0, 0, s)
        assert abs(part - abs(sums[t] - float(w.a[i]))) <= 1e-6 * float(w.a[i])
    p.close()


@pytest.mark.parametrize("d", [5, 17, 50, 64])
def test_wide_passes_equal_the_materialized_plan(ot, d):
    """d > 3: the register-tiled row passes and the register-tiled materializer form
    every entry in the same order, so min_row's thr, argmin and counts equal those of
    the materialized rows bit for bit (ragged sizes: rows and columns not multiples
    of the 64-row / 64-column tiles)."""
    import torch
    rng = np.random.default_rng(100 + d)
    n, m = 333, 1201
    x = torch.from_numpy(rng.random((n, d), dtype=np.float32)).cuda()
    y = torch.from_numpy((rng.random((m, d)) * 1.2).astype(np.float32)).cuda()
    a = rng.random(n).astype(np.float32) + 0.2
    a[::41] = 0.0
    a = torch.from_numpy((a / a.sum()).astype(np.float32)).cuda()
    b = torch.full((m,), 1.0 / m, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=0.05, scale="mean", n_iters=6)
    T = p.materialize_rows(torch.arange(n, device="cuda"))
    Tsub = p.materialize_rows(torch.tensor([n - 1, 0, 200, 200], device="cuda"))
    assert torch.equal(Tsub, T[[n - 1, 0, 200, 200]])      # row lists in any order, repeats
    massful = a > 0
    rowmax = T.max(1).values
    thr = rowmax[massful].min()
    mr = p.sparsify_min_row(block_rows=100)
    assert mr["thr"] == float(thr)
    assert mr["argmin"] == int(torch.nonzero(massful & (rowmax == thr))[0])
    assert torch.equal(mr["counts"], torch.where(massful, (T >= thr).sum(1), torch.zeros_like(mr["counts"])))
    r, c = p.marginal_residual()
    Td = T.double()
    assert abs(r - (Td.sum(1) - a.double()).abs().sum().item()) <= 1e-6
    assert abs(c - (Td.sum(0) - b.double()).abs().sum().item()) <= 1e-6
    p.close()
