"""The allocation-free residual entry point, checked against the plan-based one.

ot_marginal_residual_noalloc is for callers that cannot allocate device memory
when they need a residual (their device memory belongs to another allocator, or
a cudaMalloc would stall their other streams). It must return the same two sums
as ot_marginal_residual on the same potentials. This file is collected last so
that a run stopping at the first failure has already run every other test; it
also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import helpers as H

pytestmark = pytest.mark.gpu


def _problem(seed, n, m, d, scale):
    from log_domain_sinkhorn_online_b200.workloads import Workload
    rng = np.random.default_rng(seed)
    x = rng.random((n, d)).astype(np.float32)
    y = (rng.random((m, d)) * 0.9 + 0.05).astype(np.float32)
    a = rng.random(n) + 0.2
    b = rng.random(m) + 0.2
    a[::97] = 0.0  # a few massless rows
    return Workload("noalloc", x, y, (a / a.sum()).astype(np.float32), (b / b.sum()).astype(np.float32),
                    eps=0.02, scale=scale, n_iters=25)


def _via_plan_and_noalloc(pkg, B, w):
    import torch
    x, y, a, b = H.to_dev(w)
    plan = pkg.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=w.n_iters)
    want = plan.marginal_residual()
    st, r, c = B.ot_marginal_residual_noalloc(
        x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), plan.f.data_ptr(), plan.g.data_ptr(),
        w.n, w.m, w.d, plan.info.eps, plan.info.inv_scale_cost, torch.cuda.current_stream().cuda_stream)
    plan.close()
    return st, (r, c), want


def test_noalloc_residual_matches_plan_residual_twice_in_a_row():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import log_domain_sinkhorn_online_b200 as pkg
    from log_domain_sinkhorn_online_b200 import _binding as B
    # calls in a row on different problems: none may see the previous one's
    # leftovers in the shared scratch; the fourth fills the scratch exactly
    # (OT_NOALLOC_MAX_POINTS rows: every partial slot, the results right after),
    # the fifth runs the generic kernel at the largest d
    for w in (_problem(1, 3001, 2777, 3, "mean"), _problem(2, 1500, 4100, 2, "none"),
              _problem(3, 700, 650, 17, "max_cost"), _problem(4, B.OT_NOALLOC_MAX_POINTS, 64, 3, "mean"),
              _problem(5, 900, 800, 64, "none")):
        st, got, want = _via_plan_and_noalloc(pkg, B, w)
        assert st == 0
        assert abs(got[0] - want[0]) <= H.RES_TOL, (got, want)
        assert abs(got[1] - want[1]) <= H.RES_TOL, (got, want)


def test_noalloc_rejects_sizes_above_its_maximum():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from log_domain_sinkhorn_online_b200 import _binding as B
    L = B.lib()
    r = ctypes.c_double()
    big = B.OT_NOALLOC_MAX_POINTS + 1
    st = L.ot_marginal_residual_noalloc(16, 16, 16, 16, 16, 16, big, 10, 3, 0.1, 1.0,
                                        ctypes.byref(r), None, None)
    assert st == B.OT_ERR_UNSUPPORTED
    assert "at most" in B.ot_last_error_string()
