"""GPU checks of the C-ABI conveniences around the solve (-m gpu):
 - the optional residual history (ot_options.resid_history): entry k - 1 is the
   in-loop ||T1 - a||_1 after iteration k, bit-identical to the final residual
   a shorter solve reports, NaN where no f-update measured one, and close to the
   float64 oracle's residual along the oracle's own trajectory on a
   well-conditioned problem;
 - ot_sinkhorn_pointcloud_host (host arrays in, host potentials out): the same
   potentials, bit for bit, as the device entry point, and a plan that owns its
   device copies and serves rows;
 - a plan destroyed while another device is current returns its workspace to
   its own device (checked through the library's behaviour on one device: the
   destroy under a changed current device is not available with one GPU, so the
   plan is destroyed from a second host thread, which starts with device 0).
"""
import threading

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


def _w(n=1500, m=1300):
    from log_domain_sinkhorn_online_b200 import workloads
    return workloads.w2(n=n, m=m)


def test_residual_history_matches_shorter_solves(ot):
    import torch
    w = _w()
    x, y, a, b = H.to_dev(w)
    hist = torch.full((40,), -1.0, dtype=torch.float64, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=30, resid_history=hist)
    h = hist.cpu().numpy()
    assert p.info.iterations == 30
    assert h[29] == p.info.residual           # the final f-update's measurement
    assert np.isfinite(h[:30]).all() and np.isnan(h[30:]).all()
    p.close()
    for k in (1, 7, 16, 17):
        q = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=k)
        assert q.info.residual == h[k - 1], (k, q.info.residual, h[k - 1])
        q.close()


def test_residual_history_device_loop_and_launches_agree(ot):
    import torch
    w = _w(900, 1100)
    x, y, a, b = H.to_dev(w)
    hs = []
    for loop in (1, 0):
        hist = torch.empty(25, dtype=torch.float64, device="cuda")
        ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=25, device_loop=loop,
                    resid_history=hist).close()
        hs.append(hist.cpu().numpy())
    assert np.isfinite(hs[0]).all()
    np.testing.assert_allclose(hs[0], hs[1], rtol=1e-5, atol=1e-9)


def test_residual_history_against_the_oracle_trajectory(ot, orc):
    """On a well-conditioned problem the GPU's in-loop residual after iteration k
    stays within 1e-5 of the oracle's residual after its own iteration k."""
    import torch
    from log_domain_sinkhorn_online_b200 import workloads
    w = workloads.w1()
    x, y, a, b = H.to_dev(w)
    K = 40
    hist = torch.empty(K, dtype=torch.float64, device="cuda")
    ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=K, resid_history=hist).close()
    h = hist.cpu().numpy()
    c = orc.inv_scale_cost(w.x, w.y, w.scale)
    f, g = np.zeros(w.n), np.zeros(w.m)
    for k in range(K):
        f, g, _, r = orc.sinkhorn(w.x, w.y, w.a, w.b, c, w.eps, 1, f0=f, g0=g)
        assert abs(h[k] - r) <= 1e-5, (k, h[k], r)


def test_residual_history_annealing_marks_stage_ends(ot):
    import torch
    w = _w(700, 800)
    x, y, a, b = H.to_dev(w)
    hist = torch.empty(3 * 5 + 4, dtype=torch.float64, device="cuda")
    # eps_init = 4 eps, decay 0.5: stages at 4, 2, 1 (x eps), 5 + 5 + 4 iterations
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=4, eps_init=4 * w.eps, eps_decay=0.5,
                    iters_per_stage=5, resid_history=hist)
    h = hist.cpu().numpy()
    assert p.info.stages == 3 and p.info.iterations == 14
    assert np.isnan(h[4]) and np.isnan(h[9])       # last iteration of the first two stages
    assert np.isfinite(np.delete(h[:14], [4, 9])).all()
    assert h[13] == p.info.residual and np.isnan(h[14:]).all()
    p.close()


def test_host_entry_point_matches_the_device_one(ot):
    import torch
    from log_domain_sinkhorn_online_b200 import _binding as B
    w = _w(1200, 1000)
    x, y, a, b = H.to_dev(w)
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=20)
    fd, gd = p.f.cpu().numpy(), p.g.cpu().numpy()
    rows = torch.arange(0, 1200, 37, device="cuda")
    Td = p.materialize_rows(rows).cpu().numpy()
    p.close()
    hx, hy, ha, hb = (np.ascontiguousarray(v) for v in (w.x, w.y, w.a, w.b))
    for pinned in (False, True):
        f = torch.zeros(1200, dtype=torch.float32)
        g = torch.zeros(1000, dtype=torch.float32)
        src = [torch.from_numpy(v) for v in (hx, hy, ha, hb)]
        if pinned:
            src = [t.pin_memory() for t in src]
            f, g = f.pin_memory(), g.pin_memory()
        st, plan, info = B.ot_sinkhorn_pointcloud_host(
            *(t.data_ptr() for t in src), 1200, 1000, 3, w.eps, B.OT_SCALE_MEAN, 20, 0.0,
            f.data_ptr(), g.data_ptr(), torch.cuda.current_stream().cuda_stream, None, want_plan=pinned)
        assert st == B.OT_OK and info.iterations == 20
        np.testing.assert_array_equal(f.numpy(), fd)
        np.testing.assert_array_equal(g.numpy(), gd)
        if plan:
            out = torch.empty((rows.numel(), 1000), device="cuda")
            B.ot_materialize_rows(plan, rows.data_ptr(), rows.numel(), out.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
            np.testing.assert_array_equal(out.cpu().numpy(), Td)
            B.ot_plan_destroy(plan)


def test_plan_destroyed_from_another_thread(ot):
    """The plan's workspace and stream go back to the plan's own device even when
    the destroying thread has not selected it; a later plan then reuses them."""
    import torch
    w = _w(800, 900)
    x, y, a, b = H.to_dev(w)
    ref = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=10)
    fr = ref.f.cpu().numpy()
    ref.close()
    for _ in range(3):
        p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=10)
        t = threading.Thread(target=p.close)
        t.start()
        t.join()
        q = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=10)
        np.testing.assert_array_equal(q.f.cpu().numpy(), fr)
        q.close()
    torch.cuda.synchronize()


def test_residual_history_with_tol_and_block_sparse(ot):
    import torch
    w = _w(2000, 1800)
    x, y, a, b = H.to_dev(w)
    # a tolerance met inside the run: the history stops at the returned state
    hist = torch.empty(400, dtype=torch.float64, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=0.05, scale=w.scale, n_iters=400, tol=1e-4, resid_history=hist)
    h = hist.cpu().numpy()
    k = p.info.iterations
    assert p.info.converged == 1 and 1 <= k < 400
    assert h[k - 1] == p.info.residual and h[k - 1] <= 1e-4 and h[k - 2] > 1e-4
    assert np.isnan(h[k + 1:]).all()
    p.close()
    # block-sparse iterations record the admitted plan's residual after every iteration
    hist = torch.empty(6, dtype=torch.float64, device="cuda")
    p = ot.sinkhorn(x, y, a, b, eps=w.eps, scale=w.scale, n_iters=6, block_sparse=True, sparse_delta=1e-7,
                    sparse_dense_frac=1.0, resid_history=hist)
    h = hist.cpu().numpy()
    assert np.isfinite(h).all() and h[5] == p.info.residual
    p.close()
