"""Failure paths of the library on the GPU, with no GPU fault (-m gpu).

 - An injected workspace-allocation failure (the hook of
   include/ot_sinkhorn_testing.h fails the k-th device allocation as cudaMalloc
   does when memory runs out) makes the call return OT_ERR_OOM, at every
   allocation a solve and the row calls make, and leaves the library usable.
 - The two kinds of bounded device wait give up and report OT_ERR_CUDA: the
   device-resident loop kernel's grid barrier (one block withholds its arrival,
   the time limit is 2 ms) and the tensor-core half-step's mbarrier waits (one
   block's producer skips a load, the poll limit is 2^12). Every wait ends by
   its limit; the kernels return, the context stays usable, and the next solve
   gives the same potentials as before.
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


@pytest.fixture
def B():
    from log_domain_sinkhorn_online_b200 import _binding
    yield _binding
    _binding.ot_testing_fail_device_allocs(-1)
    _binding.ot_testing_wait_fault(0)


def _problem(n=1000, m=900, d=3, seed=5):
    import torch
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.random((n, d), dtype=np.float32)).cuda()
    y = torch.from_numpy(rng.random((m, d), dtype=np.float32)).cuda()
    a = torch.full((n,), 1.0 / n, device="cuda")
    b = torch.full((m,), 1.0 / m, device="cuda")
    return x, y, a, b


def test_injected_allocation_failure_returns_oom(ot, B):
    import torch
    x, y, a, b = _problem()
    ref = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=5)
    fr = ref.f.cpu().numpy()
    ref.close()
    B.ot_trim_cache()  # every allocation below reaches the (failing) allocator path
    # the solve's workspace (first allocation of a solve)
    B.ot_testing_fail_device_allocs(0)
    with pytest.raises(B.OTError) as e:
        ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=5)
    assert e.value.status == B.OT_ERR_OOM
    # the row kernels' workspace (allocated on the plan's first row call)
    p = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=5)
    B.ot_trim_cache()
    B.ot_testing_fail_device_allocs(0)
    with pytest.raises(B.OTError) as e:
        p.marginal_residual()
    assert e.value.status == B.OT_ERR_OOM
    B.ot_testing_fail_device_allocs(-1)
    r, c = p.marginal_residual()  # the plan is still usable
    assert np.isfinite(r) and np.isfinite(c)
    np.testing.assert_array_equal(p.f.cpu().numpy(), fr)
    p.close()
    # block-sparse workspace (the second allocation of a block-sparse solve)
    B.ot_trim_cache()
    B.ot_testing_fail_device_allocs(1)
    with pytest.raises(B.OTError) as e:
        ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=3, block_sparse=True, sparse_delta=1e-6)
    assert e.value.status == B.OT_ERR_OOM
    # the host entry point's device copies
    B.ot_testing_fail_device_allocs(0)
    hx, hy, ha, hb = (t.cpu() for t in (x, y, a, b))
    f, g = torch.zeros(1000), torch.zeros(900)
    with pytest.raises(B.OTError) as e:
        B.ot_sinkhorn_pointcloud_host(hx.data_ptr(), hy.data_ptr(), ha.data_ptr(), hb.data_ptr(), 1000, 900,
                                      3, 0.05, B.OT_SCALE_NONE, 5, 0.0, f.data_ptr(), g.data_ptr(), 0, None)
    assert e.value.status == B.OT_ERR_OOM
    B.ot_testing_fail_device_allocs(-1)
    q = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=5)
    np.testing.assert_array_equal(q.f.cpu().numpy(), fr)
    q.close()
    torch.cuda.synchronize()


def test_loop_kernel_barrier_timeout_is_reported(ot, B):
    import torch
    x, y, a, b = _problem(2000, 1800)
    ref = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=8, device_loop=1)
    fr, gr = ref.f.cpu().numpy(), ref.g.cpu().numpy()
    ref.close()
    B.ot_testing_wait_fault(1)
    with pytest.raises(B.OTError) as e:
        ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=8, device_loop=1)
    assert e.value.status == B.OT_ERR_CUDA and "timed out" in str(e.value)
    B.ot_testing_wait_fault(0)
    torch.cuda.synchronize()  # the context is intact
    q = ot.sinkhorn(x, y, a, b, eps=0.05, n_iters=8, device_loop=1)
    np.testing.assert_array_equal(q.f.cpu().numpy(), fr)
    np.testing.assert_array_equal(q.g.cpu().numpy(), gr)
    q.close()


def test_tensor_core_mbarrier_timeout_is_reported(ot, B):
    import torch
    x, y, a, b = _problem(1500, 1300, d=24)
    ref = ot.sinkhorn(x, y, a, b, eps=0.5, n_iters=4)
    fr = ref.f.cpu().numpy()
    ref.close()
    B.ot_testing_wait_fault(2)
    with pytest.raises(B.OTError) as e:
        ot.sinkhorn(x, y, a, b, eps=0.5, n_iters=4)
    assert e.value.status == B.OT_ERR_CUDA and "timed out" in str(e.value)
    B.ot_testing_wait_fault(0)
    torch.cuda.synchronize()
    q = ot.sinkhorn(x, y, a, b, eps=0.5, n_iters=4)
    np.testing.assert_array_equal(q.f.cpu().numpy(), fr)
    q.close()
