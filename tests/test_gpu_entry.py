"""The plan-entry float path at the ends of its range (-m gpu).

Every row call (materializer, residual, min_row, sparsify) evaluates
T_ij = exp((f_i + g_j - C_ij)/eps) through one device function (moscot PR #846,
"Behavioural changes": one float path for threshold and values). Its range
reduction keeps the base-2 exponent e2 on a float64 grid of 2^-23, returns 0
below e2 = -126 and saturates to +inf from e2 = 128 on; these tests pin what that
means for a caller, against exp() evaluated in float64 on the host:
 - normal results (2^-126 <= T < 2^128) within 1e-6 relative (the bar of the
   parity tests is 1e-5);
 - T = 0 below 2^-126 (entries under the smallest normal float are flushed) and
   for a potential of -inf;
 - T = +inf from 2^128 on.
The cost is zero (every point at the origin, d = 1, eps = 1), so e2 =
(f_0 + g_j) log2(e) sweeps the range through the column potentials.
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


def _rows_at(ot, g, f0=0.0, eps=1.0):
    import torch
    m = g.size
    x = torch.zeros((1, 1), device="cuda")
    y = torch.zeros((m, 1), device="cuda")
    a = torch.ones(1, device="cuda")
    b = torch.full((m,), 1.0 / m, device="cuda")
    f = torch.tensor([f0], dtype=torch.float32, device="cuda")
    gt = torch.from_numpy(g.astype(np.float32)).cuda()
    p = ot.sinkhorn(x, y, a, b, eps=eps, n_iters=0, warm_start=True, f=f, g=gt)
    T = p.materialize_rows(torch.zeros(1, dtype=torch.int64, device="cuda")).cpu().numpy()[0]
    p.close()
    return T.astype(np.float64)


def test_entry_across_the_float_range(ot):
    e2 = np.concatenate([np.linspace(-220.0, 140.0, 60001),
                         [-126.01, -125.99, 63.999, 64.0, 127.99, 128.01]])
    g = (e2 * np.log(2.0)).astype(np.float32)            # f_0 = 0, eps = 1
    T = _rows_at(ot, g)
    ref = np.exp(g.astype(np.float64))                   # the exact entry of the float32 inputs
    tiny, huge = 2.0 ** -126, 2.0 ** 128
    normal = (ref >= tiny * (1 + 1e-6)) & (ref < huge * (1 - 1e-6))
    rel = np.abs(T[normal] - ref[normal]) / ref[normal]
    assert rel.max() <= 1e-6, rel.max()
    assert np.all(T[ref < tiny * (1 - 1e-6)] == 0.0)
    assert np.all(np.isposinf(T[ref >= huge * (1 + 1e-6)]))
    assert np.all(T >= 0.0) and not np.isnan(T).any()


def test_massless_potential_gives_zero(ot):
    g = np.array([0.0, -np.inf, 1.0, -np.inf], dtype=np.float32)
    T = _rows_at(ot, g)
    assert T[1] == 0.0 and T[3] == 0.0
    assert abs(T[0] - 1.0) <= 1e-6 and abs(T[2] - np.e) <= 1e-6 * np.e
    T = _rows_at(ot, np.zeros(8, np.float32), f0=-np.inf)
    assert np.all(T == 0.0)
