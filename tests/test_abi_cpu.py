"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments (host-side validation) before any
CUDA call. Valid calls on a machine without a GPU fail loudly (no fallback)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


@pytest.fixture(scope="module")
def B():
    from log_domain_sinkhorn_online_b200 import build, _binding
    build.build()
    _binding.lib()
    return _binding


def _declared():
    txt = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"^OT_API [^(]*?\b(ot_\w+)\(", txt, re.M)))


def test_header_declares_the_binding_names(B):
    assert _declared() == sorted(B.EXPORTED)


def test_library_exports_every_declared_symbol(B):
    L = B.lib()
    for name in _declared():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {B._LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (ot_\w+)$", out, re.M)))
    assert exported == _declared()


def test_version_and_defaults(B):
    assert B.ot_version() == 4
    o = B.ot_options_default()
    assert (o.warm_start, o.check_every, o.use_graphs, o.iters_per_stage) == (0, 16, 1, 20)
    assert (o.scale_value, o.eps_init, o.eps_decay) == (1.0, 0.0, 0.7)
    assert (o.timing, o.col_splits, o.rows_per_thread, o.tensor_cores, o.device_loop) == (0, 0, 0, 1, -1)
    assert (o.block_sparse, o.sparse_block, o.sparse_verify, o.sparse_delta, o.sparse_dense_frac) == \
        (0, 0, 1, 0.0, 0.5)


def test_struct_sizes_match_header_layout(B):
    assert ctypes.sizeof(B.OtOptions) == 4 * 4 + 3 * 8 + 6 * 4 + 4 * 4 + 2 * 8 + 4 * 8
    assert ctypes.sizeof(B.OtInfo) == 4 * 4 + 3 * 8 + 4 * 8 + 8 + 6 * 8 + 8 + 3 * 8


FAKE = 0x1000  # never dereferenced: validation fails first


def _call(B, **kw):
    args = dict(x=FAKE, y=FAKE, a=FAKE, b=FAKE, n=10, m=10, d=3, eps=0.1, scale_cost=0, n_iters=5,
                tol=0.0, f=FAKE, g=FAKE, stream=None, opt=None)
    args.update(kw)
    opt = args.pop("opt")
    plan = ctypes.c_void_p()
    return B.lib().ot_sinkhorn_pointcloud(*args.values(), ctypes.byref(opt) if opt else None,
                                          ctypes.byref(plan), None), plan.value


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), -1), (dict(g=None), -1), (dict(n=0), -1), (dict(m=-3), -1),
    (dict(d=0), -1), (dict(d=65), -6), (dict(eps=0.0), -1), (dict(eps=float("nan")), -1),
    (dict(eps=float("inf")), -1), (dict(scale_cost=7), -1), (dict(n_iters=-1), -1),
    (dict(n_iters=0), -1), (dict(n=2 ** 31), -2),
])
def test_invalid_arguments_are_rejected(B, kw, code):
    st, plan = _call(B, **kw)
    assert st == code and plan is None
    assert B.ot_last_error_string() != "no error"


def test_option_validation(B):
    o = B.ot_options_default()
    o.check_every = 0
    assert _call(B, opt=o)[0] == -1
    o = B.ot_options_default()
    o.eps_init, o.eps_decay = 1.0, 1.5
    assert _call(B, opt=o)[0] == -1
    o = B.ot_options_default()
    assert _call(B, scale_cost=3, opt=o)[0] in (0, -3)  # 1.0 is valid: the call reaches the device
    o.scale_value = -2.0
    assert _call(B, scale_cost=3, opt=o)[0] == -1


def test_block_sparse_options_are_validated(B):
    def sp(**kw):
        o = B.ot_options_default()
        o.block_sparse = 1
        for k, v in kw.items():
            setattr(o, k, v)
        return o
    assert _call(B, d=5, tol=1e-2, opt=sp())[0] == -6          # d > 3 is not supported
    assert _call(B, tol=1e-2, opt=sp(sparse_block=64))[0] == -1
    assert _call(B, tol=0.0, opt=sp())[0] == -1                  # delta from tol needs tol > 0
    assert _call(B, tol=0.0, opt=sp(sparse_delta=-1.0))[0] == -1
    assert _call(B, tol=1e-2, opt=sp(sparse_dense_frac=1.5))[0] == -1
    assert _call(B, tol=0.0, opt=sp(sparse_delta=1e-6))[0] in (0, -3)  # valid: reaches the device


def test_row_calls_reject_null_plan(B):
    L = B.lib()
    assert L.ot_materialize_rows(None, FAKE, 1, FAKE, None) == -1
    assert L.ot_marginal_residual(None, None, None, None) == -1
    assert L.ot_sparsify_min_row(None, 0, None, None, None, None, None, None) == -1
    assert L.ot_sparsify_csr(None, 0, 0.5, FAKE, FAKE, FAKE, 1, None, None) == -1
    assert L.ot_marginal_residual_range(None, 0, 1, 0, 1, None, None, None) == -1
    assert L.ot_min_row_range(None, 0, 1, 0, None, None, None, None) == -1
    assert L.ot_kept_counts_range(None, 0, 1, 0, 0.5, None, None, None) == -1
    assert L.ot_row_pass_stats(None, None, None) == -1
    L.ot_plan_destroy(None)  # no-op


def test_lowrank_rows_validate_on_the_host(B):
    L = B.lib()
    # rank outside [1, 128] is unsupported, bad sizes / eps are invalid, k = 0 is a no-op
    assert L.ot_materialize_rows_lowrank(FAKE, FAKE, FAKE, 4, 5, 0, FAKE, 1, FAKE, None) == -6
    assert L.ot_materialize_rows_lowrank(FAKE, FAKE, FAKE, 4, 5, 129, FAKE, 1, FAKE, None) == -6
    assert L.ot_materialize_rows_lowrank(FAKE, FAKE, FAKE, 0, 5, 3, FAKE, 1, FAKE, None) == -1
    assert L.ot_materialize_rows_lowrank(None, FAKE, FAKE, 4, 5, 3, FAKE, 1, FAKE, None) == -1
    assert L.ot_materialize_rows_lowrank(FAKE, FAKE, FAKE, 4, 5, 3, FAKE, 0, FAKE, None) == 0
    assert L.ot_materialize_rows_lrcost(FAKE, FAKE, FAKE, FAKE, 4, 5, 3, 0.0, 1.0, 0.0, FAKE, 1, FAKE,
                                        None) == -1
    assert L.ot_materialize_rows_lrcost(FAKE, FAKE, None, FAKE, 4, 5, 3, 0.0, 1.0, 0.1, FAKE, 1, FAKE,
                                        None) == -1


def test_valid_call_without_gpu_fails_loudly(B):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st, plan = _call(B)
    assert st == -3 and plan is None


def test_residual_history_needs_an_array(B):
    o = B.ot_options_default()
    o.resid_history_len = 5  # no array
    assert _call(B, opt=o)[0] == B.OT_ERR_INVALID_ARG
    o.resid_history_len = -1
    assert _call(B, opt=o)[0] == B.OT_ERR_INVALID_ARG
    o = B.ot_options_default()
    o.sparse_mask_out = FAKE  # a mask needs block-sparse iterations
    o.sparse_mask_len = 100
    assert _call(B, opt=o)[0] == B.OT_ERR_INVALID_ARG


def test_host_entry_point_validates_before_touching_memory(B):
    L = B.lib()
    for n, d, code in ((0, 3, B.OT_ERR_INVALID_ARG), (4, 0, B.OT_ERR_INVALID_ARG),
                       (4, 65, B.OT_ERR_UNSUPPORTED), (1 << 31, 3, B.OT_ERR_OVERFLOW)):
        st = L.ot_sinkhorn_pointcloud_host(FAKE, FAKE, FAKE, FAKE, n, 4, d, 0.1, 0, 1, 0.0, FAKE, FAKE,
                                           None, None, None, None)
        assert st == code, (n, d, st)
    st = L.ot_sinkhorn_pointcloud_host(None, FAKE, FAKE, FAKE, 4, 4, 3, 0.1, 0, 1, 0.0, FAKE, FAKE,
                                       None, None, None, None)
    assert st == B.OT_ERR_INVALID_ARG
