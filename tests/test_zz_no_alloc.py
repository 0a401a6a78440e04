"""piq_upper_factor_noalloc: the damping + upper-factor step for callers that
must not allocate device memory, checked against piq_upper_factor (which takes
a caller workspace).  Named to be collected after every other test file.

The allocation-free entry keeps its scratch in one fixed region inside the
library, shared by every call on a device; these tests call it several times in
a row, with different sizes, to show that what a previous call left there does
not leak into the next result.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from tests.parity import REL_TOL
from workloads import make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _noalloc(H, damp, perm):
    """Straight through the C ABI: no workspace argument exists."""
    lib = piq.load_library()
    U = torch.empty_like(H)
    lam = ctypes.c_double(0.0)
    rc = lib.piq_upper_factor_noalloc(
        ctypes.c_void_p(H.data_ptr()), H.shape[0], ctypes.c_float(damp),
        None if perm is None else ctypes.c_void_p(perm.data_ptr()),
        ctypes.c_void_p(U.data_ptr()), ctypes.byref(lam),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, U, lam.value


def _layer_hessian(inp, act, seed):
    spec = small_spec(8, inp, 4 * inp, seed=seed, sigma_ln=0.8)
    Hx = O.hessian_ref(make_x_bits(spec))
    H = torch.from_numpy(Hx.astype(np.float32)).cuda()
    perm = None
    if act:
        perm = torch.from_numpy(O.act_order_perm_ref(Hx).astype(np.int32)).cuda()
    return H, perm


def _assert_close(U_a, U_b):
    scale = U_b.abs().amax(dim=1, keepdim=True).clamp_min(1e-30)
    assert float(((U_a - U_b).abs() / scale).max()) < REL_TOL


def test_calls_in_a_row_match_the_workspace_entry():
    first = None
    for inp, act, seed in ((512, False, 1), (136, True, 2), (512, False, 1)):
        H, perm = _layer_hessian(inp, act, seed)
        rc, U, lam = _noalloc(H, 0.01, perm)
        assert rc == piq.PIQ_OK, piq.status_string(rc)
        U_ref, lam_ref = piq.upper_factor(H, 0.01, perm=perm)
        _assert_close(U, U_ref)
        assert abs(lam - lam_ref) <= 1e-6 * abs(lam_ref)
        if first is None:
            first = U
        elif inp == first.shape[0]:
            _assert_close(U, first)  # the same input again, after a different size


def test_matches_the_oracle():
    # the same U the float64 oracle forms from the listing (cholesky(inv(H_d)).T),
    # to the accuracy of the workspace entry's FP32 factorization
    for inp, act, seed in ((512, False, 3), (264, True, 4)):
        spec = small_spec(8, inp, 4 * inp, seed=seed, sigma_ln=0.8)
        Hx = O.hessian_ref(make_x_bits(spec))
        perm, Ux, lam_x = O.gptq_prepare_ref(Hx, 0.01, act)
        H = torch.from_numpy(Hx.astype(np.float32)).cuda()
        pg = torch.from_numpy(perm.astype(np.int32)).cuda() if act else None
        rc, U, lam = _noalloc(H, 0.01, pg)
        assert rc == piq.PIQ_OK, piq.status_string(rc)
        U = U.cpu().numpy().astype(np.float64)
        assert abs(lam - lam_x) <= 1e-5 * lam_x
        assert np.count_nonzero(np.tril(U, -1)) == 0
        assert (np.abs(U - Ux) / np.abs(Ux).max(axis=1, keepdims=True)).max() < 2e-5


def test_larger_than_the_region_is_rejected():
    H = torch.zeros(piq.NOALLOC_MAX_IN + 8, piq.NOALLOC_MAX_IN + 8, device="cuda")
    rc, _, _ = _noalloc(H, 0.01, None)
    assert rc == piq.PIQ_ERR_INVALID_ARG
