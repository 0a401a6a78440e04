"""Host-side fault injection (PIQ_FAULT) through the C ABI, on the CPU.

The library reads PIQ_FAULT at every compute call and, after checking the
arguments, returns the injected failure before touching a device, so these
calls never reach the GPU: the pointers below are host buffers that nothing
dereferences.  Callers' error handling (status codes, piq_last_cuda_error, the
binding's PiqError) is what this exercises; no GPU fault is made.
"""
import ctypes
import os

import numpy as np
import pytest

import post_int4_weight_gptq_b200 as piq
from post_int4_weight_gptq_b200 import build as piq_build


@pytest.fixture(scope="module")
def lib():
    piq_build.build()
    return piq.load_library()


@pytest.fixture
def fault(monkeypatch):
    def set_(value):
        if value is None:
            monkeypatch.delenv("PIQ_FAULT", raising=False)
        else:
            monkeypatch.setenv("PIQ_FAULT", value)
    yield set_
    monkeypatch.delenv("PIQ_FAULT", raising=False)


def _buf(nbytes):
    """A 256-byte aligned host address inside a numpy buffer (kept alive by the caller)."""
    raw = np.zeros(nbytes + 256, dtype=np.uint8)
    addr = raw.ctypes.data
    return raw, ctypes.c_void_p(addr + (-addr) % 256)


def _gptq(lib):
    out, inp, n = 64, 256, 512
    keep = [_buf(4 * out * inp), _buf(2 * n * inp), _buf(out * inp // 2), _buf(4 * out * 4),
            _buf(1 << 16)]
    W, X, q, s, ws = (k[1] for k in keep)
    err = ctypes.c_double(0.0)
    return lib.gptq_quantize_layer(W, out, inp, X, n, 4, 128, ctypes.c_float(0.01), 0, q, s,
                                   None, None, ctypes.byref(err), ws, 1 << 16, None)


def _awq(lib):
    out, inp, n = 64, 256, 512
    keep = [_buf(4 * out * inp), _buf(2 * n * inp), _buf(4 * inp), _buf(out * inp // 2),
            _buf(4 * out * 4), _buf(1 << 16)]
    W, X, sv, q, sc, ws = (k[1] for k in keep)
    grid = (ctypes.c_float * 2)(0.0, 0.5)
    best = ctypes.c_float(0.0)
    errs = (ctypes.c_double * 2)()
    return lib.awq_search_layer(W, out, inp, X, n, 4, 128, grid, 2, ctypes.byref(best), sv, q,
                                sc, errs, ws, 1 << 16, None)


def _factor(lib):
    keep = [_buf(4 * 64 * 64), _buf(4 * 64 * 64), _buf(1 << 16)]
    H, U, ws = (k[1] for k in keep)
    lam = ctypes.c_double(0.0)
    return lib.piq_upper_factor(H, 64, ctypes.c_float(0.01), None, U, ctypes.byref(lam), ws,
                                1 << 16, None)


def _factor_noalloc(lib):
    keep = [_buf(4 * 64 * 64), _buf(4 * 64 * 64)]
    H, U = (k[1] for k in keep)
    lam = ctypes.c_double(0.0)
    return lib.piq_upper_factor_noalloc(H, 64, ctypes.c_float(0.01), None, U,
                                        ctypes.byref(lam), None)


CALLS = [_gptq, _awq, _factor, _factor_noalloc]


@pytest.mark.parametrize("call", CALLS)
@pytest.mark.parametrize("value,status", [("notpd", piq.PIQ_ERR_NOT_PD),
                                          ("timeout", piq.PIQ_ERR_TIMEOUT),
                                          ("oom", piq.PIQ_ERR_CUDA)])
def test_injected_status(lib, fault, call, value, status):
    fault(value)
    assert call(lib) == status
    if value == "oom":
        assert "cudaErrorMemoryAllocation" in piq.last_cuda_error()
        assert "PIQ_FAULT" in piq.last_cuda_error()


@pytest.mark.parametrize("call", CALLS)
def test_argument_errors_come_before_injection(lib, fault, call):
    # an invalid argument is reported as such even with a fault injected
    fault("notpd")
    keep = _buf(4096)
    lam = ctypes.c_double(0.0)
    rc = lib.piq_upper_factor(None, 64, ctypes.c_float(0.01), None, keep[1], ctypes.byref(lam),
                              keep[1], 4096, None)
    assert rc == piq.PIQ_ERR_INVALID_ARG


@pytest.mark.parametrize("value", [None, "", "something-else"])
def test_no_injection_reaches_the_device_check(lib, fault, value):
    # without a recognised fault the call goes on to look for a B200; on this
    # CPU-only machine that fails with a device or CUDA status, never with an
    # injected one
    if os.environ.get("CUDA_VISIBLE_DEVICES", None) != "" and _has_gpu():
        pytest.skip("a GPU is present: the call would run for real")
    fault(value)
    rc = _factor(lib)
    assert rc in (piq.PIQ_ERR_CUDA, piq.PIQ_ERR_UNSUPPORTED_DEVICE)


def _has_gpu():
    import torch
    return torch.cuda.is_available()


def test_wait_selftest_checks_its_arguments(lib):
    keep = _buf(256)
    where = ctypes.c_int(0)
    assert lib.piq_wait_selftest(10, ctypes.byref(where), keep[1], 256, None) == \
        piq.PIQ_ERR_INVALID_ARG
    assert lib.piq_wait_selftest(10**11, ctypes.byref(where), keep[1], 256, None) == \
        piq.PIQ_ERR_INVALID_ARG
    assert lib.piq_wait_selftest(10**6, ctypes.byref(where), None, 256, None) == \
        piq.PIQ_ERR_INVALID_ARG
    assert lib.piq_wait_selftest(10**6, ctypes.byref(where), keep[1], 64, None) == \
        piq.PIQ_ERR_WORKSPACE_TOO_SMALL
