"""The C-ABI library builds, loads and exports what include/piq.h declares.
No GPU: only calls that return before touching a device are made."""
import ctypes
import os
import re

import pytest

import post_int4_weight_gptq_b200 as piq
from post_int4_weight_gptq_b200 import build as piq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    piq_build.build()
    return piq.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "piq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "gptq_quantize_layer" in names and "awq_search_layer" in names
    for name in names:
        assert hasattr(lib, name), name
    # and the binding covers exactly the declared functions, in order
    assert list(piq.SIGNATURES) == names


def test_status_strings(lib):
    for code in range(-6, 1):
        assert piq.status_string(code) != "unknown status"
    assert piq.status_string(-99) == "unknown status"


def test_hessian_bytes_printed_on_the_page(lib):
    # "GPTQ versus AWQ objectives", sizing block: 8,192^2 x 4 B = 268 MB and
    # 28,672^2 x 4 B = 3.29 GB.
    assert piq.hessian_bytes(8192) == 268_435_456
    assert piq.hessian_bytes(28672) == 3_288_334_336


def test_workspace_queries_are_monotone(lib):
    a = piq.gptq_workspace_bytes(256, 512, 2048)
    b = piq.gptq_workspace_bytes(512, 512, 2048)
    c = piq.gptq_workspace_bytes(256, 1024, 2048)
    assert 0 < a < b and a < c
    hb = piq.hessian_bytes(512)
    assert a >= 2 * hb  # H (then U) and the factor's working copy
    assert piq.gptq_workspace_bytes(256, 512, 2048, act_order=True) >= a
    assert piq.awq_workspace_bytes(256, 512, 2048, 20) > piq.awq_workspace_bytes(256, 512, 2048, 1)


def test_bad_arguments_rejected_before_any_device_work(lib):
    null = None
    err = ctypes.c_double()
    # bits out of range, in not a multiple of 8, g < 1, null pointers
    for bits, inp, g in ((5, 512, 128), (4, 500, 128), (4, 512, 0), (1, 512, 128)):
        rc = lib.gptq_quantize_layer(null, 16, inp, null, 64, bits, g, 0.01, 0, null, null, null,
                                     null, ctypes.byref(err), null, 0, null)
        assert rc == piq.PIQ_ERR_INVALID_ARG
    rc = lib.piq_hessian(null, 10, 64, null, 0, null)
    assert rc == piq.PIQ_ERR_INVALID_ARG
    out = ctypes.c_size_t()
    assert lib.piq_awq_workspace_bytes(16, 64, 64, 65, ctypes.byref(out)) == piq.PIQ_ERR_INVALID_ARG
    assert lib.piq_awq_workspace_bytes(16, 64, 64, 0, ctypes.byref(out)) == piq.PIQ_ERR_INVALID_ARG


def test_library_is_sm100a_only(lib):
    # every kernel was compiled for sm_100a alone
    assert "-gencode" in piq_build.ARCH and "arch=compute_100a,code=sm_100a" in piq_build.ARCH


def test_widened_entries_reject_missing_buffers(lib):
    # the zero-point buffer of the asymmetric entry and the channel scales of
    # the composed entry are required; a misaligned s is refused (the pointer
    # is only checked, never read)
    null = None
    err = ctypes.c_double()
    rc = lib.gptq_quantize_layer_asym(null, 16, 64, null, 64, 4, 32, 0.01, 0, null, null, null,
                                      null, null, ctypes.byref(err), null, 0, null)
    assert rc == piq.PIQ_ERR_INVALID_ARG
    for s_ptr in (None, ctypes.c_void_p(4)):
        rc = lib.awq_gptq_quantize_layer(null, 16, 64, null, 64, s_ptr, 4, 32, 0.01, 0, null,
                                         null, null, null, ctypes.byref(err), null, 0, null)
        assert rc == piq.PIQ_ERR_INVALID_ARG
    rc = lib.piq_layer_output_error(null, 16, 64, null, null, null, null, null, 7, 32, null, 64,
                                    ctypes.byref(err), null, 0, null)
    assert rc == piq.PIQ_ERR_INVALID_ARG


def test_binding_refuses_host_tensors(lib):
    import torch
    W = torch.zeros(16, 64)
    X = torch.zeros(64, 64, dtype=torch.bfloat16)
    s = torch.ones(64)
    with pytest.raises(TypeError):
        piq.gptq_quantize_layer(W, X, sym=False)
    with pytest.raises(TypeError):
        piq.awq_gptq_quantize_layer(W, X, s)


def test_empty_and_oversized_layers_rejected(lib):
    # empty layers (no rows, no inputs, no samples) and sizes past the supported
    # maximum are refused before any device work; the fake buffer address is
    # aligned and never read
    fake = ctypes.c_void_p(1 << 12)
    err = ctypes.c_double()
    out = ctypes.c_size_t()
    for rows, inp, n in ((0, 64, 64), (16, 0, 64), (16, 64, 0), ((1 << 24) + 1, 64, 64),
                         (16, (1 << 20) + 8, 64)):
        rc = lib.gptq_quantize_layer(fake, rows, inp, fake, n, 4, 32, 0.01, 0, fake, fake, None,
                                     None, ctypes.byref(err), fake, 1 << 30, None)
        assert rc == piq.PIQ_ERR_INVALID_ARG, (rows, inp, n)
        grid = (ctypes.c_float * 2)(0.0, 0.5)
        rc = lib.awq_search_layer(fake, rows, inp, fake, n, 4, 32, grid, 2, None, fake, fake,
                                  fake, None, fake, 1 << 30, None)
        assert rc == piq.PIQ_ERR_INVALID_ARG, (rows, inp, n)
    for args in ((0, 64, 64, 128, 0), (16, 0, 64, 128, 0), (16, 64, 0, 128, 0), (16, 64, 64, 0, 0)):
        assert lib.piq_gptq_workspace_bytes(*args, ctypes.byref(out)) == piq.PIQ_ERR_INVALID_ARG


def _lower_cols(m, n_tiles):
    # column tiles of row tile m (128 rows) that reach the lower triangle (48 columns each)
    return min(n_tiles, (128 * m + 127) // 48 + 1)


@pytest.mark.parametrize("m_tiles,n_tiles", [(1, 1), (1, 7), (3, 1), (8, 3), (9, 3), (17, 40),
                                             (64, 171), (215, 574), (224, 3), (23, 598)])
@pytest.mark.parametrize("lower", [False, True])
def test_gemm_tile_order_visits_every_tile_once_by_row_groups(lib, m_tiles, n_tiles, lower):
    import numpy as np
    mt, nt = piq.gemm_tile_order(m_tiles, n_tiles, lower)
    cols = [_lower_cols(m, n_tiles) if lower else n_tiles for m in range(m_tiles)]
    assert len(mt) == sum(cols)
    assert ((mt >= 0) & (mt < m_tiles)).all() and (nt >= 0).all()
    assert (nt < np.asarray(cols)[mt]).all()
    assert len(set(zip(mt.tolist(), nt.tolist()))) == len(mt)    # each tile once
    # groups of eight row tiles, one after another; column tiles outer inside a
    # group wherever every row of the group has the column
    grp = mt // 8
    assert (np.diff(grp) >= 0).all()
    for g0 in range(0, m_tiles, 8):
        sel = grp == g0 // 8
        full = nt[sel] < cols[g0]
        assert (np.diff(nt[sel][full]) >= 0).all()
        assert full[:full.sum()].all()                              # full columns first


def test_gemm_tile_order_rejects_bad_sizes(lib):
    assert lib.piq_gemm_tile_order(0, 3, 0, 0, None, None) < 0
    assert lib.piq_gemm_tile_order(3, 0, 1, 0, None, None) < 0
    import numpy as np
    a = np.empty(2, dtype=np.int32)
    assert lib.piq_gemm_tile_order(2, 2, 0, 2, a.ctypes.data, a.ctypes.data) < 0  # 4 tiles
