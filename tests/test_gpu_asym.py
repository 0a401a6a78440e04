"""GPTQ with a scale and zero-point per group (gptq_quantize_layer_asym)
against the oracle's asymmetric sweep (``oracle/gptq.py``, sym=False)."""
import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from oracle.pack import dequant_ref
from tests.parity import REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import C1, make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _check_asym(W, X, bits, g, act_order, damp=0.01):
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    out = piq.gptq_quantize_layer(Wg, Xg, bits=bits, g=g, damp=damp, act_order=act_order,
                                  sym=False)
    perm, U, _ = O.gptq_prepare_ref(O.hessian_ref(X), damp, act_order)
    assert np.array_equal(out.perm.cpu().numpy(), perm)
    g_idx = O.g_idx_ref(perm, g)
    assert np.array_equal(out.g_idx.cpu().numpy(), g_idx)
    maxq = 2 ** bits - 1
    u_mem = unpack_gpu(out.qweight, bits) + 2 ** (bits - 1)     # the stored codes
    z_gpu = out.zeros.cpu().numpy().astype(np.int16)
    assert u_mem.min() >= 0 and u_mem.max() <= maxq
    assert z_gpu.min() >= 0 and z_gpu.max() <= maxq
    codes_q = (u_mem - z_gpu[:, g_idx])[:, perm]
    stats, c_ref, s_ref, z_ref = teacher_forced_compare(
        codes_q, W.astype(np.float64)[:, perm], U, bits, g, gpu_zeros=z_gpu)
    assert np.array_equal(z_gpu, z_ref)
    sc = out.scales.cpu().numpy().astype(np.float64)
    s16 = s_ref.astype(np.float16).astype(np.float64)
    live = s16 > 0
    assert np.array_equal(sc == 0, ~live)
    assert (np.abs(sc[live] - s16[live]) / s16[live]).max() < REL_TOL
    e_ref = O.output_error_ref(W, dequant_ref(c_ref, s_ref, perm, g), X)
    assert rel(out.err, e_ref) < REL_TOL, (out.err, e_ref)
    # the packed layer read back through the library's error entry
    e_lib = piq.layer_output_error(Wg, out.qweight, out.scales, Xg, bits, g, g_idx=out.g_idx,
                                   zeros=out.zeros)
    assert rel(e_lib, e_ref) < REL_TOL, (e_lib, e_ref)
    return stats, out, e_ref


def test_tiny_layer_asym():
    W, X = make_weight(C1), make_x_bits(C1)
    _check_asym(W, X, 4, 128, False)


@pytest.mark.parametrize("out,inp,n,g,bits,act", [
    (129, 520, 1500, 128, 4, False),    # whole-block groups, ragged rows and last block
    (64, 520, 1600, 256, 3, False),     # a group carried into the next block (zero reloaded)
    (64, 600, 1800, 200, 3, False),     # group starts inside blocks
    (100, 264, 900, 40, 4, True),       # act-order, small groups
    (33, 1032, 3000, 128, 2, True),     # act-order, 2-bit
    (48, 136, 500, 1000, 4, False),     # one group per row, carried across a block
    (8, 8, 64, 8, 2, False),            # smallest layer
])
def test_asym_variants(out, inp, n, g, bits, act):
    spec = small_spec(out, inp, n, seed=3 * out + inp + n, sigma_ln=0.8)
    W = make_weight(spec)
    W += 0.02 * np.sin(np.arange(out, dtype=np.float32))[:, None]   # rows off centre
    _check_asym(W, make_x_bits(spec), bits, g, act)


def test_one_signed_and_zero_rows():
    # rows that start all positive or all negative (zero-points at the ends of
    # the range while the updates keep the sign) and an all-zero row (scale 0,
    # zero-point 0: its errors are 0, so it stays zero) on the same layer
    spec = small_spec(16, 256, 1024, seed=77, sigma_ln=0.5)
    W = make_weight(spec)
    W[0:4] = np.abs(W[0:4]) + 0.01
    W[4:8] = -np.abs(W[4:8]) - 0.01
    W[8] = 0.0
    _, out, _ = _check_asym(W, make_x_bits(spec), 4, 64, False)
    z = out.zeros.cpu().numpy()
    assert np.all(z[8] == 0) and np.all(out.scales[8].cpu().numpy() == 0)


def test_asym_and_sym_share_the_factor():
    # the same H, order and U: only the rounding differs, so the two calls
    # agree on perm and g_idx, and both errors match the oracle (checked above)
    W, X = make_weight(C1), make_x_bits(C1)
    a = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), act_order=True)
    b = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), act_order=True, sym=False)
    assert torch.equal(a.perm, b.perm) and torch.equal(a.g_idx, b.g_idx)
    assert b.zeros is not None and a.zeros is None


def test_deterministic():
    W, X = make_weight(C1), make_x_bits(C1)
    a = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), sym=False)
    b = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), sym=False)
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.zeros, b.zeros)
    assert a.err == b.err
