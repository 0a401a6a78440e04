"""AWQ scaling then GPTQ rounding (awq_gptq_quantize_layer, awq_then_gptq_layer)
against the FP64 oracle of the composition (``oracle/compose.py``)."""
import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from tests.parity import REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import C1, make_channel_scales, make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _oracle_prepare(W, X, s, damp, act_order):
    Ws, Xs = O.scaled_layer_ref(W, X, s)
    perm, U, lam = O.gptq_prepare_ref(O.hessian_ref(Xs), damp, act_order)
    return Ws, perm, U


def _check_scaled(W, X, s, bits, g, act_order, damp=0.01, out=None, s_ref=None):
    """GPU composition on (W, X, s) against the oracle on (W, X, s_ref or s)."""
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    sg = torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).cuda()
    if out is None:
        out = piq.awq_gptq_quantize_layer(Wg, Xg, sg, bits=bits, g=g, damp=damp,
                                          act_order=act_order)
    s_o = np.asarray(s if s_ref is None else s_ref, dtype=np.float64)
    Ws, perm, U = _oracle_prepare(W, X, s_o, damp, act_order)
    assert np.array_equal(out.perm.cpu().numpy(), perm)
    assert np.array_equal(out.g_idx.cpu().numpy(), O.g_idx_ref(perm, g))
    codes_q = unpack_gpu(out.qweight, bits)[:, perm]
    stats, c_ref, sc_ref = teacher_forced_compare(codes_q, Ws[:, perm], U, bits, g)
    sc = out.scales.cpu().numpy().astype(np.float64)
    s16 = sc_ref.astype(np.float16).astype(np.float64)
    assert (np.abs(sc - s16) / np.maximum(s16, 1e-30)).max() < REL_TOL
    What = O.awq_gptq_dequant_ref(c_ref, sc_ref, perm, s_o, g)
    e_ref = O.output_error_ref(W, What, X)
    assert rel(out.err, e_ref) < REL_TOL, (out.err, e_ref)
    # the packed result read back through the library's own error entry
    e_lib = piq.layer_output_error(Wg, out.qweight, out.scales, Xg, bits, g, g_idx=out.g_idx,
                                   s=sg)
    assert rel(e_lib, e_ref) < REL_TOL, (e_lib, e_ref)
    return stats, out, e_ref


def test_tiny_layer_with_channel_scales():
    W, X = make_weight(C1), make_x_bits(C1)
    _check_scaled(W, X, make_channel_scales(512, 1), 4, 128, False)


@pytest.mark.parametrize("out,inp,n,g,bits,act", [
    (129, 520, 1500, 128, 4, False),    # ragged rows, ragged last block
    (64, 600, 1800, 200, 3, False),     # group wider than a block, not a multiple
    (100, 264, 900, 40, 4, True),       # act-order on the scaled diagonal, small groups
    (33, 1032, 3000, 128, 3, True),     # act-order, INT3
    (8, 8, 64, 8, 2, False),            # smallest layer, 2-bit
])
def test_scaled_layer_variants(out, inp, n, g, bits, act):
    spec = small_spec(out, inp, n, seed=out + 2 * inp + n, sigma_ln=0.8)
    _check_scaled(make_weight(spec), make_x_bits(spec), make_channel_scales(inp, inp, 0.7), bits,
                  g, act)


@pytest.mark.parametrize("act_order", [False, True])
def test_unit_scales_are_plain_gptq(act_order):
    # s = 1: every scaling step is an exact identity, so the outputs must equal
    # gptq_quantize_layer's bit for bit, error included.
    W, X = make_weight(C1), make_x_bits(C1)
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    ones = torch.ones(512, dtype=torch.float32, device="cuda")
    a = piq.awq_gptq_quantize_layer(Wg, Xg, ones, act_order=act_order)
    b = piq.gptq_quantize_layer(Wg, Xg, act_order=act_order)
    for x, y in zip(a[:4], b[:4]):
        assert torch.equal(x, y)
    assert a.err == b.err


@pytest.mark.parametrize("bits", [3, 4])
def test_awq_then_gptq_end_to_end(bits):
    # AWQ's search on the GPU and in the oracle must pick the same alpha; the
    # composed layer is then compared with the oracle run on the oracle's own s.
    W, X = make_weight(C1), make_x_bits(C1)
    a, out = piq.awq_then_gptq_layer(to_gpu_w(W), to_gpu_x(X), bits=bits, g=128)
    ar = O.awq_ref(W, X, bits, 128)
    assert a.best_alpha == pytest.approx(ar.best_alpha, abs=1e-7)
    s_gpu = a.s.cpu().numpy()
    assert np.allclose(s_gpu, ar.s, rtol=2e-6, atol=0)
    _check_scaled(W, X, s_gpu, bits, 128, False, out=out, s_ref=ar.s)
    # the composition lowers the error against AWQ's own rounding at that alpha
    assert out.err < a.err_per_alpha[ar.best_index]


@pytest.mark.parametrize("bad", [0.0, -1.0, float("nan"), float("inf")])
def test_invalid_channel_scale_is_reported(bad):
    W, X = make_weight(C1), make_x_bits(C1)
    s = make_channel_scales(512, 3)
    s[77] = bad
    with pytest.raises(piq.PiqError) as e:
        piq.awq_gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), torch.from_numpy(s).cuda(),
                                    act_order=True)
    assert e.value.status == piq.PIQ_ERR_INVALID_ARG
    # the context is still usable
    out = piq.awq_gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X),
                                      torch.from_numpy(make_channel_scales(512, 3)).cuda())
    assert np.isfinite(out.err)


def test_deterministic():
    W, X = make_weight(C1), make_x_bits(C1)
    s = torch.from_numpy(make_channel_scales(512, 5)).cuda()
    a = piq.awq_gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), s, act_order=True)
    b = piq.awq_gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), s, act_order=True)
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)
    assert a.err == b.err
