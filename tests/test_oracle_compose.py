"""Pins of the AWQ-then-GPTQ composition oracle (``oracle/compose.py``).

The composition is GPTQ run on the scaled layer (W diag(s), X diag(1/s)) with
What = code * scale / s_j ("GPTQ versus AWQ objectives", serving decision
list; uplatz.com report, section 3.2).  Each pin ties it to something other
than itself: plain GPTQ, AWQ's own quantizer, the error identity of the
factorisation, and the power-of-two invariance of the scaling.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from oracle.awq import awq_dequant_ref
from oracle.pack import to_memory_order
from workloads import C1, bf16_bits_from_f32, make_weight, make_x_bits


def _layer(seed, out, inp, n, corr=0.6):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((n, inp))
    X = Z + corr * np.roll(Z, 1, axis=1)
    X *= rng.lognormal(0, 0.8, inp)
    W = (rng.standard_normal((out, inp)) * 0.02).astype(np.float32)
    s = rng.lognormal(0, 0.5, inp)
    return W, bf16_bits_from_f32(X.astype(np.float32)), s


@pytest.mark.parametrize("act_order", [False, True])
def test_alpha_zero_is_plain_gptq(act_order):
    # alpha = 0 gives s = 1: the composition must be GPTQ itself, bit for bit.
    W, X = make_weight(C1), make_x_bits(C1)
    s = O.awq_scales_ref(O.channel_mean_abs_ref(X), 0.0)
    assert np.all(s == 1.0)
    r = O.awq_gptq_ref(W, X, s, bits=4, g=128, act_order=act_order)
    p = O.gptq_ref(W, X, bits=4, g=128, act_order=act_order)
    assert np.array_equal(r.perm, p.perm)
    assert np.array_equal(r.codes, p.codes)
    assert np.array_equal(r.scales, p.scales)


@pytest.mark.parametrize("bits,g", [(4, 128), (3, 64)])
def test_diagonal_hessian_is_awq_rounding(bits, g):
    # One-hot calibration rows make X'^T X' exactly diagonal for any s; GPTQ
    # then pushes no error and must round W diag(s) exactly as AWQ's own group
    # quantizer does at the same s.
    rng = np.random.default_rng(23)
    inp, n = 256, 1024
    Xf = np.zeros((n, inp), dtype=np.float32)
    Xf[np.arange(n), rng.integers(0, inp, n)] = rng.standard_normal(n).astype(np.float32)
    X = bf16_bits_from_f32(Xf)
    W = make_weight(C1)[:, :inp]
    s = rng.lognormal(0, 0.7, inp)
    r = O.awq_gptq_ref(W, X, s, bits=bits, g=g)
    c, sc = O.group_rtn_ref(W.astype(np.float64) * s[None, :], bits, g)
    assert np.array_equal(r.codes, c)
    assert np.array_equal(r.scales, sc)


@pytest.mark.parametrize("act_order", [False, True])
def test_error_identity_through_the_original_inputs(act_order):
    # GPTQ on (W', X'): sum err^2 = ||X' dW'^T||^2 + lam ||dW'||^2, and
    # X' dW'^T = X (W - code * scale / s)^T.  The right side uses the original
    # X and AWQ's reconstruction, so scaling X or What the wrong way fails it.
    W, X, s = _layer(5, 7, 96, 400)
    r = O.awq_gptq_ref(W, X, s, bits=4, g=32, act_order=act_order)
    Q_mem = to_memory_order(r.codes * r.scales[:, np.arange(96) // 32], r.perm)
    dWs = W.astype(np.float64) * s[None, :] - Q_mem
    lhs = float(np.sum(r.err ** 2)) - r.lam * float(np.sum(dWs ** 2))
    What = O.awq_gptq_dequant_ref(r.codes, r.scales, r.perm, s, 32, fp16=False)
    rhs = O.output_error_ref(W, What, X)
    assert lhs == pytest.approx(rhs, rel=1e-9)
    # the same What through AWQ's own reconstruction (natural order only)
    if not act_order:
        assert np.allclose(What, awq_dequant_ref(r.codes, r.scales, s, 32), rtol=0, atol=1e-15)


def test_codes_invariant_to_power_of_two_scale():
    # s -> 4 s multiplies W' by 4 and X' by 1/4: X'^T X' and lam scale by 1/16,
    # U by 4, err U is unchanged, so the codes are the same and the scales x4.
    W, X, s = _layer(6, 8, 128, 512)
    for act_order in (False, True):
        r1 = O.awq_gptq_ref(W, X, s, bits=3, g=64, act_order=act_order)
        r2 = O.awq_gptq_ref(W, X, 4.0 * s, bits=3, g=64, act_order=act_order)
        assert np.array_equal(r1.perm, r2.perm)
        assert np.array_equal(r1.codes, r2.codes)
        assert np.array_equal(r2.scales, 4.0 * r1.scales)


def test_blocked_equals_literal():
    W, X, s = _layer(8, 16, 320, 900)
    a = O.awq_gptq_ref(W, X, s, bits=4, g=64, act_order=True)
    b = O.awq_gptq_ref(W, X, s, bits=4, g=64, act_order=True, blocked=True)
    assert np.array_equal(a.codes, b.codes)
    assert np.allclose(a.scales, b.scales, rtol=1e-12, atol=0)


@pytest.mark.parametrize("bits", [3, 4])
def test_gptq_rounding_after_awq_scaling_lowers_the_error(bits):
    # The serving decision list: at aggressive bit widths GPTQ's compensation
    # recovers more than a scale alone, and the two compose.  On the tiny
    # layer the composed error is below AWQ's own at the same alpha.
    W, X = make_weight(C1), make_x_bits(C1)
    a, r = O.awq_then_gptq_ref(W, X, bits=bits, g=128)
    e_awq = a.err[a.best_index]
    e_comp = O.output_error_ref(W, O.awq_gptq_dequant_ref(r.codes, r.scales, r.perm, a.s, 128,
                                                          fp16=False), X)
    assert e_comp < e_awq
