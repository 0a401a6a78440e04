"""Pins of the asymmetric-group quantizer of the oracle (a scale and zero-point
per group: the uplatz.com report, GPTQ key parameters, Group Size).

The pages give no formula, so the quantizer is a reading (min/max affine
rounding over a range widened to hold 0).  Its arithmetic is pinned by a
hand-worked example and by the nearest-grid-point property; GPTQ's machinery
around it by the same identities the symmetric sweep satisfies: diagonal H
reduces to rounding, the factorisation's error identity, Babai's nearest
plane on the group's grid, and an exhaustive search on tiny layers.
"""
from __future__ import annotations

import itertools

import numpy as np
import pytest

import oracle as O
from oracle.gptq import gptq_sweep_asym_ref, gptq_sweep_blocked_asym_ref
from oracle.pack import to_memory_order
from workloads import C1, bf16_bits_from_f32, make_weight


def _layer(seed, out, inp, n, corr=0.6):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((n, inp))
    X = Z + corr * np.roll(Z, 1, axis=1) + 0.5 * corr * np.roll(Z, 2, axis=1)
    X *= rng.lognormal(0, 0.7, inp)
    W = (rng.standard_normal((out, inp)) * 0.02 + 0.01 * rng.standard_normal((out, 1)))
    return W.astype(np.float32), bf16_bits_from_f32(X.astype(np.float32))


def test_asym_rounding_worked_example(golden):
    d = golden("asym_rtn_worked_example.json")
    W = np.array(d["W"])
    c, sc, z = O.rtn_asym_ref(W, d["bits"], d["g"])
    assert sc[:, 0].tolist() == d["scales"]
    assert z[:, 0].tolist() == d["zeros"]
    assert (c + z[:, [0]]).tolist() == d["u"]
    assert (c * sc[:, [0]]).tolist() == d["What"]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_asym_rounding_is_nearest_grid_point(bits):
    # every weight goes to the nearest point of its group's grid
    # {(u - zero) * scale : 0 <= u <= 2^bits - 1}; the zero-point is a code.
    rng = np.random.default_rng(bits)
    W = rng.standard_normal((40, 96)) * 0.02 + rng.standard_normal((40, 1)) * 0.02
    g, maxq = 32, 2 ** bits - 1
    c, sc, z = O.rtn_asym_ref(W, bits, g)
    assert z.min() >= 0 and z.max() <= maxq
    u = np.arange(maxq + 1)
    for r in range(W.shape[0]):
        for k in range(W.shape[1]):
            grid = (u - z[r, k // g]) * sc[r, k // g]
            dist = np.abs(W[r, k] - grid)
            assert dist[c[r, k] + z[r, k // g]] <= dist.min() * (1 + 1e-12) + 1e-300


def test_zero_weights_are_exact_and_range_covers_the_group():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((16, 64)) * 0.02
    W[:, ::5] = 0.0
    c, sc, z = O.rtn_asym_ref(W, 4, 16)
    What = c * np.repeat(sc, 16, axis=1)
    assert np.all(What[:, ::5] == 0.0)
    # the grid spans the widened range up to half a step at each end
    lo = np.minimum(W.reshape(16, 4, 16).min(axis=2), 0)
    hi = np.maximum(W.reshape(16, 4, 16).max(axis=2), 0)
    assert np.all(-z * sc <= lo + 0.5 * sc * (1 + 1e-12))
    assert np.all((15 - z) * sc >= hi - 0.5 * sc * (1 + 1e-12))


def test_diagonal_hessian_reduces_to_asym_rounding():
    rng = np.random.default_rng(12)
    inp, n = 256, 1024
    Xf = np.zeros((n, inp), dtype=np.float32)
    Xf[np.arange(n), rng.integers(0, inp, n)] = rng.standard_normal(n).astype(np.float32)
    X = bf16_bits_from_f32(Xf)
    H = O.hessian_ref(X)
    W = make_weight(C1)[:, :inp] + 0.01
    for bits, g in ((4, 128), (3, 64), (2, 256)):
        r = O.gptq_ref(W, H=H, bits=bits, g=g, sym=False)
        c, s, z = O.rtn_asym_ref(W, bits, g)
        assert np.array_equal(r.codes, c)
        assert np.array_equal(r.scales, s)
        assert np.array_equal(r.zeros, z)


@pytest.mark.parametrize("act_order", [False, True])
def test_asym_error_identity(act_order):
    W, X = _layer(13, 9, 96, 400)
    r = O.gptq_ref(W, X, bits=3, g=32, act_order=act_order, sym=False)
    Q_q = r.codes * r.scales[:, np.arange(96) // 32]
    dW = W.astype(np.float64) - to_memory_order(Q_q, r.perm)
    lhs = float(np.sum(r.err ** 2)) - r.lam * float(np.sum(dW ** 2))
    rhs = O.output_error_ref(W, W.astype(np.float64) - dW, X)
    assert lhs == pytest.approx(rhs, rel=1e-9)


def _babai_codes(w, Hd, scale, cmin, cmax):
    """Babai's nearest plane (uplatz.com report, section 2.3) on the grid
    scale * Z, each coordinate rounded then clipped to [cmin, cmax]."""
    Lr = np.linalg.cholesky(Hd[::-1, ::-1])
    R = Lr[::-1, ::-1]
    y = w @ R
    q = np.zeros(w.size)
    for j in range(w.size):
        q[j] = np.clip(np.round(y[j] / (scale * R[j, j])), cmin, cmax)
        y = y - q[j] * scale * R[j, :]
    return q


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_asym_gptq_equals_babai_nearest_plane(bits):
    # One group per row: scale and zero-point are fixed by the original row.
    W, X = _layer(27 + bits, 6, 40, 160)
    H = O.hessian_ref(X)
    r = O.gptq_ref(W, H=H, bits=bits, g=40, sym=False)
    Hd, _ = O.damped_ref(H, 0.01)
    maxq = 2 ** bits - 1
    for row in range(W.shape[0]):
        w = W[row].astype(np.float64)
        lo, hi = min(w.min(), 0.0), max(w.max(), 0.0)
        scale = (hi - lo) / maxq
        zero = np.round(-lo / scale)
        q = _babai_codes(w, Hd, scale, -zero, maxq - zero)
        assert np.array_equal(q.astype(np.int64), r.codes[row].astype(np.int64))
        assert r.zeros[row, 0] == zero


def _exhaustive_min(w, H, scale, zero, maxq):
    cand = np.arange(maxq + 1, dtype=np.float64) - zero
    n = w.size
    tail = np.array(list(itertools.product(cand, repeat=4)))
    best = np.inf
    for head in itertools.product(cand, repeat=n - 4):
        d = np.concatenate([np.broadcast_to(np.array(head), (tail.shape[0], n - 4)), tail], 1)
        d = w[None, :] - scale * d
        best = min(best, float(np.einsum("ki,ij,kj->k", d, H, d).min()))
    return best


def test_exhaustive_tiny_layer_bounds_asym_gptq():
    # out = 1, in = 8, bits = 3, one group: all 8^8 stored-code vectors.
    ratios_g, ratios_r = [], []
    for seed in range(3):
        W, X = _layer(200 + seed, 1, 8, 24, corr=0.9)
        H = O.hessian_ref(X)
        r = O.gptq_ref(W, H=H, bits=3, g=8, sym=False)
        c, s, z = O.rtn_asym_ref(W, 3, 8)
        w = W[0].astype(np.float64)
        scale, zero = r.scales[0, 0], r.zeros[0, 0]
        assert scale == s[0, 0] and zero == z[0, 0]
        e_star = _exhaustive_min(w, H, scale, zero, 7)
        dg, dr = w - scale * r.codes[0], w - scale * c[0]
        e_g, e_r = dg @ H @ dg, dr @ H @ dr
        assert e_star <= e_g * (1 + 1e-12) and e_star <= e_r * (1 + 1e-12)
        ratios_g.append(e_g / e_star)
        ratios_r.append(e_r / e_star)
    assert np.median(ratios_g) <= np.median(ratios_r)


@pytest.mark.parametrize("inp,g", [(520, 96), (264, 40), (136, 128), (200, 1000)])
def test_asym_blocked_equals_literal(inp, g):
    W, X = _layer(inp + g, 12, inp, 3 * inp)
    H = O.hessian_ref(X)
    perm, U, _ = O.gptq_prepare_ref(H, 0.01, False)
    Wp = W.astype(np.float64)
    c1, s1, z1, _, _, _ = gptq_sweep_asym_ref(Wp, U, 4, g)
    c2, s2, z2, _, _ = gptq_sweep_blocked_asym_ref(Wp, U, 4, g)
    assert np.array_equal(c1, c2) and np.array_equal(z1, z2)
    assert np.allclose(s1, s2, rtol=1e-12, atol=0)


def test_asym_codes_invariant_to_power_of_two_weight_scale():
    W, X = _layer(31, 8, 64, 256)
    a = O.gptq_ref(W, X, g=32, sym=False)
    b = O.gptq_ref(W * 4.0, X, g=32, sym=False)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.zeros, b.zeros)
    assert np.array_equal(b.scales, 4.0 * a.scales)


def test_pack_asym_roundtrip():
    rng = np.random.default_rng(5)
    bits, g, inp = 4, 16, 64
    zeros = rng.integers(0, 16, (3, inp // g))
    u = rng.integers(0, 16, (3, inp))
    g_idx = np.arange(inp) // g
    codes = u - zeros[:, g_idx]
    q = O.pack_asym_ref(codes, zeros, g_idx, bits)
    assert np.array_equal(O.unpack_ref(q, bits) + 2 ** (bits - 1), u)
