"""Oracle invariants over many small random layers (hypothesis, derandomized).

Each property is one the pages and the mathematics fix, checked on layers the
fixed pins do not cover (odd widths, group sizes, bit widths, both quantizers):
the factorisation's error identity, blocked = literal, a diagonal Hessian
reducing to rounding, and s = 1 reducing the composition to plain GPTQ.
"""
import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as O
from oracle.gptq import gptq_sweep_asym_ref, gptq_sweep_blocked_asym_ref
from oracle.pack import to_memory_order
from workloads import bf16_bits_from_f32

SETTINGS = settings(derandomize=True, max_examples=60, deadline=None)


def _layer(seed, out, inp, n, corr):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((n, inp))
    X = Z + corr * np.roll(Z, 1, axis=1)
    X *= rng.lognormal(0, 0.6, inp)
    W = rng.standard_normal((out, inp)) * 0.02 + 0.005 * rng.standard_normal((out, 1))
    return W.astype(np.float32), bf16_bits_from_f32(X.astype(np.float32))


layers = st.fixed_dictionaries({
    "seed": st.integers(0, 10_000),
    "out": st.integers(1, 6),
    "inp": st.sampled_from([8, 16, 24, 40, 64, 96]),
    "g": st.sampled_from([4, 8, 12, 16, 32, 1000]),
    "bits": st.sampled_from([2, 3, 4]),
    "act": st.booleans(),
    "sym": st.booleans(),
    "corr": st.floats(0.0, 0.9),
})


@SETTINGS
@given(layers)
def test_error_identity(p):
    # sum err^2 = tr(dW H_d dW^T) = ||X dW^T||^2 + lam ||dW||^2 for every layer
    W, X = _layer(p["seed"], p["out"], p["inp"], 4 * p["inp"], p["corr"])
    g = min(p["g"], p["inp"])
    r = O.gptq_ref(W, X, bits=p["bits"], g=g, act_order=p["act"], sym=p["sym"])
    Q_q = r.codes * r.scales[:, np.arange(p["inp"]) // g]
    dW = W.astype(np.float64) - to_memory_order(Q_q, r.perm)
    lhs = float(np.sum(r.err ** 2)) - r.lam * float(np.sum(dW ** 2))
    rhs = O.output_error_ref(W, W.astype(np.float64) - dW, X)
    assert abs(lhs - rhs) <= 1e-9 * max(abs(rhs), 1e-30) + 1e-18


@SETTINGS
@given(layers)
def test_blocked_equals_literal(p):
    W, X = _layer(p["seed"], p["out"], p["inp"], 4 * p["inp"], p["corr"])
    _, U, _ = O.gptq_prepare_ref(O.hessian_ref(X), 0.01, False)
    Wp = W.astype(np.float64)
    g, bits = p["g"], p["bits"]
    if p["sym"]:
        c1, s1, _, _ = O.gptq_sweep_ref(Wp, U, bits, g)
        c2, s2, _ = O.gptq.gptq_sweep_blocked_ref(Wp, U, bits, g, block=16)
        z1 = z2 = None
    else:
        c1, s1, z1, _, _, _ = gptq_sweep_asym_ref(Wp, U, bits, g)
        c2, s2, z2, _, _ = gptq_sweep_blocked_asym_ref(Wp, U, bits, g, block=16)
    assert np.array_equal(c1, c2)
    assert np.allclose(s1, s2, rtol=1e-12, atol=0)
    if z1 is not None:
        assert np.array_equal(z1, z2)


@SETTINGS
@given(layers)
def test_diagonal_hessian_is_rounding(p):
    rng = np.random.default_rng(p["seed"])
    inp, n = p["inp"], 8 * p["inp"]
    Xf = np.zeros((n, inp), dtype=np.float32)
    Xf[np.arange(n), rng.integers(0, inp, n)] = rng.standard_normal(n).astype(np.float32)
    X = bf16_bits_from_f32(Xf)
    W, _ = _layer(p["seed"], p["out"], inp, 4, 0.0)
    r = O.gptq_ref(W, X, bits=p["bits"], g=p["g"], sym=p["sym"])
    if p["sym"]:
        c, s = O.rtn_ref(W, p["bits"], p["g"])
    else:
        c, s, z = O.rtn_asym_ref(W, p["bits"], p["g"])
        assert np.array_equal(r.zeros, z)
    assert np.array_equal(r.codes, c) and np.array_equal(r.scales, s)


@SETTINGS
@given(layers)
def test_unit_scales_compose_to_plain_gptq(p):
    W, X = _layer(p["seed"], p["out"], p["inp"], 4 * p["inp"], p["corr"])
    a = O.awq_gptq_ref(W, X, np.ones(p["inp"]), bits=p["bits"], g=p["g"], act_order=p["act"])
    b = O.gptq_ref(W, X, bits=p["bits"], g=p["g"], act_order=p["act"])
    assert np.array_equal(a.perm, b.perm) and np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scales, b.scales)


awq_layers = st.fixed_dictionaries({
    "seed": st.integers(0, 10_000),
    "out": st.integers(1, 6),
    "inp": st.sampled_from([16, 32, 64, 96]),
    "g": st.sampled_from([8, 16, 32, 1000]),
    "bits": st.sampled_from([2, 3, 4]),
    "k": st.integers(-3, 3),
})


@settings(derandomize=True, max_examples=40, deadline=None)
@given(awq_layers)
def test_awq_search_properties(p):
    # alpha = 0 is plain group rounding; the chosen alpha is the first minimum
    # of the scored errors; s -> 2^k s keeps the codes (scales x 2^k)
    from oracle.awq import awq_dequant_ref
    W, X = _layer(p["seed"], p["out"], p["inp"], 4 * p["inp"], 0.5)
    grid = [0.0, 0.25, 0.5, 0.75]
    a = O.awq_ref(W, X, p["bits"], p["g"], grid)
    c, s = O.rtn_ref(W, p["bits"], p["g"])
    g = min(p["g"], p["inp"])
    e_rtn = O.output_error_ref(W, awq_dequant_ref(c, s, np.ones(p["inp"]), g), X)
    assert abs(a.err[0] - e_rtn) <= 1e-12 * max(e_rtn, 1e-300)
    assert a.best_index == int(np.flatnonzero(a.err == a.err.min())[0])
    s_best = O.awq_scales_ref(a.m, grid[a.best_index])
    c1, sc1 = O.group_rtn_ref(W * s_best[None, :], p["bits"], p["g"])
    c2, sc2 = O.group_rtn_ref(W * (2.0 ** p["k"] * s_best)[None, :], p["bits"], p["g"])
    assert np.array_equal(c1, a.codes) and np.array_equal(c1, c2)
    assert np.array_equal(sc2, 2.0 ** p["k"] * sc1)


def test_sweep_identity_on_r():
    # The identity the GPU sweep is built on: with H_d = R R^T (R upper, the
    # reversed Cholesky factor) and U = inv(R), the listing's loop satisfies
    # W0 - Q = err U row by row (W0 the weights before any update, Q = code *
    # scale, err the pushed errors), so err = (W0 - Q) R and the current weights
    # at the start of a block G are W0_G + acc_G inv(R_GG) with
    # acc = sum_{p < b} (W0 - Q)_p R[p, :].
    from workloads import make_weight, make_x_bits, small_spec
    spec = small_spec(12, 256, 900, seed=71, sigma_ln=0.9, n_outlier=3, outlier_gain=20.0)
    W, X = make_weight(spec).astype(np.float64), make_x_bits(spec)
    H = O.hessian_ref(X)
    perm, U, lam = O.gptq_prepare_ref(H, 0.01, False)
    Hd = H + lam * np.eye(H.shape[0])
    Jr = slice(None, None, -1)
    R = np.linalg.cholesky(Hd[Jr, Jr])[Jr, Jr]
    assert np.allclose(R @ R.T, Hd, rtol=0, atol=1e-9 * np.abs(Hd).max())
    codes, scales, v, err = O.gptq_sweep_ref(W, U, 4, 64)
    Q = codes * np.repeat(scales, 64, axis=1)
    assert np.allclose(err, (W - Q) @ R, rtol=0, atol=1e-9 * np.abs(err).max())
    # block-start weights of the block [128, 192): v * scale there equals
    # W0 + acc inv(R_GG) before any of the block's own updates, at its first column
    b = 128
    acc = (W - Q)[:, :b] @ R[:b, b:]
    Wb = W[:, b:] + acc @ np.linalg.inv(R[b:, b:])
    assert np.allclose(v[:, b] * scales[:, b // 64], Wb[:, 0], rtol=0, atol=1e-9)


def test_syrk_hessian_equals_the_product():
    # the BLAS symmetric rank-k route to H = X^T X against the plain product,
    # over a chunk boundary and a ragged width (bf16 bit patterns as inputs)
    rng = np.random.default_rng(41)
    X = (rng.standard_normal((2500, 131)) * rng.lognormal(0.0, 1.0, 131)).astype(np.float32)
    Xb = (X.view(np.uint32) >> 16).astype(np.uint16)
    H1 = O.hessian_ref(Xb)
    H2 = O.hessian_syrk_ref(Xb, chunk=1000)
    assert np.array_equal(H2, H2.T)
    assert np.abs(H1 - H2).max() <= 1e-13 * np.abs(H1).max()


@pytest.mark.parametrize("n", [1, 2, 7, 130])
def test_r_route_factor_equals_the_listing(n):
    # U = inv(R) with R = J chol(J H_d J) J is the listing's cholesky(inv(H_d)).T
    rng = np.random.default_rng(n)
    A = rng.standard_normal((n + 5, n))
    Hd, _ = O.damped_ref(A.T @ A, 0.01)
    U1 = O.upper_factor_ref(Hd)
    U2 = O.upper_factor_r_ref(Hd)
    assert np.array_equal(np.tril(U2, -1), np.zeros_like(U2))
    assert (np.abs(U1 - U2) / np.abs(np.diag(U1))[:, None]).max() < 1e-12
    assert np.abs(U2.T @ U2 @ Hd - np.eye(n)).max() < 1e-10


def test_row_chunks_sweep_like_one_call():
    # rows are independent given U: the pooled sweep over chunks of rows
    # (tests/oracle_pool.py, used at full size) gives one call's codes, and its
    # scales and quotients up to the rounding order of the block products
    from oracle.gptq import gptq_sweep_blocked_ref
    from tests.oracle_pool import sweep_rows
    rng = np.random.default_rng(8)
    W = rng.standard_normal((70, 300)) * 0.02
    A = rng.standard_normal((320, 300))
    Hd, _ = O.damped_ref(A.T @ A, 0.01)
    U = O.upper_factor_r_ref(Hd)
    one = gptq_sweep_blocked_ref(W, U, 4, 128)
    for workers in (1, 2):
        codes, scales, v = sweep_rows(W, U, 4, 128, chunk=32, workers=workers)
        assert np.array_equal(codes, one[0])
        # the BLAS block products may round in another order for another row count
        assert np.abs(scales - one[1]).max() <= 1e-12 * np.abs(one[1]).max()
        assert np.abs(v - one[2]).max() <= 1e-12 * np.abs(one[2]).max()
