"""Pins of the FP64 oracle to facts other than itself (CPU only).

Each test names what fixes the expected value: a hand-worked example under
tests/golden/, a closed form, an algebraic identity of the method, an
independent algorithm the pages name (Babai's nearest plane), or brute force on
tiny inputs.
"""
import itertools

import numpy as np
import pytest

import oracle as O
from oracle.awq import awq_dequant_ref
from oracle.gptq import NO_FORCE, gptq_sweep_blocked_ref
from oracle.pack import dequant_ref, to_memory_order
from workloads import C1, bf16_bits_from_f32, make_weight, make_x_bits, small_spec


# ---------------------------------------------------------------- H, damping, U
def test_hessian_and_damping_worked_example(golden):
    d = golden("hessian_worked_example.json")
    X = np.array(d["X"], dtype=np.float64)
    H = O.hessian_ref(X)
    assert np.array_equal(H, np.array(d["H"], dtype=np.float64))
    Hd, lam = O.damped_ref(H, d["damp"])
    assert lam == pytest.approx(d["lambda"], rel=1e-15)
    assert np.allclose(Hd, np.array(d["Hd"]), rtol=1e-15, atol=0)


def test_hessian_of_bf16_bits_is_exact():
    # bfloat16 values are exact in float64; integer-valued data sums exactly.
    rng = np.random.default_rng(5)
    Xi = rng.integers(-8, 9, size=(300, 24)).astype(np.float32)
    H = O.hessian_ref(bf16_bits_from_f32(Xi))
    Xd = Xi.astype(np.int64)
    assert np.array_equal(H, (Xd.T @ Xd).astype(np.float64))


def test_upper_factor_closed_form(golden):
    d = golden("upper_factor_2x2.json")
    U = O.upper_factor_ref(np.array(d["Hd"], dtype=np.float64))
    assert np.allclose(U, np.array(d["U"]), rtol=1e-14, atol=1e-16)


def test_upper_factor_matches_reversed_cholesky_route():
    # Independent route: L' = chol(J Hd J), U = J inv(L') J  (J reverses indices)
    rng = np.random.default_rng(1)
    for n in (5, 64, 200):
        A = rng.standard_normal((3 * n, n)) * rng.lognormal(0, 1, n)
        Hd, _ = O.damped_ref(A.T @ A, 0.01)
        U = O.upper_factor_ref(Hd)
        Lr = np.linalg.cholesky(Hd[::-1, ::-1])
        U2 = np.linalg.inv(Lr)[::-1, ::-1]
        assert np.allclose(np.triu(U), U, atol=0)
        assert np.max(np.abs(U - U2)) <= 1e-10 * np.max(np.abs(U))
        assert np.allclose(U.T @ U @ Hd, np.eye(n), atol=1e-9)


def test_not_positive_definite_raises():
    H = np.zeros((4, 4))
    Hd, lam = O.damped_ref(H, 0.01)
    assert lam == 0.0
    with pytest.raises(np.linalg.LinAlgError):
        O.upper_factor_ref(Hd)


# --------------------------------------------------------------------- the sweep
def test_sweep_worked_example(golden):
    d = golden("sweep_worked_example.json")
    U = np.array(d["U"], dtype=np.float64)
    w = np.array([d["w"]], dtype=np.float64)
    codes, scales, v, e = O.gptq_sweep_ref(w, U, d["bits"], d["g"])
    assert codes[0].tolist() == d["codes"]
    assert scales[0].tolist() == d["scales"]
    assert v[0].tolist() == d["v"]
    assert e[0].tolist() == d["err"]


def test_sweep_clip_example(golden):
    # both ends of the code range bind: an update pushes one code past qmax and
    # another past -qmax-1
    d = golden("sweep_clip_example.json")
    U = np.array(d["U"], dtype=np.float64)
    w = np.array([d["w"]], dtype=np.float64)
    for sweep in (lambda: O.gptq_sweep_ref(w, U, d["bits"], d["g"]),
                  lambda: O.gptq_sweep_ref(w, U, d["bits"], d["g"], dtype=np.float32)):
        codes, scales, v, e = sweep()
        assert codes[0].tolist() == d["codes"]
        assert scales[0].tolist() == d["scales"]
        assert v[0].tolist() == d["v"]
        assert e[0].tolist() == d["err"]
    codes, scales, v = O.gptq_sweep_blocked_ref(w, U, d["bits"], d["g"], block=4)
    assert codes[0].tolist() == d["codes"] and v[0].tolist() == d["v"]


def _random_layer(seed, out, inp, n, corr=0.6):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((n, inp))
    X = Z + corr * np.roll(Z, 1, axis=1) + 0.5 * corr * np.roll(Z, 2, axis=1)
    X *= rng.lognormal(0, 0.7, inp)
    X = bf16_bits_from_f32(X.astype(np.float32))
    W = (rng.standard_normal((out, inp)) * 0.02).astype(np.float32)
    return W, X


def _babai_codes(w, Hd, scale, qmax):
    """Babai's nearest plane for min_q ||(w - scale*q) R||, Hd = R R^T with R upper
    (uplatz.com report, section 2.3 'Geometric Interpretation'), with the rounding
    clipped to the code range as the quantizer does."""
    Lr = np.linalg.cholesky(Hd[::-1, ::-1])
    R = Lr[::-1, ::-1]                      # upper, Hd = R R^T
    y = w @ R
    n = w.size
    q = np.zeros(n)
    for j in range(n):
        t = y[j] / (scale * R[j, j])
        q[j] = np.clip(np.round(t), -qmax - 1, qmax)
        y = y - q[j] * scale * R[j, :]
    return q


@pytest.mark.parametrize("bits", [3, 4])
def test_gptq_equals_babai_nearest_plane(bits):
    # One group per row (g >= in): the scale is fixed by the original row, and
    # GPTQ must pick exactly the codes of the nearest-plane algorithm.
    W, X = _random_layer(7 + bits, 6, 40, 160)
    H = O.hessian_ref(X)
    r = O.gptq_ref(W, H=H, bits=bits, g=40)
    Hd, _ = O.damped_ref(H, 0.01)
    qmax = 2 ** (bits - 1) - 1
    for row in range(W.shape[0]):
        scale = np.max(np.abs(W[row].astype(np.float64))) / qmax
        q = _babai_codes(W[row].astype(np.float64), Hd, scale, qmax)
        assert np.array_equal(q.astype(np.int64), r.codes[row].astype(np.int64))


@pytest.mark.parametrize("act_order", [False, True])
def test_error_identity(act_order):
    # W0 - Q = Err U  =>  sum(err^2) = tr(dW Hd dW^T) = ||X dW^T||^2 + lam ||dW||^2
    W, X = _random_layer(3, 9, 96, 400)
    r = O.gptq_ref(W, X, bits=4, g=32, act_order=act_order)
    Q_q = r.codes * r.scales[:, np.arange(96) // 32]
    dW = W.astype(np.float64) - to_memory_order(Q_q, r.perm)
    lhs = float(np.sum(r.err ** 2)) - r.lam * float(np.sum(dW ** 2))
    rhs = O.output_error_ref(W, W.astype(np.float64) - dW, X)
    assert lhs == pytest.approx(rhs, rel=1e-9)


def test_diagonal_hessian_reduces_to_rtn():
    # One-hot rows give an exactly diagonal X^T X; U is then diagonal, no error
    # is pushed, and GPTQ must equal group RTN bit for bit.
    rng = np.random.default_rng(11)
    inp, n = 256, 1024
    Xf = np.zeros((n, inp), dtype=np.float32)
    Xf[np.arange(n), rng.integers(0, inp, n)] = rng.standard_normal(n).astype(np.float32)
    X = bf16_bits_from_f32(Xf)
    H = O.hessian_ref(X)
    assert np.count_nonzero(H - np.diag(np.diag(H))) == 0
    W = make_weight(C1)[:, :inp]
    for bits, g in ((4, 128), (3, 64), (4, 256)):
        r = O.gptq_ref(W, H=H, bits=bits, g=g)
        c, s = O.rtn_ref(W, bits, g)
        assert np.array_equal(r.codes, c)
        assert np.array_equal(r.scales, s)


def test_rtn_is_nearest_code_brute_force():
    # Brute force over every code: the nearest grid point, ties to the even code.
    rng = np.random.default_rng(2)
    W = rng.standard_normal((5, 48))
    W[0, 3] = 2.5 * np.abs(W[0]).max() / 7   # a v = +-2.5 tie candidate region
    for bits, g in ((4, 16), (3, 48), (2, 8)):
        qmax = 2 ** (bits - 1) - 1
        codes, scales = O.rtn_ref(W, bits, g)
        cand = np.arange(-qmax - 1, qmax + 1)
        for r_ in range(W.shape[0]):
            for j in range(W.shape[1]):
                sc = np.abs(W[r_, (j // g) * g:(j // g + 1) * g]).max() / qmax
                assert scales[r_, j // g] == sc
                dist = np.abs(W[r_, j] / sc - cand)
                best = cand[dist == dist.min()]
                want = best[0] if best.size == 1 else best[best % 2 == 0][0]
                assert codes[r_, j] == want
        # the largest |w| of a group lands exactly on +-qmax
        for s0 in range(0, W.shape[1], g):
            k = np.argmax(np.abs(W[:, s0:s0 + g]), axis=1)
            assert np.all(np.abs(codes[np.arange(5), s0 + k]) == qmax)


def test_blocked_equals_literal():
    W, X = make_weight(C1), make_x_bits(C1)
    H = O.hessian_ref(X)
    for g, block in ((128, 128), (64, 128), (128, 64), (256, 128)):
        a = O.gptq_ref(W, H=H, g=g)
        b = O.gptq_ref_blocked(W, H=H, g=g, block=block)
        assert np.array_equal(a.codes, b.codes)
        assert np.allclose(a.scales, b.scales, rtol=1e-12)


@pytest.mark.parametrize("inp,g", [(520, 96), (600, 200), (136, 128), (264, 40), (200, 1000)])
def test_blocked_equals_literal_ragged(inp, g):
    W, X = _random_layer(inp + g, 7, inp, 3 * inp)
    H = O.hessian_ref(X)
    a = O.gptq_ref(W, H=H, g=g)
    b = O.gptq_ref_blocked(W, H=H, g=g)
    assert np.array_equal(a.codes, b.codes)
    for bb, ee in O.block_partition_ref(inp, g):
        assert ee - bb <= 128
        for s in range(0, inp, g):
            if bb < s < ee:
                assert min(s + g, inp) <= ee


def test_scale_invariances():
    W, X = _random_layer(4, 8, 64, 256)
    r = O.gptq_ref(W, X, g=32)
    X2 = bf16_bits_from_f32(((X.astype(np.uint32) << 16).view(np.float32) * 4.0))
    r2 = O.gptq_ref(W, X2, g=32)
    assert np.array_equal(r.codes, r2.codes)
    r3 = O.gptq_ref(W * 2.0, X, g=32)
    assert np.array_equal(r.codes, r3.codes)
    assert np.array_equal(r3.scales, 2.0 * r.scales)


def test_forcing_hook_changes_only_forced_trajectory():
    W, X = _random_layer(9, 4, 64, 256)
    r = O.gptq_ref(W, X, g=32)
    force = np.full(r.codes.shape, NO_FORCE, dtype=np.int16)
    force[2, 10] = r.codes[2, 10] + 1
    f = O.gptq_ref(W, X, g=32, force=force)
    assert f.codes[2, 10] == r.codes[2, 10] + 1
    assert np.array_equal(f.codes[[0, 1, 3]], r.codes[[0, 1, 3]])
    assert np.array_equal(f.codes[2, :10], r.codes[2, :10])


# ------------------------------------------------------------- act-order, pack
def test_act_order_worked_example(golden):
    d = golden("act_order_worked_example.json")
    H = np.diag(np.array(d["diag"], dtype=np.float64))
    perm = O.act_order_perm_ref(H)
    assert perm.tolist() == d["perm"]
    assert O.g_idx_ref(perm, d["g"]).tolist() == d["g_idx"]


def test_act_order_is_a_descending_stable_permutation():
    W, X = _random_layer(21, 5, 128, 512)
    r = O.gptq_ref(W, X, g=32, act_order=True)
    diag = np.diag(O.hessian_ref(X))
    assert sorted(r.perm.tolist()) == list(range(128))
    d = diag[r.perm]
    assert np.all(d[:-1] >= d[1:])
    assert np.array_equal(r.g_idx[r.perm], np.arange(128) // 32)


def test_pack_worked_example(golden):
    d = golden("pack_worked_example.json")
    for case in d["cases"]:
        q = O.pack_ref(np.array([case["codes"]]), case["bits"])
        assert q.shape == (1, 1) and q.dtype == np.uint32
        assert q[0, 0] == int(case["word_hex"], 16)
        assert O.unpack_ref(q, case["bits"])[0].tolist() == case["codes"]


def test_pack_roundtrip_random():
    rng = np.random.default_rng(0)
    for bits in (2, 3, 4):
        qmax = 2 ** (bits - 1) - 1
        c = rng.integers(-qmax - 1, qmax + 1, size=(7, 64))
        assert np.array_equal(O.unpack_ref(O.pack_ref(c, bits), bits), c)


# -------------------------------------------------------------------------- AWQ
def test_awq_channel_mean_worked_example(golden):
    d = golden("awq_channel_mean_example.json")
    X = np.array(d["X"], dtype=np.float64)
    m = O.channel_mean_abs_ref(X)
    assert m.tolist() == d["m"]
    assert O.awq_scales_ref(m, d["alpha"]).tolist() == d["s"]


def test_awq_alpha_zero_is_rtn_and_best_not_worse():
    W, X = make_weight(C1), make_x_bits(C1)
    a = O.awq_ref(W, X, bits=4, g=128)
    c, s = O.rtn_ref(W, 4, 128)
    c0, s0 = O.group_rtn_ref(W * O.awq_scales_ref(a.m, 0.0)[None, :], 4, 128)
    assert np.array_equal(c0, c) and np.array_equal(s0, s)
    e_rtn = O.output_error_ref(W, awq_dequant_ref(c, s, np.ones(512), 128), X)
    assert a.err[0] == pytest.approx(e_rtn, rel=1e-12)
    assert a.err[a.best_index] == a.err.min() <= a.err[0]
    assert a.best_index == int(np.flatnonzero(a.err == a.err.min())[0])


def test_awq_codes_invariant_to_power_of_two_scale():
    W, X = make_weight(C1), make_x_bits(C1)
    m = O.channel_mean_abs_ref(X)
    s = O.awq_scales_ref(m, 0.35)
    c1, sc1 = O.group_rtn_ref(W * s[None, :], 4, 128)
    c2, sc2 = O.group_rtn_ref(W * (8.0 * s)[None, :], 4, 128)
    assert np.array_equal(c1, c2) and np.array_equal(sc2, 8.0 * sc1)


# --------------------------------------------- claims the pages make (qualitative)
def test_gptq_beats_rtn_in_distribution():
    # "GPTQ versus AWQ objectives", TL;DR and toy table: error feedback lowers
    # the calibration output error against plain rounding.
    W, X = make_weight(C1), make_x_bits(C1)
    r = O.gptq_ref_blocked(W, X)
    c, s = O.rtn_ref(W)
    e_g = O.output_error_ref(W, dequant_ref(r.codes, r.scales, r.perm, 128), X)
    e_r = O.output_error_ref(W, dequant_ref(c, s, np.arange(512), 128), X)
    assert e_g < e_r


@pytest.mark.parametrize("bits", [4, 3])
def test_toy_table_orderings(bits):
    # "GPTQ versus AWQ objectives", the toy table (output MSE, synthetic layer
    # with four outlier channels, INT4 g128): on the calibration set
    # AWQ < GPTQ < round-to-nearest; with the outliers moved to other channels
    # the order turns to round-to-nearest < AWQ < GPTQ (GPTQ's compensation
    # fitted the calibration covariance).  The tiny layer (five outlier
    # channels x20) shows both orders; the table's values are not reproduced
    # (its layer is under-specified).
    from oracle.awq import awq_dequant_ref
    W, X = make_weight(C1), make_x_bits(C1)
    X_moved = make_x_bits(C1, seed=1, permute_seed=1)   # fresh draw, outliers moved
    g = O.gptq_ref_blocked(W, X, bits=bits)
    c, s = O.rtn_ref(W, bits)
    a = O.awq_ref(W, X, bits)
    recon = {"rtn": dequant_ref(c, s, np.arange(512), 128, fp16=False),
             "gptq": dequant_ref(g.codes, g.scales, g.perm, 128, fp16=False),
             "awq": awq_dequant_ref(a.codes, a.scales, a.s, 128)}
    e = {k: O.output_error_ref(W, v, X) for k, v in recon.items()}
    e_moved = {k: O.output_error_ref(W, v, X_moved) for k, v in recon.items()}
    assert e["awq"] < e["gptq"] < e["rtn"]
    assert e_moved["rtn"] < e_moved["awq"] < e_moved["gptq"]


def _exhaustive_min(w, H, scale, qmax):
    n = w.size
    cand = np.arange(-qmax - 1, qmax + 1, dtype=np.float64)
    best = np.inf
    # enumerate the leading n-4 codes in Python, the last 4 vectorised
    tail = np.array(list(itertools.product(cand, repeat=4)))
    for head in itertools.product(cand, repeat=n - 4):
        d = np.concatenate([np.broadcast_to(np.array(head), (tail.shape[0], n - 4)), tail], 1)
        d = w[None, :] - scale * d
        e = np.einsum("ki,ij,kj->k", d, H, d)
        best = min(best, float(e.min()))
    return best


def test_exhaustive_tiny_layer_bounds_gptq():
    # out = 1, in = 8, bits = 3, one group: every code vector enumerated.
    ratios_g, ratios_r = [], []
    for seed in range(4):
        W, X = _random_layer(100 + seed, 1, 8, 24, corr=0.9)
        H = O.hessian_ref(X)
        r = O.gptq_ref(W, H=H, bits=3, g=8)
        c, s = O.rtn_ref(W, 3, 8)
        w = W[0].astype(np.float64)
        scale = r.scales[0, 0]
        e_star = _exhaustive_min(w, H, scale, 3)
        dg = w - scale * r.codes[0]
        dr = w - scale * c[0]
        e_g, e_r = dg @ H @ dg, dr @ H @ dr
        assert e_star <= e_g * (1 + 1e-12) and e_star <= e_r * (1 + 1e-12)
        ratios_g.append(e_g / e_star)
        ratios_r.append(e_r / e_star)
    assert np.median(ratios_g) <= np.median(ratios_r)


def test_hessian_sizes_printed_on_the_page():
    # "GPTQ versus AWQ objectives", the sizing block: H is in x in FP32;
    # 8,192^2 x 4 B = 268 MB and 28,672^2 x 4 B = 3.29 GB.
    assert 8192 * 8192 * 4 == 268_435_456 and round(268_435_456 / 1e6) == 268
    assert 28672 * 28672 * 4 == 3_288_334_336 and round(3_288_334_336 / 1e9, 2) == 3.29
    X = bf16_bits_from_f32(np.ones((2, 8), np.float32))
    assert O.hessian_ref(X).astype(np.float32).nbytes == 8 * 8 * 4


def test_sweep_working_precision():
    # float64 is the oracle (the default); the float32 mode runs the same loop in
    # the GPU sweep's working precision, and on the tiny layer it drifts
    # from float64 by far less than the 1e-4 tie window, deciding every code the
    # same way away from ties
    from tests.parity import fp32_drift, tie_distance
    W, X = make_weight(C1), make_x_bits(C1)
    perm, U, _ = O.gptq_prepare_ref(O.hessian_ref(X), C1.damp, False)
    Wp = W.astype(np.float64)[:, perm]
    ref = O.gptq_sweep_ref(Wp, U, 4, 128)
    c64 = O.gptq_sweep_ref(Wp, U, 4, 128, dtype=np.float64, log=False)[0]
    assert np.array_equal(c64, ref[0])
    c32, s32, v32, _ = O.gptq_sweep_ref(Wp, U, 4, 128, dtype=np.float32)
    drift = fp32_drift(Wp, U, 4, 128, ref)
    assert 0.0 < drift < 5e-5
    for k in np.nonzero((c32 != ref[0]).any(axis=1))[0]:
        j = int(np.argmax(c32[k] != ref[0][k]))  # first difference of the row: a tie
        assert tie_distance(ref[2][k, j]) < 2 * drift
