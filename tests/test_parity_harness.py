"""The GPU-vs-oracle comparison itself (tests/parity.py), on CPU.

A stand-in for the GPU is the oracle's own loop run in float32 (it decides the
same codes away from ties and may flip a few near them); planted mistakes are
made in copies of its outputs.  The comparison must accept the first and
reject every plant that is not a tie flip.
"""
import numpy as np
import pytest

import oracle as O
from tests.parity import fp32_drift, teacher_forced_compare, tie_distance
from workloads import make_weight, make_x_bits, small_spec


def _layer(bits, g, seed, out=48, inp=512, n=2048):
    spec = small_spec(out, inp, n, seed=seed, sigma_ln=0.8)
    W, X = make_weight(spec), make_x_bits(spec)
    _, U, _ = O.gptq_prepare_ref(O.hessian_ref(X), 0.01, False)
    return W.astype(np.float64), U


@pytest.mark.parametrize("bits,g", [(4, 128), (3, 64)])
def test_float32_run_passes(bits, g):
    Wp, U = _layer(bits, g, 5 + bits)
    c32, s32, _, _ = O.gptq_sweep_ref(Wp, U, bits, g, dtype=np.float32)
    ref = O.gptq_sweep_ref(Wp, U, bits, g)
    tol = max(1e-4, 2 * fp32_drift(Wp, U, bits, g, ref))
    stats, codes, scales = teacher_forced_compare(c32, Wp, U, bits, g, tie_tol=tol,
                                                  bound="forced")
    assert np.array_equal(codes, c32)                # the forced run reproduces the stand-in
    assert stats["forced"] <= 1e-3 * c32.size
    assert np.allclose(scales, s32, rtol=1e-5, atol=0)


def test_planted_code_error_is_rejected():
    Wp, U = _layer(4, 128, 11)
    c, _, v, _ = O.gptq_sweep_ref(Wp, U, 4, 128)
    # the code of row 3 farthest from a tie, moved by one
    j = int(np.argmax(tie_distance(v[3])))
    bad = c.copy()
    bad[3, j] = bad[3, j] - 1 if bad[3, j] > -8 else bad[3, j] + 1
    with pytest.raises(AssertionError, match="tie distance"):
        teacher_forced_compare(bad, Wp, U, 4, 128)


def test_planted_tie_flip_is_accepted_and_counted():
    # flip the code at the row's closest tie and let the loop continue from the
    # flipped code; with a window just wide enough to hold that tie the
    # comparison must accept it as one forced decision
    Wp, U = _layer(4, 128, 13)
    c, s, v, _ = O.gptq_sweep_ref(Wp, U, 4, 128)
    row = 7
    j = int(np.argmin(tie_distance(v[row])))           # the row's closest tie
    force = np.full_like(c, O.gptq.NO_FORCE)
    other = np.floor(v[row, j]) if c[row, j] == np.ceil(v[row, j]) else np.ceil(v[row, j])
    force[row, j] = int(np.clip(other, -8, 7))
    flipped, _, _, _ = O.gptq_sweep_ref(Wp, U, 4, 128, force=force)
    assert flipped[row, j] != c[row, j]
    # a window just wide enough for that tie: the flip is a tie decision
    tol = float(tie_distance(v[row, j])) * 1.01 + 1e-12
    stats, codes, _ = teacher_forced_compare(flipped, Wp, U, 4, 128, tie_tol=max(tol, 1e-4),
                                             bound="forced")
    assert stats["forced"] == 1 and np.array_equal(codes, flipped)
    # under the raw bound the same flip counts by every code of its row that
    # then differs: on that row alone they are more than 0.1% of the codes
    one = slice(row, row + 1)
    assert stats["mismatches"] > 1e-3 * flipped[one].size
    with pytest.raises(AssertionError, match="differ before forcing"):
        teacher_forced_compare(flipped[one], Wp[one], U, 4, 128, tie_tol=max(tol, 1e-4))


def test_planted_zero_point_error_is_rejected():
    Wp, U = _layer(3, 64, 17)
    c, s, z, zv, _, _ = O.gptq_sweep_asym_ref(Wp, U, 3, 64)
    # the zero-point of (row 2, group 3), farthest from a tie, moved by one
    assert tie_distance(zv[2, 3]) > 1e-3
    zbad = z.copy()
    zbad[2, 3] += 1 if zbad[2, 3] < 7 else -1
    with pytest.raises(AssertionError):
        teacher_forced_compare(c, Wp, U, 3, 64, gpu_zeros=zbad)


def test_scale_mismatch_is_visible_to_the_caller():
    # the harness returns the oracle's scales; a scale off by more than the
    # 1e-3 contract shows in the comparison the tests make
    Wp, U = _layer(4, 128, 19)
    c, s, _, _ = O.gptq_sweep_ref(Wp, U, 4, 128)
    _, _, scales = teacher_forced_compare(c, Wp, U, 4, 128)
    assert np.array_equal(scales, s)
    assert (np.abs(s * 1.002 - scales) / scales).max() > 1e-3


@pytest.mark.parametrize("g,sym", [(128, True), (64, True), (200, True), (64, False)])
def test_blocked_forced_equals_literal_forced(g, sym):
    # the wide layers' forced re-runs use the blocked sweep: with the same
    # forced sites (codes, and zero-points for asymmetric groups) it must
    # reproduce the literal loop
    Wp, U = _layer(4, g, 23, out=12, inp=520, n=2100)
    rng = np.random.default_rng(3)
    force = np.full(Wp.shape, O.gptq.NO_FORCE, dtype=np.int16)
    sites = rng.integers(0, Wp.size, 20)
    force.flat[sites] = rng.integers(-8, 8, 20)
    if sym:
        c1, s1, v1, _ = O.gptq_sweep_ref(Wp, U, 4, g, force=force)
        c2, s2, v2 = O.gptq_sweep_blocked_ref(Wp, U, 4, g, force=force)
    else:
        force = np.clip(force, -1, 15).astype(np.int16)
        force[force == -1] = O.gptq.NO_FORCE
        fz = np.full((Wp.shape[0], -(-Wp.shape[1] // g)), O.gptq.NO_FORCE, dtype=np.int16)
        fz[2, 3] = 5
        c1, s1, z1, zv1, v1, _ = O.gptq_sweep_asym_ref(Wp, U, 4, g, force=force, force_zero=fz)
        c2, s2, z2, v2, zv2 = O.gptq_sweep_blocked_asym_ref(Wp, U, 4, g, force=force,
                                                             force_zero=fz)
        assert np.array_equal(z1, z2) and z2[2, 3] == 5
        assert np.allclose(zv1, zv2, rtol=0, atol=1e-9)
    assert np.array_equal(c1, c2)
    assert np.array_equal(c1[force != O.gptq.NO_FORCE], force[force != O.gptq.NO_FORCE])
    assert np.allclose(s1, s2, rtol=1e-12, atol=0)
    assert np.allclose(v1, v2, rtol=0, atol=1e-9)
