"""AWQ scale-search parity (awq_search_layer) against the FP64 oracle."""
import numpy as np
import pytest

import oracle as O
import post_int4_weight_gptq_b200 as piq
from tests.parity import REL_TOL, rel, tie_distance, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import AWQ_GRID, C1, make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _check(W, X, bits, g, grid=AWQ_GRID):
    res = piq.awq_search_layer(to_gpu_w(W), to_gpu_x(X), bits=bits, g=g, alpha_grid=grid)
    ref = O.awq_ref(W, X, bits, g, grid=list(grid))
    errs = np.array(res.err_per_alpha)
    assert (np.abs(errs - ref.err) / ref.err).max() < REL_TOL
    srt = np.sort(ref.err)
    tie_ambiguous = len(srt) > 1 and (srt[1] - srt[0]) / srt[0] < 1e-4
    if not tie_ambiguous:
        assert res.best_alpha == np.float32(ref.best_alpha)
    a = res.best_alpha
    s = O.awq_scales_ref(ref.m, float(a))
    assert np.allclose(res.s.cpu().numpy(), s, rtol=1e-6)
    c, sc = O.group_rtn_ref(W.astype(np.float64) * s[None, :], bits, g)
    got = unpack_gpu(res.qweight, bits)
    mism = got != c
    if mism.any():
        cols = np.arange(W.shape[1]) // g
        v = W.astype(np.float64) * s[None, :] / np.where(sc > 0, sc, 1)[:, cols]
        assert (tie_distance(v[mism]) < 1e-4).all() and mism.mean() < 1e-3
    s16 = res.scales.cpu().numpy().astype(np.float64)
    ref16 = sc.astype(np.float16).astype(np.float64)
    assert (np.abs(s16 - ref16) / np.maximum(ref16, 1e-30)).max() < REL_TOL
    return res, ref


def test_tiny_layer():
    W, X = make_weight(C1), make_x_bits(C1)
    res, ref = _check(W, X, 4, 128)
    assert res.err_per_alpha[ref.best_index] <= res.err_per_alpha[0]


@pytest.mark.parametrize("out,inp,n,g,bits", [(129, 520, 700, 128, 4), (64, 264, 300, 64, 3),
                                              (300, 136, 2000, 136, 4)])
def test_variants(out, inp, n, g, bits):
    spec = small_spec(out, inp, n, seed=inp, n_outlier=max(1, inp // 50), outlier_gain=50.0)
    _check(make_weight(spec), make_x_bits(spec), bits, g)


def test_alpha_zero_is_rtn():
    W, X = make_weight(C1), make_x_bits(C1)
    res = piq.awq_search_layer(to_gpu_w(W), to_gpu_x(X), alpha_grid=(0.0,))
    qw, sc = piq.rtn_quantize_layer(to_gpu_w(W))
    assert res.best_alpha == 0.0
    assert (res.qweight == qw).all() and (res.scales == sc).all()
    assert (res.s == 1).all()
