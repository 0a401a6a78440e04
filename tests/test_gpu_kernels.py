"""Per-step parity of the CUDA path against the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from tests.parity import (REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu)
from workloads import C1, bf16_bits_from_f32, make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _layer(out, inp, n, seed=0, **kw):
    spec = small_spec(out, inp, n, seed=seed, **kw)
    return make_weight(spec), make_x_bits(spec)


@pytest.mark.parametrize("n,inp", [(2048, 512), (1000, 136), (77, 264), (4100, 1032), (64, 8),
                                   (12300, 264)])
def test_hessian_matches_exact(n, inp):
    W, X = _layer(8, inp, n, seed=n + inp)
    H = np.triu(piq.hessian(to_gpu_x(X)).cpu().numpy()).astype(np.float64)
    Hx = O.hessian_ref(X)
    d = np.sqrt(np.outer(np.diag(Hx), np.diag(Hx)))
    iu = np.triu_indices(inp)
    err = np.abs(H - Hx)[iu] / np.maximum(d[iu], 1e-30)
    assert err.max() < 2e-5, err.max()


def test_hessian_accumulates():
    W, X = _layer(8, 264, 600, seed=3)
    Xg = to_gpu_x(X)
    H = piq.hessian(Xg[:300].contiguous())
    piq.hessian(Xg[300:].contiguous(), H=H, accumulate=True)
    Hx = O.hessian_ref(X)
    iu = np.triu_indices(264)
    d = np.sqrt(np.outer(np.diag(Hx), np.diag(Hx)))[iu]
    assert (np.abs(H.cpu().numpy().astype(np.float64) - Hx)[iu] / d).max() < 2e-5


@pytest.mark.parametrize("inp,act", [(512, False), (520, False), (136, True), (1032, True)])
def test_upper_factor_matches_oracle(inp, act):
    W, X = _layer(8, inp, 4 * inp, seed=inp)
    Hx = O.hessian_ref(X)
    perm, Ux, lam_x = O.gptq_prepare_ref(Hx, 0.01, act)
    Hg = torch.from_numpy(Hx.astype(np.float32)).cuda()
    pg = torch.from_numpy(perm.astype(np.int32)).cuda() if act else None
    U, lam = piq.upper_factor(Hg, 0.01, perm=pg)
    U = U.cpu().numpy().astype(np.float64)
    assert rel(lam, lam_x) < 1e-5
    assert np.count_nonzero(np.tril(U, -1)) == 0
    scale = np.abs(Ux).max(axis=1, keepdims=True)
    e_u = (np.abs(U - Ux) / scale).max()
    Hd, _ = O.damped_ref(Hx[np.ix_(perm, perm)], 0.01)
    e_inv = np.abs(U.T @ U @ Hd - np.eye(inp)).max()
    print(f"upper factor in={inp} act={act}: max |dU|/rowmax {e_u:.3g}, |U^T U H_d - I| {e_inv:.3g}")
    # an FP32 factorization (this step entry's precision): errors of a few
    # units of float32 rounding times the conditioning of these layers
    assert e_u < 2e-5
    assert e_inv < 1e-4


@pytest.mark.parametrize("inp", [512, 1032])
def test_fp32_step_entries_stay_on_the_tensor_cores(inp):
    # the FP32 factor and sweep step entries: 16-byte aligned operands, so no
    # product falls back to the SIMT kernel
    W, X = _layer(16, inp, 3 * inp, seed=inp + 1)
    Hx = O.hessian_ref(X)
    f0 = piq.simt_gemm_fallbacks()
    U, _ = piq.upper_factor(torch.from_numpy(Hx.astype(np.float32)).cuda(), 0.01)
    piq.gptq_sweep(to_gpu_w(W), U, 4, 128)
    assert piq.simt_gemm_fallbacks() == f0


def test_not_positive_definite_reports_status():
    H = torch.zeros(64, 64, device="cuda")
    with pytest.raises(piq.PiqError) as e:
        piq.upper_factor(H, 0.01)
    assert e.value.status == piq.PIQ_ERR_NOT_PD


@pytest.mark.parametrize("out,inp,g,bits", [(256, 512, 128, 4), (129, 520, 96, 4),
                                            (64, 600, 200, 3), (33, 264, 32, 4),
                                            (40, 200, 1000, 3), (17, 136, 128, 2)])
def test_sweep_given_u(out, inp, g, bits):
    # Same (fp32) U on both sides isolates the sweep from the factorization.
    W, X = _layer(out, inp, 3 * inp, seed=out * inp)
    Hx = O.hessian_ref(X)
    _, Ux, _ = O.gptq_prepare_ref(Hx, 0.01, False)
    U32 = np.ascontiguousarray(Ux, dtype=np.float32)
    codes, qscale = piq.gptq_sweep(to_gpu_w(W), torch.from_numpy(U32).cuda(), bits, g)
    # the step entry runs the sweep in FP32: a tie flip may change the rest of
    # its row, so the forced sites (not the raw differences) are bounded
    stats, c_ref, s_ref = teacher_forced_compare(codes.cpu().numpy(), W.astype(np.float64),
                                                 U32.astype(np.float64), bits, g,
                                                 bound="forced")
    qs = qscale.cpu().numpy().astype(np.float64)
    assert (np.abs(qs - s_ref) / np.maximum(s_ref, 1e-30)).max() < REL_TOL, stats


def test_output_error_gemm_matches_oracle():
    # output error of an RTN-packed layer; several tiles plus ragged edges
    W, X = _layer(300, 520, 1500, seed=9)
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    qw, sc = piq.rtn_quantize_layer(Wg, 4, 128)
    e = piq.layer_output_error(Wg, qw, sc, Xg, 4, 128)
    codes = unpack_gpu(qw, 4)
    What = codes * np.repeat(sc.cpu().numpy().astype(np.float64), 128, axis=1)[:, :520]
    ex = O.output_error_ref(W, What, X)
    assert rel(e, ex) < REL_TOL  # bf16 rounding of W - What is the dominant term


@pytest.mark.parametrize("out,inp,n", [
    (300, 520, 1500),  # n small against in: the direct product X D^T
    (520, 264, 4100),  # n large against in and out: the route through H = X^T X
])
def test_output_error_routes(out, inp, n):
    # a packed layer with act-order groups and AWQ channel scales, on ragged sizes
    W, X = _layer(out, inp, n, seed=out + n, sigma_ln=1.0, n_outlier=3, outlier_gain=30.0)
    rng = np.random.default_rng(out)
    g, bits = 64, 4
    ng = -(-inp // g)
    perm = rng.permutation(inp)
    g_idx = np.empty(inp, np.int32)
    g_idx[perm] = np.arange(inp) // g
    s = np.exp(rng.normal(0.0, 0.5, inp)).astype(np.float32)
    codes = rng.integers(-8, 8, (out, inp))
    sc16 = rng.uniform(0.002, 0.01, (out, ng)).astype(np.float16)
    qw = torch.from_numpy(O.pack_ref(codes, bits).view(np.int32)).cuda()
    e = piq.layer_output_error(to_gpu_w(W), qw, torch.from_numpy(sc16).cuda(),
                               to_gpu_x(X), bits, g,
                               g_idx=torch.from_numpy(g_idx).cuda(),
                               s=torch.from_numpy(s).cuda())
    What = codes * sc16.astype(np.float64)[:, g_idx] / s.astype(np.float64)
    assert rel(e, O.output_error_ref(W, What, X)) < REL_TOL


def test_rtn_matches_oracle():
    W, _ = _layer(129, 520, 16, seed=4)
    for bits, g in ((4, 128), (3, 64), (4, 96), (2, 520)):
        qw, sc = piq.rtn_quantize_layer(to_gpu_w(W), bits, g)
        c, s = O.rtn_ref(W, bits, g)
        got = unpack_gpu(qw, bits)
        mism = got != c
        if mism.any():  # only at fp32-vs-fp64 rounding ties
            qmax = 2 ** (bits - 1) - 1
            cols = np.arange(520) // g
            v = W.astype(np.float64) / s[:, cols]
            from tests.parity import tie_distance
            assert (tie_distance(v[mism]) < 1e-4).all()
            assert mism.mean() < 1e-3
        assert np.array_equal(sc.cpu().numpy(), s.astype(np.float16))
