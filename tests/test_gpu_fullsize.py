"""Parity at the full workload sizes, in the launch configuration bench.py uses.

The oracle builds H and U in float64 on the host cores, sweeps every row with
its blocked loop (the same arithmetic as the literal one) and then:
  * codes: all rows, compared teacher-forced with the GPU's codes under the
    contract of tests/parity.py (at most 0.1% of the codes differ before
    forcing, every differing decision within 1e-4 of a rounding tie);
  * scales: all rows, within 1e-3 (the GPU stores fp16, the oracle is rounded
    the same way);
  * output error: the oracle's codes (after forcing) dequantized with fp16
    scales, scored in float64 on X (and on the shifted X' for q_proj).
That runs by default for the q_proj and act-order down_proj layers (tens of
seconds of host time each).  For the 70B-shaped layer, H (32768 x 28672^2)
and U (28672^3) alone take several minutes of host float64, so by default the
GPU runs it at full size and the oracle checks what it computes cheaply: the
packed output on sampled rows and samples (the error kernel at K = 28672),
GPTQ against round-to-nearest on that sample, and the layout.  The complete
comparison runs with PIQ_FULLSIZE_SLOW=1 (or split across hosts with
tests/fullsize_split.py: dump on the GPU machine, check anywhere).
"""
import os

import numpy as np
import pytest

import oracle as O
import post_int4_weight_gptq_b200 as piq
from oracle.gptq import gptq_sweep_blocked_ref
from oracle.pack import dequant_ref
from tests.oracle_pool import sweep_rows
from tests.parity import REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import AWQ_GRID, C2, C3, C4, C5, make_weight, make_x_bits

pytestmark = [pytest.mark.gpu]
SLOW = os.environ.get("PIQ_FULLSIZE_SLOW") == "1"

_cache = {}


def _layer(spec):
    """(W, X, perm, U) of a workload, the float64 H and U computed once."""
    if spec.name not in _cache:
        _cache.clear()  # one large layer at a time
        W = make_weight(spec)
        X = make_x_bits(spec)
        # the symmetric rank-k H and U = inv(R): the same matrices as the
        # listing's product and cholesky(inv(H_d)).T, in fewer host flops
        # (pinned in test_oracle_properties)
        H = O.hessian_syrk_ref(X)
        perm, U, _ = O.gptq_prepare_ref(H, spec.damp, spec.act_order, via_r=True)
        del H
        _cache[spec.name] = (W, X, perm, U)
    return _cache[spec.name]


def _gptq_full(spec, bits=None, shift=False):
    bits = spec.bits if bits is None else bits
    W, X, perm, U = _layer(spec)
    f0 = piq.simt_gemm_fallbacks()
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), bits=bits, g=spec.g,
                                  damp=spec.damp, act_order=spec.act_order)
    assert piq.simt_gemm_fallbacks() == f0  # every product on the tensor cores
    e2_gpu = X2 = None
    if shift:
        X2 = make_x_bits(spec, seed=spec.seed + 1, permute_seed=spec.seed + 1)
        e2_gpu = piq.layer_output_error(to_gpu_w(W), out.qweight, out.scales, to_gpu_x(X2), bits,
                                        spec.g, g_idx=out.g_idx)
    codes_mem = unpack_gpu(out.qweight, bits)
    sc_gpu = out.scales.cpu().numpy().astype(np.float64)
    assert np.array_equal(out.perm.cpu().numpy(), perm)
    assert np.array_equal(out.g_idx.cpu().numpy(), O.g_idx_ref(perm, spec.g))
    Wp = W.astype(np.float64)[:, perm]
    ref = sweep_rows(Wp, U, bits, spec.g)  # all rows, chunks on the host cores
    stats, c_ref, s_ref = teacher_forced_compare(codes_mem[:, perm], Wp, U, bits, spec.g,
                                                 ref=ref)
    s16 = s_ref.astype(np.float16).astype(np.float64)
    live = s16 > 0
    assert (np.abs(sc_gpu[live] - s16[live]) / s16[live]).max() < REL_TOL
    What = dequant_ref(c_ref, s_ref, perm, spec.g)
    e_ref = O.output_error_ref(W, What, X)
    assert rel(out.err, e_ref) < REL_TOL, (out.err, e_ref)
    if shift:
        e2_ref = O.output_error_ref(W, What, X2)
        assert rel(e2_gpu, e2_ref) < REL_TOL, (e2_gpu, e2_ref)
    print(f"{spec.name} {bits}-bit: {stats}")
    return stats


def test_q_proj_7b_full():
    # W 4096x4096, X 131072x4096 (lognormal channel stds, 41 channels x30),
    # 4-bit g128; also the error on the shifted X'
    _gptq_full(C2, shift=True)


def test_down_proj_7b_act_order_full():
    # W 4096x11008, X 65536x11008 Student-t(4), act-order
    _gptq_full(C3)


@pytest.mark.parametrize("bits", [4, 3])
def test_down_proj_70b_full(bits):
    # W 8192x28672, X 32768x28672, H 28672^2 (3.29 GB in fp32)
    _gptq_full(C4, bits=bits)


def test_down_proj_70b_sampled():
    """The 70B-shaped layer (W 8192x28672, X 32768x28672) at full size on the
    GPU; the oracle scores the packed output on 64 sampled rows and 2048
    sampled calibration rows: its float64 error of the dequantized codes
    equals the GPU error kernel on the same slices (K = 28672), and is below
    the round-to-nearest error of the same rows."""
    import torch
    _cache.clear()
    spec = C4
    W, X = make_weight(spec), make_x_bits(spec)
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), bits=spec.bits, g=spec.g,
                                  damp=spec.damp, act_order=spec.act_order)
    inp = W.shape[1]
    assert np.array_equal(out.perm.cpu().numpy(), np.arange(inp))
    assert np.array_equal(out.g_idx.cpu().numpy(), np.arange(inp) // spec.g)
    sc = out.scales.cpu().numpy().astype(np.float64)
    assert np.isfinite(sc).all() and (sc > 0).all()
    assert np.isfinite(out.err) and out.err > 0
    rng = np.random.default_rng(2024)
    rows = np.sort(rng.choice(W.shape[0], 64, replace=False))
    samples = np.sort(rng.choice(X.shape[0], 2048, replace=False))
    Ws, Xs = W[rows], X[samples]
    codes = unpack_gpu(out.qweight, spec.bits)[rows]
    What = dequant_ref(codes, sc[rows], np.arange(inp), spec.g)
    e_ref = O.output_error_ref(Ws, What, Xs)
    qw = out.qweight[torch.from_numpy(rows).cuda()].contiguous()
    s_rows = out.scales[torch.from_numpy(rows).cuda()].contiguous()
    e_gpu = piq.layer_output_error(to_gpu_w(Ws), qw, s_rows, to_gpu_x(Xs), spec.bits, spec.g,
                                   g_idx=out.g_idx)
    assert rel(e_gpu, e_ref) < REL_TOL, (e_gpu, e_ref)
    c_rtn, s_rtn = O.rtn_ref(Ws, spec.bits, spec.g)
    e_rtn = O.output_error_ref(Ws, dequant_ref(c_rtn, s_rtn, np.arange(inp), spec.g), Xs)
    assert e_ref < e_rtn, (e_ref, e_rtn)
    print(f"{spec.name}: sampled error {e_ref:.6g} (GPU kernel {e_gpu:.6g}), RTN {e_rtn:.6g}")


def test_awq_8192_full():
    _cache.clear()
    W, X = make_weight(C5), make_x_bits(C5)
    res = piq.awq_search_layer(to_gpu_w(W), to_gpu_x(X), C5.bits, C5.g, AWQ_GRID)
    ref = O.awq_ref(W, X, C5.bits, C5.g, grid=list(AWQ_GRID))
    errs = np.array(res.err_per_alpha)
    assert (np.abs(errs - ref.err) / ref.err).max() < REL_TOL
    srt = np.sort(ref.err)
    assert (srt[1] - srt[0]) / srt[0] >= 1e-4  # not tie-ambiguous on this layer
    assert res.best_alpha == np.float32(ref.best_alpha)
    # the returned per-channel scales and the codes at the chosen alpha
    s_ref = O.awq_scales_ref(O.channel_mean_abs_ref(X), ref.best_alpha)
    assert (np.abs(res.s.cpu().numpy() - s_ref) / s_ref).max() < 1e-6


def _widened_full(spec, s=None, sym=True, sample_rows=48):
    """Full-size parity of the AWQ-scaled call (channel scales s) or of
    asymmetric groups (sym=False) on one layer, as _gptq_full does for plain
    GPTQ.  The oracle's Hessian is that of X diag(1/s), summed over row chunks."""
    from oracle.gptq import gptq_sweep_asym_ref, gptq_sweep_blocked_asym_ref
    W, X = make_weight(spec), make_x_bits(spec)
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    if s is not None:
        import torch
        out = piq.awq_gptq_quantize_layer(Wg, Xg, torch.from_numpy(s).cuda(), spec.bits, spec.g,
                                          spec.damp, spec.act_order)
    else:
        out = piq.gptq_quantize_layer(Wg, Xg, spec.bits, spec.g, spec.damp, spec.act_order,
                                      sym=sym)
    bits, g = spec.bits, spec.g
    s64 = np.ones(W.shape[1]) if s is None else s.astype(np.float64)
    H = np.zeros((W.shape[1], W.shape[1]))
    for r0 in range(0, X.shape[0], 8192):
        xc = O.x_to_f64(X[r0:r0 + 8192]) / s64[None, :]
        H += xc.T @ xc
    perm, U, _ = O.gptq_prepare_ref(H, spec.damp, spec.act_order)
    del H
    assert np.array_equal(out.perm.cpu().numpy(), perm)
    Wp = (W.astype(np.float64) * s64[None, :])[:, perm]
    rows = np.sort(np.random.default_rng(123).choice(W.shape[0], sample_rows, replace=False))
    g_idx = O.g_idx_ref(perm, g)
    if sym:
        codes_q = unpack_gpu(out.qweight, bits)[rows][:, perm]
        stats, _, s_ref = teacher_forced_compare(codes_q, Wp[rows], U, bits, g)  # noqa
    else:
        z_gpu = out.zeros.cpu().numpy().astype(np.int16)
        u = unpack_gpu(out.qweight, bits) + 2 ** (bits - 1)
        codes_q = (u - z_gpu[:, g_idx])[rows][:, perm]
        stats, _, s_ref, _ = teacher_forced_compare(codes_q, Wp[rows], U, bits, g,
                                                    gpu_zeros=z_gpu[rows])
    sc_gpu = out.scales.cpu().numpy().astype(np.float64)[rows]
    s16 = s_ref.astype(np.float16).astype(np.float64)
    live = s16 > 0
    assert (np.abs(sc_gpu[live] - s16[live]) / s16[live]).max() < REL_TOL
    if sym:
        c_all, sc_all, _ = gptq_sweep_blocked_ref(Wp, U, bits, g)
    else:
        c_all, sc_all, _, _, _ = gptq_sweep_blocked_asym_ref(Wp, U, bits, g)
    What = dequant_ref(c_all, sc_all, perm, g) / s64[None, :]
    e_ref = O.output_error_ref(W, What, X)
    assert rel(out.err, e_ref) < REL_TOL, (out.err, e_ref)
    return stats


@pytest.mark.skipif(not SLOW, reason="minutes of host float64; PIQ_FULLSIZE_SLOW=1")
def test_q_proj_7b_awq_scaled_full():
    # the q_proj layer through awq_gptq_quantize_layer with seeded channel scales
    from workloads import make_channel_scales
    _widened_full(C2, s=make_channel_scales(C2.inp, 7, 0.5))


@pytest.mark.skipif(not SLOW, reason="minutes of host float64; PIQ_FULLSIZE_SLOW=1")
def test_q_proj_7b_asym_full():
    _widened_full(C2, sym=False)
