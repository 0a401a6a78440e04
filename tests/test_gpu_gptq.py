"""End-to-end GPTQ parity (gptq_quantize_layer) against the FP64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from oracle.pack import dequant_ref
from tests.parity import REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import C1, make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _check_layer(W, X, bits, g, act_order, damp=0.01):
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), bits=bits, g=g, damp=damp,
                                  act_order=act_order)
    perm_gpu = out.perm.cpu().numpy()
    Hx = O.hessian_ref(X)
    perm, U, lam = O.gptq_prepare_ref(Hx, damp, act_order)
    assert np.array_equal(perm_gpu, perm)
    assert np.array_equal(out.g_idx.cpu().numpy(), O.g_idx_ref(perm, g))
    codes_mem = unpack_gpu(out.qweight, bits)
    codes_q = codes_mem[:, perm]
    Wp = W.astype(np.float64)[:, perm]
    stats, c_ref, s_ref = teacher_forced_compare(codes_q, Wp, U, bits, g)
    sc = out.scales.cpu().numpy().astype(np.float64)
    s16 = s_ref.astype(np.float16).astype(np.float64)
    assert (np.abs(sc - s16) / np.maximum(s16, 1e-30)).max() < REL_TOL
    e_ref = O.output_error_ref(W, dequant_ref(c_ref, s_ref, perm, g), X)
    assert rel(out.err, e_ref) < REL_TOL, (out.err, e_ref)
    return stats, out, e_ref


def test_tiny_layer_config():
    # W 256x512 ~N(0, 0.02^2); X 2048x512 with 5 channels x20; 4-bit, g128
    W, X = make_weight(C1), make_x_bits(C1)
    stats, out, e = _check_layer(W, X, 4, 128, False)
    c, s = O.rtn_ref(W)
    e_rtn = O.output_error_ref(W, dequant_ref(c, s, np.arange(512), 128), X)
    assert out.err < e_rtn


@pytest.mark.parametrize("out,inp,n,g,bits,act", [
    (129, 520, 1500, 128, 4, False),    # ragged rows, ragged last block
    (64, 600, 1800, 200, 3, False),     # group wider than a block, not a multiple
    (100, 264, 900, 40, 4, True),       # act-order, small groups
    (33, 1032, 3000, 128, 3, True),     # act-order, INT3
    (48, 136, 500, 1000, 4, False),     # one group per row
    (8, 8, 64, 8, 2, False),            # smallest layer, 2-bit
])
def test_layer_variants(out, inp, n, g, bits, act):
    spec = small_spec(out, inp, n, seed=out + inp + n, sigma_ln=0.8)
    _check_layer(make_weight(spec), make_x_bits(spec), bits, g, act)


def test_diagonal_hessian_equals_rtn():
    # one-hot rows: X^T X exactly diagonal, so GPTQ reduces to group RTN
    rng = np.random.default_rng(7)
    inp, n = 256, 2048
    Xf = np.zeros((n, inp), dtype=np.float32)
    Xf[np.arange(n), rng.integers(0, inp, n)] = 1.0
    from workloads import bf16_bits_from_f32
    X = bf16_bits_from_f32(Xf)
    W = make_weight(C1)[:64, :inp].copy()
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), bits=4, g=64)
    qw, sc = piq.rtn_quantize_layer(to_gpu_w(W), 4, 64)
    assert torch.equal(out.qweight, qw) and torch.equal(out.scales, sc)


def test_deterministic():
    W, X = make_weight(C1), make_x_bits(C1)
    a = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X))
    b = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X))
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)
    assert a.err == b.err


def test_zero_inputs_not_positive_definite():
    W = make_weight(C1)
    X = np.zeros((256, 512), dtype=np.uint16)
    with pytest.raises(piq.PiqError) as e:
        piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X))
    assert e.value.status == piq.PIQ_ERR_NOT_PD
    # the status is per call: the next call on the same context succeeds
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(make_x_bits(C1)))
    assert np.isfinite(out.err) and out.err > 0


def test_workspace_too_small():
    W, X = make_weight(C1), make_x_bits(C1)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    import ctypes
    lib = piq.load_library()
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    qw = torch.empty(256, 64, dtype=torch.int32, device="cuda")
    sc = torch.empty(256, 4, dtype=torch.float16, device="cuda")
    rc = lib.gptq_quantize_layer(ctypes.c_void_p(Wg.data_ptr()), 256, 512,
                                 ctypes.c_void_p(Xg.data_ptr()), 2048, 4, 128, 0.01, 0,
                                 ctypes.c_void_p(qw.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
                                 None, None, None, ctypes.c_void_p(ws.data_ptr()), 1024, None)
    assert rc == piq.PIQ_ERR_WORKSPACE_TOO_SMALL


def test_shifted_inputs_error_entry():
    # the held-out / shifted score goes through piq_layer_output_error
    spec = small_spec(64, 256, 1024, seed=5, sigma_ln=1.0, n_outlier=3, outlier_gain=30.0)
    W, X = make_weight(spec), make_x_bits(spec)
    X2 = make_x_bits(spec, seed=1, permute_seed=1)
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), g=128)
    e2 = piq.layer_output_error(to_gpu_w(W), out.qweight, out.scales, to_gpu_x(X2), 4, 128,
                                g_idx=out.g_idx)
    codes = unpack_gpu(out.qweight, 4)
    What = codes * np.repeat(out.scales.cpu().numpy().astype(np.float64), 128, axis=1)
    assert rel(e2, O.output_error_ref(W, What, X2)) < REL_TOL


def test_clip_example_step_entry(golden):
    # the hand-worked sweep where the clip binds at +qmax and -qmax-1, through
    # the sweep step entry with the example's U
    d = golden("sweep_clip_example.json")
    U = torch.tensor(d["U"], dtype=torch.float32, device="cuda")
    w = torch.tensor([d["w"]], dtype=torch.float32, device="cuda")
    codes, qscale = piq.gptq_sweep(w, U, d["bits"], d["g"])
    assert codes.cpu().numpy()[0].tolist() == d["codes"]
    assert qscale.cpu().numpy()[0].tolist() == d["scales"]


@pytest.mark.parametrize("bits,act", [(2, False), (3, True), (2, True)])
def test_clip_binds(bits, act):
    # at 2 and 3 bits the error feedback pushes many weights past the code
    # range; the oracle clips them and the GPU must decide the same codes
    spec = small_spec(96, 520, 2000, seed=40 + bits, sigma_ln=1.0, n_outlier=5,
                      outlier_gain=30.0)
    W, X = make_weight(spec), make_x_bits(spec)
    Hx = O.hessian_ref(X)
    perm, U, _ = O.gptq_prepare_ref(Hx, 0.01, act)
    _, _, v, _ = O.gptq_sweep_ref(W.astype(np.float64)[:, perm], U, bits, 128)
    qmax = 2 ** (bits - 1) - 1
    assert (np.round(v) > qmax).sum() + (np.round(v) < -qmax - 1).sum() > 0
    _check_layer(W, X, bits, 128, act)


@pytest.mark.parametrize("act", [False, True])
def test_dead_input_channel(act):
    # an input channel that is zero in every sample: H_jj = 0 and its row and
    # column vanish; damping keeps H_d positive definite (page 1, damping)
    spec = small_spec(64, 264, 1000, seed=51, sigma_ln=0.8)
    W, X = make_weight(spec), make_x_bits(spec).copy()
    X[:, 17] = 0
    X[:, 200] = 0
    assert O.hessian_ref(X)[17, 17] == 0.0
    _check_layer(W, X, 4, 128, act)


def test_zero_weight_rows():
    # an all-zero row and a row with an all-zero group: scale 0, codes 0
    spec = small_spec(40, 384, 1200, seed=52, sigma_ln=0.8)
    W, X = make_weight(spec).copy(), make_x_bits(spec)
    W[5] = 0.0
    W[9, 128:256] = 0.0
    stats, out, _ = _check_layer(W, X, 4, 128, False)
    codes = unpack_gpu(out.qweight, 4)
    sc = out.scales.cpu().numpy()
    assert (codes[5] == 0).all() and (sc[5] == 0).all()
