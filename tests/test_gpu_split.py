"""The single-layer split on the GPU: statistics of sample shards, their sum,
and GPTQ of row blocks from the summed H (the two C-ABI calls the split uses).

On one GPU the ranks' work is done one after the other; with two or more GPUs
the split itself runs over NCCL and must give the same bits as that.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from oracle.pack import dequant_ref
from post_int4_weight_gptq_b200.split import row_range, sample_range
from tests.parity import REL_TOL, rel, teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layer(seed=61):
    spec = small_spec(100, 520, 3000, seed=seed, sigma_ln=0.9, n_outlier=5, outlier_gain=25.0)
    return make_weight(spec), make_x_bits(spec)


def _emulated_split(W, X, world, act):
    """The split's steps for `world` ranks, one after the other on this GPU."""
    Hs, sqs = [], []
    for r in range(world):
        s0, s1 = sample_range(X.shape[0], r, world)
        H, sq = piq.layer_statistics(to_gpu_x(X[s0:s1]), want_sumsq=True)
        Hs.append(H)
        sqs.append(sq)
    H = Hs[0].clone()
    sq = sqs[0].clone()
    for t in Hs[1:]:
        H += t
    for t in sqs[1:]:
        sq += t
    parts = []
    for r in range(world):
        r0, r1 = row_range(W.shape[0], r, world)
        parts.append(piq.gptq_rows_from_h(to_gpu_w(W[r0:r1]), H, sq, bits=4, g=128,
                                          act_order=act))
    return parts, H


@pytest.mark.parametrize("act", [False, True])
def test_split_meets_the_contract(act):
    W, X = _layer()
    parts, _ = _emulated_split(W, X, 2, act)
    codes = np.concatenate([unpack_gpu(p.qweight, 4) for p in parts])
    scales = np.concatenate([p.scales.cpu().numpy() for p in parts]).astype(np.float64)
    err = sum(p.err for p in parts)
    perm = parts[0].perm.cpu().numpy()
    assert all(np.array_equal(p.perm.cpu().numpy(), perm) for p in parts)
    Hx = O.hessian_ref(X)
    perm_ref, U, _ = O.gptq_prepare_ref(Hx, 0.01, act)
    assert np.array_equal(perm, perm_ref)
    Wp = W.astype(np.float64)[:, perm]
    stats, c_ref, s_ref = teacher_forced_compare(codes[:, perm], Wp, U, 4, 128)
    s16 = s_ref.astype(np.float16).astype(np.float64)
    assert (np.abs(scales - s16) / np.maximum(s16, 1e-30)).max() < REL_TOL
    e_ref = O.output_error_ref(W, dequant_ref(c_ref, s_ref, perm, 128), X)
    assert rel(err, e_ref) < REL_TOL, (err, e_ref)


def test_row_blocks_equal_one_call_on_all_rows():
    # given H, rows are independent: blocks of rows give the bits of one call
    W, X = _layer(62)
    parts, H = _emulated_split(W, X, 3, False)
    whole = piq.gptq_rows_from_h(to_gpu_w(W), H, None, bits=4, g=128)
    assert torch.equal(torch.cat([p.qweight for p in parts]), whole.qweight)
    assert torch.equal(torch.cat([p.scales for p in parts]), whole.scales)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from post_int4_weight_gptq_b200.split import gptq_layer_split
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    W, X = _layer()
    s0, s1 = sample_range(X.shape[0], rank, world)
    qw, sc, perm, g_idx, err = gptq_layer_split(to_gpu_w(W, f"cuda:{rank}"),
                                                to_gpu_x(X[s0:s1], f"cuda:{rank}"), bits=4, g=128)
    q.put((rank, qw.cpu().numpy(), sc.cpu().numpy(), err))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
@pytest.mark.timeout(600)
def test_two_gpus_give_the_bits_of_the_emulated_split():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=500) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W, X = _layer()
    parts, _ = _emulated_split(W, X, 2, False)
    qw = torch.cat([p.qweight for p in parts]).cpu().numpy()
    sc = torch.cat([p.scales for p in parts]).cpu().numpy()
    for _, qw_r, sc_r, err_r in res:
        assert np.array_equal(qw_r, qw) and np.array_equal(sc_r, sc)
        assert err_r == pytest.approx(sum(p.err for p in parts), rel=1e-12)


# ---------------------------------------------------------------- AWQ, rows split

GRID = tuple(k / 20.0 for k in range(20))


def _emulated_awq_split(W, X, world):
    """awq_layer_split's steps for `world` ranks, one after the other on this GPU."""
    from post_int4_weight_gptq_b200.split import first_minimum
    Xg = to_gpu_x(X)
    blocks = [row_range(W.shape[0], r, world) for r in range(world)]
    res = [piq.awq_search_layer(to_gpu_w(W[r0:r1]), Xg, bits=4, g=128, alpha_grid=GRID)
           for r0, r1 in blocks]
    errs = [sum(r.err_per_alpha[k] for r in res) for k in range(len(GRID))]
    k = first_minimum(errs)
    for i, (r0, r1) in enumerate(blocks):
        if first_minimum(res[i].err_per_alpha) != k:
            res[i] = piq.awq_search_layer(to_gpu_w(W[r0:r1]), Xg, bits=4, g=128,
                                          alpha_grid=[GRID[k]])
    return GRID[k], res, errs


def test_awq_row_blocks_equal_one_call_on_all_rows():
    # s depends on X only and each alpha's error is a sum over rows: blocks of
    # rows scored apart and summed choose the whole layer's alpha, and give its bits
    W, X = _layer(63)
    alpha, parts, errs = _emulated_awq_split(W, X, 3)
    whole = piq.awq_search_layer(to_gpu_w(W), to_gpu_x(X), bits=4, g=128, alpha_grid=GRID)
    assert np.float32(alpha) == np.float32(whole.best_alpha)
    # the error GEMM sums tiles of rows in FP32 before FP64: blocks of rows round
    # apart (~1e-9 relative here), far inside the gaps between alphas
    assert np.allclose(errs, whole.err_per_alpha, rtol=1e-6, atol=0)
    assert all(torch.equal(p.s, whole.s) for p in parts)
    assert torch.equal(torch.cat([p.qweight for p in parts]), whole.qweight)
    assert torch.equal(torch.cat([p.scales for p in parts]), whole.scales)
    ref = O.awq_ref(W, X, bits=4, g=128, grid=list(GRID))
    e = np.sort(ref.err)
    if (e[1] - e[0]) / e[0] > 1e-4:  # not tie-ambiguous: the oracle's alpha too
        assert alpha == ref.best_alpha


def _awq_worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from post_int4_weight_gptq_b200.split import awq_layer_split
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    W, X = _layer(63)
    alpha, s, qw, sc, errs = awq_layer_split(to_gpu_w(W, f"cuda:{rank}"),
                                             to_gpu_x(X, f"cuda:{rank}"), bits=4, g=128,
                                             alpha_grid=GRID)
    q.put((rank, alpha, s.cpu().numpy(), qw.cpu().numpy(), sc.cpu().numpy(), errs))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
@pytest.mark.timeout(600)
def test_two_gpus_give_the_awq_bits_of_the_emulated_split():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_awq_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=500) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W, X = _layer(63)
    alpha, parts, errs = _emulated_awq_split(W, X, 2)
    qw = torch.cat([p.qweight for p in parts]).cpu().numpy()
    sc = torch.cat([p.scales for p in parts]).cpu().numpy()
    for _, alpha_r, s_r, qw_r, sc_r, errs_r in res:
        assert alpha_r == alpha
        assert np.array_equal(s_r, parts[0].s.cpu().numpy())
        assert np.array_equal(qw_r, qw) and np.array_equal(sc_r, sc)
        assert np.allclose(errs_r, errs, rtol=1e-12, atol=0)
