"""The single-layer split over ranks (post_int4_weight_gptq_b200/split.py) on CPU:
world_size 2 over gloo.

The two compute steps are stood in for by the FP64 oracle (statistics of a
sample shard; GPTQ of a block of rows given H, its error share through H), so
what is tested is the plumbing: the sample and row ranges, the all-reduce of H
and of the act-order key, the all-reduce of the error shares and the gather
of the packed rows.  The result must equal the oracle's GPTQ of the whole
layer on all samples.
"""
import collections
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

Res = collections.namedtuple("Res", "qweight scales perm g_idx err")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    import sys
    sys.path.insert(0, ROOT)
    from workloads import make_weight, make_x_bits, small_spec
    spec = small_spec(10, 256, 900, seed=31, sigma_ln=0.9, n_outlier=3, outlier_gain=20.0)
    return make_weight(spec), make_x_bits(spec)


def _oracle_stats(X):
    import oracle as O
    H = O.hessian_ref(X)
    return torch.from_numpy(H), torch.from_numpy(np.diag(H).copy())


def _oracle_rows(Wr, H, sq, bits, g, act):
    import oracle as O
    Hn = H.numpy()
    perm = O.act_order_perm_ref(np.diag(sq.numpy())) if act else np.arange(Hn.shape[0])
    perm, U, _ = O.gptq_prepare_ref(Hn, 0.01, act, perm=perm)
    W = Wr.numpy().astype(np.float64)
    codes, scales, _, _ = O.gptq_sweep_ref(W[:, perm], U, bits, g)
    qweight, sc16, g_idx = _pack(codes, scales, perm, bits, g)
    D = W - O.dequant_ref(codes, sc16.astype(np.float64), perm, g)
    err = float(np.einsum("ri,ij,rj->", D, Hn, D))
    return Res(torch.from_numpy(qweight.view(np.int32)), torch.from_numpy(sc16),
               torch.from_numpy(perm), torch.from_numpy(g_idx), err)


def _pack(codes, scales, perm, bits, g):
    """Quantization-order codes -> packed memory-order words, fp16 scales, g_idx."""
    import oracle as O
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return (O.pack_ref(codes[:, inv], bits), scales.astype(np.float16), O.g_idx_ref(perm, g))


def _worker(rank, world, port, act, q):
    try:
        _work(rank, world, port, act, q)
    except Exception as e:  # the parent fails fast instead of waiting on the queue
        q.put((rank, repr(e)))
        raise


def _work(rank, world, port, act, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from post_int4_weight_gptq_b200.split import gptq_layer_split, sample_range
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    W, X = _layer()
    s0, s1 = sample_range(X.shape[0], rank, world)
    qw, sc, perm, g_idx, err = gptq_layer_split(
        torch.from_numpy(W), X[s0:s1], act_order=act, bits=3, g=64,
        stats_fn=_oracle_stats, rows_fn=lambda Wr, H, sq: _oracle_rows(Wr, H, sq, 3, 64, act))
    q.put((rank, qw.numpy(), sc.numpy(), perm.numpy(), g_idx.numpy(), err))
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("act", [False, True])
def test_two_ranks_equal_the_whole_layer(act):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, act, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda t: t[0])
    assert all(len(r) > 2 for r in res), res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import sys
    sys.path.insert(0, ROOT)
    import oracle as O
    W, X = _layer()
    ref = O.gptq_ref(W, X, bits=3, g=64, act_order=act)
    qw_ref, sc_ref, g_ref = _pack(ref.codes, ref.scales, ref.perm, 3, 64)
    e_ref = O.output_error_ref(W, O.dequant_ref(ref.codes, sc_ref.astype(np.float64), ref.perm,
                                                64), X)
    for rank, qw, sc, perm, g_idx, err in res:
        assert np.array_equal(qw.view(np.uint32), qw_ref)     # every rank holds all rows
        assert np.array_equal(sc, sc_ref)
        assert np.array_equal(perm, ref.perm) and np.array_equal(g_idx, g_ref)
        assert err == pytest.approx(e_ref, rel=1e-9)


def test_ranges_cover_every_row_once():
    from post_int4_weight_gptq_b200.split import row_range
    for out in (1, 7, 8, 4096, 8193):
        for world in (1, 2, 3, 8):
            rr = [row_range(out, r, world) for r in range(world)]
            assert rr[0][0] == 0 and rr[-1][1] == out
            assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
            sizes = [b - a for a, b in rr]
            assert max(sizes) - min(sizes) <= 1


# ---------------------------------------------------------------- AWQ, rows split

AwqRes = collections.namedtuple("AwqRes", "best_alpha s qweight scales err_per_alpha")


def _awq_layer(out):
    import sys
    sys.path.insert(0, ROOT)
    from workloads import make_weight, make_x_bits, small_spec
    spec = small_spec(out, 256, 700, seed=37, sigma_ln=1.0, n_outlier=4, outlier_gain=30.0)
    return make_weight(spec), make_x_bits(spec)


def _oracle_search(Wr, X, grid, bits, g):
    """Stand-in for awq_search_layer on a block of rows (the FP64 oracle)."""
    import oracle as O
    r = O.awq_ref(Wr.numpy(), X, bits=bits, g=g, grid=grid)
    return AwqRes(r.best_alpha, torch.from_numpy(r.s.astype(np.float32)),
                  torch.from_numpy(O.pack_ref(r.codes, bits).view(np.int32)),
                  torch.from_numpy(r.scales.astype(np.float16)), list(r.err))


GRID = [k / 10.0 for k in range(10)]


def _awq_worker(rank, world, port, out, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world))
        import sys
        sys.path.insert(0, ROOT)
        import datetime

        import torch.distributed as dist

        from post_int4_weight_gptq_b200.split import awq_layer_split
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        W, X = _awq_layer(out)
        alpha, s, qw, sc, errs = awq_layer_split(
            torch.from_numpy(W), X, bits=3, g=64, alpha_grid=GRID,
            search_fn=lambda Wr, grid: _oracle_search(Wr, X, grid, 3, 64))
        q.put((rank, alpha, s.numpy(), qw.numpy(), sc.numpy(), errs))
        dist.destroy_process_group()
    except Exception as e:  # the parent fails fast instead of waiting on the queue
        q.put((rank, repr(e)))
        raise


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,out", [(2, 12), (3, 2)])
def test_awq_rows_split_equals_the_whole_layer(world, out):
    """Each rank scores every alpha on its rows, one all-reduce sums the scores:
    the chosen alpha, s, codes and scales are the whole layer's (a rank with no
    rows, world 3 over 2 rows, still takes part in every collective)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_awq_worker, args=(r, world, port, out, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda t: t[0])
    assert all(len(r) > 2 for r in res), res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import sys
    sys.path.insert(0, ROOT)
    import oracle as O
    from post_int4_weight_gptq_b200.split import first_minimum, row_range
    W, X = _awq_layer(out)
    ref = O.awq_ref(W, X, bits=3, g=64, grid=GRID)
    if world == 2:  # rank 0's own rows prefer another alpha: its re-quantization is exercised
        r0, r1 = row_range(out, 0, world)
        own = O.awq_ref(W[r0:r1], X, bits=3, g=64, grid=GRID)
        assert first_minimum(list(own.err)) != ref.best_index
    for rank, alpha, s, qw, sc, errs in res:
        assert alpha == ref.best_alpha
        assert np.array_equal(s, ref.s.astype(np.float32))
        assert np.array_equal(qw.view(np.uint32), O.pack_ref(ref.codes, 3))
        assert np.array_equal(sc, ref.scales.astype(np.float16))
        assert np.allclose(errs, ref.err, rtol=1e-12, atol=0)


def test_first_minimum_is_the_first_on_a_tie():
    from post_int4_weight_gptq_b200.split import first_minimum
    assert first_minimum([3.0, 1.0, 2.0, 1.0]) == 1
    assert first_minimum([5.0]) == 0
    assert first_minimum([2.0, 2.0]) == 0
