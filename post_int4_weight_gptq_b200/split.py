"""One GPTQ layer split over the ranks of a torch.distributed process group.

"GPTQ versus AWQ objectives" (sizing block under "A strong answer"): the proxy
Hessian H = X^T X is a sum over calibration samples, and given H the rows of W
are independent problems (the listing's error feedback never mixes rows).  So:

  1. each rank builds the statistics of its own shard of the samples
     (piq_layer_statistics: H_r = X_r^T X_r and the act-order key), on its GPU;
  2. one all-reduce sums them: the only exchange of the path (in x in doubles,
     plus in doubles of the key); NCCL over NVLink when the group's backend is
     nccl;
  3. each rank runs GPTQ on its own block of rows of W from the summed H
     (gptq_quantize_rows_from_h: damping, factor, sweep, pack, its rows' share
     of the output error); every rank forms the same factor and permutation;
  4. the error shares are summed (one all-reduce of one double), and, when asked,
     the packed rows are gathered so every rank holds the whole layer.

The arithmetic of steps 1 and 3 is the library's; this module only moves
tensors.  The two compute calls are parameters so that the plumbing can be
exercised on hosts without the GPU library (its tests inject CPU stand-ins).

AWQ splits over the rows of W instead ("GPTQ versus AWQ objectives", AWQ
paragraph under "A strong answer": s_j = mean|x_j|^alpha depends on the inputs
only, and the output error of a candidate alpha is a sum over the rows of W):
every rank holds all of X and scores every alpha on its own rows, one
all-reduce of n_alpha doubles sums the scores, and every rank takes the same
first minimum (awq_layer_split).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_range(out: int, rank: int, world: int) -> tuple[int, int]:
    """Rows [r0, r1) of W that rank quantizes: contiguous, sizes differ by at most one."""
    base, extra = divmod(out, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def sample_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Calibration samples [s0, s1) whose statistics rank builds (same split rule)."""
    return row_range(n, rank, world)


def gptq_layer_split(W, X_shard, group=None, bits=4, g=128, damp=0.01, act_order=False,
                     gather=True, stats_fn=None, rows_fn=None):
    """GPTQ of the layer W [out, in] (every rank passes the whole W) from the
    calibration samples split over the group (X_shard [n_r, in]: this rank's
    samples).  Returns (qweight, scales, perm, g_idx, err) where qweight and
    scales hold this rank's rows, or all rows when gather is set; err is the
    layer's output error on all samples."""
    if stats_fn is None or rows_fn is None:
        import post_int4_weight_gptq_b200 as piq
        stats_fn = stats_fn or (lambda X: piq.layer_statistics(X, want_sumsq=act_order))
        rows_fn = rows_fn or (lambda Wr, H, sq: piq.gptq_rows_from_h(
            Wr, H, sq, bits=bits, g=g, damp=damp, act_order=act_order))
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    H, sq = stats_fn(X_shard)
    dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    if act_order:
        dist.all_reduce(sq, op=dist.ReduceOp.SUM, group=group)
    r0, r1 = row_range(W.shape[0], rank, world)
    res = rows_fn(W[r0:r1].contiguous(), H, sq)
    err = torch.tensor([res.err], dtype=torch.float64, device=H.device)
    dist.all_reduce(err, op=dist.ReduceOp.SUM, group=group)
    qweight, scales = res.qweight, res.scales
    if gather:
        qweight = _gather_rows(res.qweight, W.shape[0], world, group)
        scales = _gather_rows(res.scales, W.shape[0], world, group)
    return qweight, scales, res.perm, res.g_idx, float(err.item())


def _gather_rows(t, out, world, group):
    """Concatenate every rank's row block (blocks of row_range) in rank order."""
    sizes = [row_range(out, r, world) for r in range(world)]
    biggest = max(r1 - r0 for r0, r1 in sizes)
    pad = torch.zeros((biggest,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[:t.shape[0]] = t
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:r1 - r0] for p, (r0, r1) in zip(parts, sizes)], dim=0)


def first_minimum(errs) -> int:
    """Index of the smallest error, the first one on a tie (the library's rule)."""
    best = 0
    for i in range(1, len(errs)):
        if errs[i] < errs[best]:
            best = i
    return best


def awq_layer_split(W, X, group=None, bits=4, g=128, alpha_grid=None, gather=True,
                    search_fn=None):
    """AWQ search of the layer W [out, in] with its rows split over the group.
    Every rank passes the whole W and the whole calibration input X.

      1. each rank scores every alpha on its block of rows (awq_search_layer on
         W[r0:r1] and X: s is the same on every rank, the errors are this
         block's shares of the layer's errors);
      2. one all-reduce sums the n_alpha shares: the only exchange;
      3. every rank takes the first minimum of the sums; a rank whose own rows
         preferred another alpha quantizes them again at the chosen one;
      4. when asked, the packed rows are gathered.

    Returns (best_alpha, s, qweight, scales, err_per_alpha): qweight and scales
    hold this rank's rows, or all rows when gather is set; err_per_alpha are
    the layer's errors."""
    if alpha_grid is None:
        alpha_grid = tuple(k / 20.0 for k in range(20))
    alpha_grid = [float(a) for a in alpha_grid]
    if search_fn is None:
        import post_int4_weight_gptq_b200 as piq
        search_fn = lambda Wr, grid: piq.awq_search_layer(Wr, X, bits=bits, g=g,  # noqa: E731
                                                          alpha_grid=grid)
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    r0, r1 = row_range(W.shape[0], rank, world)
    Wr = W[r0:r1].contiguous()
    res = search_fn(Wr, alpha_grid) if r1 > r0 else None
    shares = res.err_per_alpha if res is not None else [0.0] * len(alpha_grid)
    errs = torch.tensor(shares, dtype=torch.float64, device=W.device)
    dist.all_reduce(errs, op=dist.ReduceOp.SUM, group=group)
    errs = errs.tolist()
    k = first_minimum(errs)
    if res is not None and first_minimum(res.err_per_alpha) != k:
        res = search_fn(Wr, [alpha_grid[k]])
    if res is None:  # no rows here: s from a one-row call keeps every rank's s alike
        one = search_fn(W[:1].contiguous(), [alpha_grid[k]])
        s = one.s
        qweight = one.qweight[:0]
        scales = one.scales[:0]
    else:
        s, qweight, scales = res.s, res.qweight, res.scales
    if gather:
        qweight = _gather_rows(qweight, W.shape[0], world, group)
        scales = _gather_rows(scales, W.shape[0], world, group)
    return alpha_grid[k], s, qweight, scales, errs
