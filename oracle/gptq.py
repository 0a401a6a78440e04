"""GPTQ, step by step, in float64.  Oracle (test infrastructure only).

Source: "GPTQ versus AWQ objectives" (inferenceinterviews.com).
* Section "A strong answer", the ``gptq_layer`` listing: the proxy Hessian
  H = X^T X ([in, in]); damping H += damp * mean(diag H) * I with damp = 0.01;
  U = the upper Cholesky factor of H^-1 (H^-1 = U^T U); qmax = 2^(bits-1) - 1;
  for each input column j: at a group start (j % g == 0) a per-row scale
  max|W[:, j:j+g]| / qmax taken from the *current* (already updated) W; the
  column rounded to nearest and clipped to [-qmax-1, qmax]; its error
  (W[:, j] - Q[:, j]) / U[j, j] pushed onto every later column as the outer
  product with U[j, j+1:].  The prose above the listing writes H = 2 X^T X; the
  factor 2 cancels (damping is relative and err * U is invariant under scaling
  H), and the listing's X^T X is used.
* Same section, the remark after the listing: implementations batch the updates
  over blocks of columns so the work runs as GEMMs, with the same arithmetic
  (``gptq_ref_blocked``).
* Section "What interviewers probe next": act-order quantizes columns in order
  of decreasing Hessian diagonal, so a group index per column is needed; the
  damping term keeps the Cholesky factorization stable.

Readings where the pages are silent (each listed in the design notes):
* Rounding is NumPy's round-half-to-even, on the true quotient W/scale.
* An all-zero group row (scale 0) gets codes 0 and error 0 (the listing would
  divide 0/0); nothing in the workloads reaches it.
* Act-order ties keep ascending index (stable sort); groups are consecutive g
  positions in quantization order; the damping mean is over the undamped
  diagonal (the listing's order of operations).
* Codes are returned in quantization order; ``perm[p]`` is the memory column
  quantized at position p.
* Asymmetric groups (``sym=False``): the uplatz.com report, section "Key
  Parameters" (Group Size), gives each group "a scale and zero-point" and no
  formula.  Read as min/max affine rounding of the group's current weights with
  the range widened to hold 0: lo = min(0, min w), hi = max(0, max w),
  scale = (hi - lo) / (2^bits - 1), zero = round(-lo / scale), stored code
  u = clip(round(w / scale) + zero, 0, 2^bits - 1), What = (u - zero) * scale.
  Widening to 0 keeps the zero-point a valid code (0 <= zero <= 2^bits - 1,
  stored like the weights) and reconstructs a zero weight exactly.  Codes are
  returned signed, c = u - zero, so What = c * scale as in the symmetric case.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .error import x_to_f64

NO_FORCE = -128  # sentinel in a ``force`` array: "this code is not forced"


def hessian_ref(X, chunk: int = 8192, dtype=np.float64) -> np.ndarray:
    """H = X^T X (the listing's proxy Hessian), summed over row chunks.  float64
    is the oracle; dtype=float32 accumulates in the FP32 the pages fix for H
    (used only to measure that precision's drift, see gptq_sweep_ref)."""
    n, inp = X.shape
    H = np.zeros((inp, inp), dtype=dtype)
    for r0 in range(0, n, chunk):
        xc = x_to_f64(X[r0:r0 + chunk]).astype(dtype)
        H += xc.T @ xc
    return H


def hessian_syrk_ref(X, chunk: int = 8192) -> np.ndarray:
    """H = X^T X in float64 with the BLAS symmetric rank-k update: each chunk adds
    its X_c^T X_c to the upper triangle (half the multiplications of a full
    product), then the lower triangle is mirrored.  The same sums as
    hessian_ref up to rounding order; used where that product takes minutes
    (pinned against hessian_ref)."""
    from scipy.linalg.blas import dsyrk
    n, inp = X.shape
    H = np.zeros((inp, inp), dtype=np.float64, order="F")
    for r0 in range(0, n, chunk):
        xc = np.asfortranarray(x_to_f64(X[r0:r0 + chunk]))
        # upper triangle of xc^T xc (trans=1), accumulated into H (beta=1)
        H = dsyrk(1.0, xc, beta=1.0, c=H, trans=1, lower=0, overwrite_c=1)
    iu = np.triu_indices(inp, 1)
    H[(iu[1], iu[0])] = H[iu]
    return np.ascontiguousarray(H)


def act_order_perm_ref(H: np.ndarray) -> np.ndarray:
    """Quantization order by decreasing diag(H); equal values keep index order."""
    return np.argsort(-np.diag(H), kind="stable").astype(np.int64)


def damped_ref(H: np.ndarray, damp: float):
    """H + damp * mean(diag H) * I; returns (H_d, lambda), in H's precision."""
    lam = float(damp) * float(np.mean(np.diag(H)))
    return H + H.dtype.type(lam) * np.eye(H.shape[0], dtype=H.dtype), lam


def upper_factor_ref(Hd: np.ndarray) -> np.ndarray:
    """U with H_d^-1 = U^T U: the transposed lower Cholesky factor of inv(H_d),
    exactly as the listing forms it.  Raises numpy.linalg.LinAlgError if H_d is
    not positive definite."""
    return np.linalg.cholesky(np.linalg.inv(Hd)).T


def upper_factor_r_ref(Hd: np.ndarray) -> np.ndarray:
    """The same U as upper_factor_ref without forming inv(H_d): with J the index
    reversal, R = J chol(J H_d J) J is upper triangular with H_d = R R^T, so
    inv(H_d) = inv(R)^T inv(R), and U = inv(R) is that factorisation's upper
    triangular factor with positive diagonal, which is unique.  One Cholesky and
    one triangular inverse (2 n^3 / 3 flop against about 7 n^3 / 3); used where
    the listing's route takes minutes (pinned against upper_factor_ref)."""
    from scipy.linalg import lapack
    Lm = np.linalg.cholesky(Hd[::-1, ::-1])
    R = np.ascontiguousarray(Lm[::-1, ::-1])
    U, info = lapack.dtrtri(R, lower=0)
    if info != 0:
        raise np.linalg.LinAlgError(f"triangular inverse failed: info {info}")
    return np.triu(U)


@dataclasses.dataclass
class GPTQResult:
    codes: np.ndarray        # int16 [out, in], quantization order (signed: What = code * scale)
    scales: np.ndarray       # float64 [out, ngroups], group of position p is p // g
    perm: np.ndarray         # int64 [in]
    g_idx: np.ndarray        # int64 [in], group of each memory-order column
    v: np.ndarray | None     # float64 [out, in]: W[:, j] / scale before rounding
    err: np.ndarray | None   # float64 [out, in]: the pushed error of each column
    U: np.ndarray
    lam: float
    bits: int
    g: int
    zeros: np.ndarray | None = None  # int16 [out, ngroups] zero-points (asymmetric groups)


def gptq_prepare_ref(H: np.ndarray, damp: float = 0.01, act_order: bool = False, perm=None,
                     via_r: bool = False):
    """Permutation (act-order), damping and the upper factor: (perm, U, lam), in
    H's precision.  ``perm`` given: that quantization order instead.  ``via_r``:
    U from upper_factor_r_ref (the same matrix, fewer flops)."""
    inp = H.shape[0]
    if perm is None:
        perm = act_order_perm_ref(H) if act_order else np.arange(inp, dtype=np.int64)
    Hp = H[np.ix_(perm, perm)]
    Hd, lam = damped_ref(Hp, damp)
    return perm, (upper_factor_r_ref(Hd) if via_r else upper_factor_ref(Hd)), lam


def _round_clip(v: np.ndarray, qmax: int) -> np.ndarray:
    return np.clip(np.round(v), -qmax - 1, qmax)


def group_quantizer_ref(Wg: np.ndarray, bits: int, sym: bool = True, dtype=np.float64,
                        force_zero=None):
    """Per-row quantizer of one group from its current weights Wg [out, <= g]:
    (scale, zero, zv, cmin, cmax); signed codes are clip(round(w / scale),
    cmin, cmax) and What = code * scale.

    sym: scale = max|w| / qmax, zero 0, codes in [-qmax - 1, qmax] (the listing).
    asym: lo = min(0, min w), hi = max(0, max w), scale = (hi - lo) / (2^bits - 1),
    zv = -lo / scale, zero = round(zv), codes in [-zero, 2^bits - 1 - zero].
    A row whose group is all zero gets scale 0 and zero 0.  ``force_zero``
    (int [out], NO_FORCE where free) overrides the rounded zero-point."""
    out = Wg.shape[0]
    if sym:
        qmax = 2 ** (bits - 1) - 1
        scale = np.abs(Wg).max(axis=1) / dtype(qmax)
        zero = np.zeros(out)
        return (scale, zero, zero.copy(), np.full(out, -qmax - 1.0), np.full(out, float(qmax)))
    maxq = 2 ** bits - 1
    lo = np.minimum(Wg.min(axis=1), dtype(0.0))
    hi = np.maximum(Wg.max(axis=1), dtype(0.0))
    scale = (hi - lo) / dtype(maxq)
    live = scale > 0
    zv = np.where(live, -lo / np.where(live, scale, dtype(1.0)), dtype(0.0))
    zero = np.round(zv)
    if force_zero is not None:
        zero = np.where(force_zero != NO_FORCE, force_zero, zero)
    return scale, zero, zv, -zero, maxq - zero


def _sweep(Wp, U, bits, g, sym, force, force_zero, log, dtype):
    W = np.array(Wp, dtype=dtype, copy=True)
    U = np.asarray(U, dtype=dtype)
    out, inp = W.shape
    ngroups = -(-inp // g)
    codes = np.zeros((out, inp), dtype=np.int16)
    scales = np.zeros((out, ngroups), dtype=np.float64)
    zeros = np.zeros((out, ngroups), dtype=np.int16)
    zvlog = np.zeros((out, ngroups))
    vlog = np.zeros((out, inp)) if log else None
    elog = np.zeros((out, inp)) if log else None
    scale = cmin = cmax = None
    for j in range(inp):
        if j % g == 0:
            fz = None if force_zero is None else force_zero[:, j // g]
            scale, zero, zv, cmin, cmax = group_quantizer_ref(W[:, j:j + g], bits, sym, dtype, fz)
            scales[:, j // g] = scale
            zeros[:, j // g] = zero.astype(np.int16)
            zvlog[:, j // g] = zv
        live = scale > 0
        v = np.where(live, W[:, j] / np.where(live, scale, dtype(1.0)), dtype(0.0))
        c = np.clip(np.round(v), cmin, cmax)
        if force is not None:
            f = force[:, j]
            c = np.where(f != NO_FORCE, f, c)
        Q = c.astype(dtype) * scale
        e = (W[:, j] - Q) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        codes[:, j] = c.astype(np.int16)
        if log:
            vlog[:, j] = v
            elog[:, j] = e
    return codes, scales, zeros, zvlog, vlog, elog


def gptq_sweep_ref(Wp: np.ndarray, U: np.ndarray, bits: int = 4, g: int = 128,
                   force: np.ndarray | None = None, log: bool = True, dtype=np.float64):
    """The listing's column loop on weights already in quantization order.

    Returns (codes int16 [out, in], scales [out, ngroups], v, err).
    ``force`` (int array [out, in], NO_FORCE where free) replaces the rounded
    code at chosen sites: the teacher-forcing hook of the parity comparison.
    ``dtype`` is the working precision: float64 is the oracle; float32 runs the
    same loop in float32, the working precision of the GPU sweep and its block
    updates, to measure how far that arithmetic alone drifts from float64 (the
    parity tie window)."""
    codes, scales, _, _, vlog, elog = _sweep(Wp, U, bits, g, True, force, None, log, dtype)
    return codes, scales, vlog, elog


def gptq_sweep_asym_ref(Wp: np.ndarray, U: np.ndarray, bits: int = 4, g: int = 128,
                        force: np.ndarray | None = None, force_zero: np.ndarray | None = None,
                        log: bool = True, dtype=np.float64):
    """The same loop with a scale and zero-point per group (asymmetric groups,
    see the module notes).  Returns (codes, scales, zeros, zv, v, err): signed
    codes (stored u = code + zero), zero-points int16 [out, ngroups] and their
    unrounded values zv = -lo / scale.  ``force_zero`` [out, ngroups] overrides
    rounded zero-points (teacher forcing)."""
    return _sweep(Wp, U, bits, g, False, force, force_zero, log, dtype)


def g_idx_from_perm(perm: np.ndarray, g: int) -> np.ndarray:
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return inv // g


def gptq_ref(W, X=None, *, H=None, bits: int = 4, g: int = 128, damp: float = 0.01,
             act_order: bool = False, force=None, log: bool = True,
             sym: bool = True) -> GPTQResult:
    """GPTQ of one layer, literally (one column at a time); ``sym=False``: a
    scale and zero-point per group."""
    if H is None:
        H = hessian_ref(X)
    perm, U, lam = gptq_prepare_ref(H, damp, act_order)
    Wp = np.asarray(W, dtype=np.float64)[:, perm]
    codes, scales, zeros, _, v, e = _sweep(Wp, U, bits, g, sym, force, None, log, np.float64)
    return GPTQResult(codes, scales, perm, g_idx_from_perm(perm, g), v, e, U, lam, bits, g,
                      None if sym else zeros)


def block_partition_ref(inp: int, g: int, block: int = 128):
    """Column blocks [b, e) of width <= ``block`` such that every group start is
    either a block start or has its whole group inside its block.  Then a group
    scale never reads a column whose pending updates from the same block have
    not been applied, so blocking leaves the arithmetic unchanged."""
    blocks = []
    b = 0
    while b < inp:
        e = min(b + block, inp)
        s = (b // g + 1) * g          # first group start after b
        while s < e:
            if min(s + g, inp) > e:   # that group would run past the block
                e = s
                break
            s += g
        blocks.append((b, e))
        b = e
    return blocks


def _sweep_blocked(Wp, U, bits, g, block, sym, force=None, force_zero=None):
    W = np.array(Wp, dtype=np.float64, copy=True)
    out, inp = W.shape
    codes = np.zeros((out, inp), dtype=np.int16)
    scales = np.zeros((out, -(-inp // g)), dtype=np.float64)
    zeros = np.zeros((out, -(-inp // g)), dtype=np.int16)
    zvlog = np.zeros((out, -(-inp // g)))
    vlog = np.zeros((out, inp))
    scale = cmin = cmax = None
    for b, e in block_partition_ref(inp, g, block):
        Err = np.zeros((out, e - b))
        for j in range(b, e):
            if j % g == 0:
                fz = None if force_zero is None else force_zero[:, j // g]
                scale, zero, zv, cmin, cmax = group_quantizer_ref(W[:, j:j + g], bits, sym,
                                                                  force_zero=fz)
                scales[:, j // g] = scale
                zeros[:, j // g] = zero.astype(np.int16)
                zvlog[:, j // g] = zv
            live = scale > 0
            v = np.where(live, W[:, j] / np.where(live, scale, 1.0), 0.0)
            c = np.clip(np.round(v), cmin, cmax)
            if force is not None:
                c = np.where(force[:, j] != NO_FORCE, force[:, j], c)
            err = (W[:, j] - c * scale) / U[j, j]
            W[:, j + 1:e] -= np.outer(err, U[j, j + 1:e])
            Err[:, j - b] = err
            codes[:, j] = c.astype(np.int16)
            vlog[:, j] = v
        if e < inp:
            W[:, e:] -= Err @ U[b:e, e:]
    return codes, scales, zeros, vlog, zvlog


def gptq_sweep_blocked_ref(Wp: np.ndarray, U: np.ndarray, bits: int = 4, g: int = 128,
                           block: int = 128, force: np.ndarray | None = None):
    """The same loop with updates deferred per column block: inside a block the
    error goes to the block's later columns; after the block one product
    Err[:, b:e] @ U[b:e, e:] updates every column past it.  (codes, scales, v).
    ``force`` is the teacher-forcing hook of ``gptq_sweep_ref``."""
    codes, scales, _, vlog, _ = _sweep_blocked(Wp, U, bits, g, block, True, force)
    return codes, scales, vlog


def gptq_sweep_blocked_asym_ref(Wp: np.ndarray, U: np.ndarray, bits: int = 4, g: int = 128,
                                block: int = 128, force: np.ndarray | None = None,
                                force_zero: np.ndarray | None = None):
    """Blocked sweep with asymmetric groups: (codes, scales, zeros, v, zv)."""
    return _sweep_blocked(Wp, U, bits, g, block, False, force, force_zero)


def gptq_ref_blocked(W, X=None, *, H=None, bits: int = 4, g: int = 128, damp: float = 0.01,
                     act_order: bool = False, block: int = 128, sym: bool = True) -> GPTQResult:
    """GPTQ with block-deferred updates (same arithmetic, faster on large layers)."""
    if H is None:
        H = hessian_ref(X)
    perm, U, lam = gptq_prepare_ref(H, damp, act_order)
    Wp = np.asarray(W, dtype=np.float64)[:, perm]
    codes, scales, zeros, v, _ = _sweep_blocked(Wp, U, bits, g, block, sym)
    return GPTQResult(codes, scales, perm, g_idx_from_perm(perm, g), v, None, U, lam, bits, g,
                      None if sym else zeros)


def rtn_ref(W, bits: int = 4, g: int = 128):
    """Plain group round-to-nearest (the toy table's first column): every group
    scale from the original weights, no error feedback.  Returns (codes, scales)."""
    W = np.asarray(W, dtype=np.float64)
    out, inp = W.shape
    qmax = 2 ** (bits - 1) - 1
    codes = np.zeros((out, inp), dtype=np.int16)
    scales = np.zeros((out, -(-inp // g)))
    for s in range(0, inp, g):
        blk = W[:, s:s + g]
        sc = np.abs(blk).max(axis=1) / qmax
        live = sc > 0
        v = np.where(live[:, None], blk / np.where(live, sc, 1.0)[:, None], 0.0)
        codes[:, s:s + g] = _round_clip(v, qmax).astype(np.int16)
        scales[:, s // g] = sc
    return codes, scales


def rtn_asym_ref(W, bits: int = 4, g: int = 128):
    """Group round-to-nearest with a scale and zero-point per group (the
    asymmetric quantizer of the module notes, no error feedback).  Returns
    (signed codes, scales, zeros); the stored code is code + zero."""
    W = np.asarray(W, dtype=np.float64)
    out, inp = W.shape
    codes = np.zeros((out, inp), dtype=np.int16)
    scales = np.zeros((out, -(-inp // g)))
    zeros = np.zeros((out, -(-inp // g)), dtype=np.int16)
    for s0 in range(0, inp, g):
        blk = W[:, s0:s0 + g]
        sc, z, _, cmin, cmax = group_quantizer_ref(blk, bits, sym=False)
        live = sc > 0
        v = np.where(live[:, None], blk / np.where(live, sc, 1.0)[:, None], 0.0)
        codes[:, s0:s0 + g] = np.clip(np.round(v), cmin[:, None], cmax[:, None]).astype(np.int16)
        scales[:, s0 // g] = sc
        zeros[:, s0 // g] = z.astype(np.int16)
    return codes, scales, zeros
