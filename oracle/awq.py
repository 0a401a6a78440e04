"""AWQ scale search, in float64.  Oracle (test infrastructure only).

Sources:
* "GPTQ versus AWQ objectives", section "A strong answer" (AWQ paragraph): input
  channel j of W is scaled up by s_j and the activation down by the same factor
  (folded into the previous op); s_j = mean|x_j|^alpha; one alpha per layer is
  grid-searched on calibration output error, then the weights are rounded to
  nearest.  "Common mistakes": every weight ends up INT4 (no FP16 channels).
* uplatz.com report, section 3.2: y = (W s)(X / s) is the same layer; the whole
  scaled matrix is quantized; the scale is found by grid search on the output
  error.

Readings where the pages are silent:
* mean|x_j| is the arithmetic mean of |x_nj| over all n calibration samples.
* The grid is alpha_k = k/20, k = 0..19 (given by the caller).
* The quantizer is the same symmetric group RTN as GPTQ's rounding step
  (scale max|W'[r, group]| / qmax, round half to even, clip), applied to
  W' = W diag(s) with no error feedback.
* The scored reconstruction is What = code * scale / s_j with the full-precision
  group scale; the first minimum wins a tie; s_j = 1 where mean|x_j| = 0.
* No normalisation of s (a constant factor does not change the codes).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .error import output_error_ref, x_to_f64


def channel_mean_abs_ref(X, chunk: int = 8192) -> np.ndarray:
    """m_j = (1/n) sum_n |x_nj| in float64."""
    n, inp = X.shape
    acc = np.zeros(inp)
    for r0 in range(0, n, chunk):
        acc += np.abs(x_to_f64(X[r0:r0 + chunk])).sum(axis=0)
    return acc / n


def awq_scales_ref(m: np.ndarray, alpha: float) -> np.ndarray:
    """s_j = m_j ** alpha, and 1 for a channel whose mean is 0."""
    m = np.asarray(m, dtype=np.float64)
    return np.where(m > 0, np.power(np.where(m > 0, m, 1.0), alpha), 1.0)


def group_rtn_ref(Wp: np.ndarray, bits: int = 4, g: int = 128):
    """Symmetric group round-to-nearest of already-scaled weights: (codes, scales)."""
    W = np.asarray(Wp, dtype=np.float64)
    out, inp = W.shape
    qmax = 2 ** (bits - 1) - 1
    codes = np.zeros((out, inp), dtype=np.int16)
    scales = np.zeros((out, -(-inp // g)))
    for s0 in range(0, inp, g):
        blk = W[:, s0:s0 + g]
        sc = np.abs(blk).max(axis=1) / qmax
        live = sc > 0
        v = np.where(live[:, None], blk / np.where(live, sc, 1.0)[:, None], 0.0)
        codes[:, s0:s0 + g] = np.clip(np.round(v), -qmax - 1, qmax).astype(np.int16)
        scales[:, s0 // g] = sc
    return codes, scales


def awq_dequant_ref(codes: np.ndarray, scales: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """What = code * scale / s_j (full-precision scales)."""
    cols = np.arange(codes.shape[1]) // g
    return codes.astype(np.float64) * scales[:, cols] / np.asarray(s)[None, :]


@dataclasses.dataclass
class AWQResult:
    best_alpha: float
    best_index: int
    m: np.ndarray
    s: np.ndarray             # scales of the chosen alpha, [in]
    codes: np.ndarray         # int16 [out, in] of W diag(s)
    scales: np.ndarray        # float64 [out, ngroups], belong to W diag(s)
    err: np.ndarray           # float64 [n_alpha]


def awq_ref(W, X, bits: int = 4, g: int = 128, grid=None) -> AWQResult:
    """Grid search of the AWQ exponent, scored by ||X W^T - X What^T||^2."""
    if grid is None:
        grid = [k / 20.0 for k in range(20)]
    W = np.asarray(W, dtype=np.float64)
    m = channel_mean_abs_ref(X)
    errs = np.zeros(len(grid))
    for k, a in enumerate(grid):
        s = awq_scales_ref(m, a)
        c, sc = group_rtn_ref(W * s[None, :], bits, g)
        errs[k] = output_error_ref(W, awq_dequant_ref(c, sc, s, g), X)
    kbest = int(np.argmin(errs))          # first minimum
    s = awq_scales_ref(m, grid[kbest])
    c, sc = group_rtn_ref(W * s[None, :], bits, g)
    return AWQResult(float(grid[kbest]), kbest, m, s, c, sc, errs)
