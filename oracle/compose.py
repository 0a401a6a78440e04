"""AWQ scaling followed by GPTQ rounding, in float64.  Oracle (test infrastructure only).

Sources:
* "GPTQ versus AWQ objectives" (inferenceinterviews.com), the serving decision
  list after the toy table: for 3-bit or similarly aggressive targets GPTQ's
  error compensation recovers more than a scale alone, and the two methods
  compose: AWQ's per-channel scaling is applied first and GPTQ's rounding after.
* uplatz.com report, section 3.2: y = (W s)(X / s) is the same layer, so the
  scaled pair (W diag(s), X diag(1/s)) can be handed to any quantizer.

Readings (the pages give nothing beyond that sentence):
* Given s > 0 (AWQ's s = mean|x_j|^alpha* for the alpha its own RTN-scored grid
  search picked, or any positive vector), GPTQ runs unchanged on the layer
  W' = W diag(s) with calibration inputs X' = X diag(1/s): its proxy Hessian is
  X'^T X', its damping, act-order and factor are taken on that Hessian, and the
  column loop runs over W'.  X' is not re-rounded to bfloat16: the scaling is a
  change of variables, not a new input.
* The codes and group scales belong to W' (as AWQ's own do), so a user
  reconstructs What = code * scale / s_j; the error is ||X (W - What)^T||^2.
* alpha is not searched again with GPTQ inside the loop: the sentence applies
  AWQ's scaling "first", and the search scores RTN as AWQ defines it.
"""
from __future__ import annotations

import numpy as np

from .awq import awq_ref
from .error import x_to_f64
from .gptq import GPTQResult, gptq_ref, gptq_ref_blocked
from .pack import dequant_ref


def scaled_layer_ref(W, X, s):
    """(W diag(s), X diag(1/s)) in float64: the same layer, X' W'^T = X W^T."""
    s = np.asarray(s, dtype=np.float64)
    return np.asarray(W, dtype=np.float64) * s[None, :], x_to_f64(X) / s[None, :]


def awq_gptq_ref(W, X, s, bits: int = 4, g: int = 128, damp: float = 0.01,
                 act_order: bool = False, blocked: bool = False, force=None) -> GPTQResult:
    """GPTQ on the AWQ-scaled layer.  Codes (quantization order) and scales
    belong to W diag(s); ``perm`` and ``g_idx`` refer to memory columns."""
    Ws, Xs = scaled_layer_ref(W, X, s)
    if blocked:
        return gptq_ref_blocked(Ws, Xs, bits=bits, g=g, damp=damp, act_order=act_order)
    return gptq_ref(Ws, Xs, bits=bits, g=g, damp=damp, act_order=act_order, force=force)


def awq_gptq_dequant_ref(codes_q, scales, perm, s, g: int, fp16: bool = True) -> np.ndarray:
    """What in memory order: code * scale / s_j (``fp16`` rounds the scales
    to half precision first, as the packed format stores them)."""
    return dequant_ref(codes_q, scales, perm, g, fp16=fp16) / np.asarray(s, dtype=np.float64)[None, :]


def awq_then_gptq_ref(W, X, bits: int = 4, g: int = 128, damp: float = 0.01,
                      act_order: bool = False, grid=None, blocked: bool = False):
    """The composed method end to end: AWQ's grid search picks alpha* and
    s = m^alpha*, then GPTQ rounds W diag(s).  Returns (AWQResult, GPTQResult)."""
    a = awq_ref(W, X, bits, g, grid)
    return a, awq_gptq_ref(W, X, a.s, bits, g, damp, act_order, blocked)
