"""Oracle: a plain, slow, FP64 CPU statement of what the quantization path computes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it and shares no code with it.

Sources (web pages on GPTQ/AWQ; cited by page title and section):
* "GPTQ versus AWQ objectives" (inferenceinterviews.com), section "A strong
  answer": the NumPy ``gptq_layer`` loop (proxy Hessian X^T X, damping by 1% of
  the mean diagonal, upper Cholesky factor of H^-1, per-row group scale taken at
  each group start, symmetric clip-round, error pushed onto later columns), the
  block-batching remark, the AWQ definition s_j = mean|x_j|^alpha with a grid
  search on calibration output error, and section "What interviewers probe
  next" (act-order by decreasing Hessian diagonal; damping).
* "A Comprehensive Analysis of Post-Training Quantization Strategies ..."
  (uplatz.com), sections 2.1-2.3 and 3.2: the same objective written as
  ||W_q X - W X||_F, group size, act-order, the Babai nearest-plane reading,
  and y = (W s)(X / s).
* "GPTQ versus AWQ objectives", the serving decision list: AWQ's scaling and
  GPTQ's rounding compose (``compose.py``).

Every function works in float64 on exact copies of the inputs (bfloat16 X values
are exact in float64).  Where the pages leave a step open, the reading taken is
stated in the function's docstring.
"""
from .gptq import (GPTQResult, act_order_perm_ref, block_partition_ref, damped_ref,
                   gptq_prepare_ref, gptq_ref, gptq_ref_blocked, gptq_sweep_asym_ref,
                   gptq_sweep_blocked_asym_ref, gptq_sweep_blocked_ref, gptq_sweep_ref,
                   group_quantizer_ref, hessian_ref, hessian_syrk_ref, rtn_asym_ref, rtn_ref,
                   upper_factor_r_ref, upper_factor_ref)
from .awq import AWQResult, awq_ref, awq_scales_ref, channel_mean_abs_ref, group_rtn_ref
from .pack import dequant_ref, g_idx_ref, pack_asym_ref, pack_ref, unpack_ref
from .error import output_error_ref, x_to_f64
from .compose import awq_gptq_dequant_ref, awq_gptq_ref, awq_then_gptq_ref, scaled_layer_ref

__all__ = [
    "GPTQResult", "act_order_perm_ref", "block_partition_ref", "damped_ref",
    "gptq_prepare_ref", "gptq_ref", "gptq_ref_blocked", "gptq_sweep_ref", "hessian_ref",
    "gptq_sweep_blocked_ref", "gptq_sweep_blocked_asym_ref",
    "rtn_ref", "upper_factor_ref", "upper_factor_r_ref", "hessian_syrk_ref", "gptq_sweep_asym_ref", "group_quantizer_ref", "rtn_asym_ref",
    "pack_asym_ref", "AWQResult", "awq_ref", "awq_scales_ref",
    "channel_mean_abs_ref", "group_rtn_ref", "dequant_ref", "g_idx_ref", "pack_ref",
    "unpack_ref", "output_error_ref", "x_to_f64", "awq_gptq_dequant_ref", "awq_gptq_ref",
    "awq_then_gptq_ref", "scaled_layer_ref",
]
