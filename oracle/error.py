"""Layer output error, the objective both methods share.

"GPTQ versus AWQ objectives", section "How to approach it": the error of a
quantized layer on calibration inputs X is ||X W^T - X What^T||^2; the
uplatz.com report (section 2.1, its displayed objective) writes the same
quantity as ||W_q X - W X||_F^2 with X stored [in, samples].

Oracle (test infrastructure only).
"""
from __future__ import annotations

import numpy as np


def x_to_f64(x) -> np.ndarray:
    """Calibration inputs as float64.  uint16 arrays are bfloat16 bit patterns
    (decoded exactly); float arrays are cast."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def output_error_ref(W, What, X, chunk: int = 8192) -> float:
    """||X W^T - X What^T||_F^2 = ||X (W - What)^T||_F^2 in float64.

    W, What: [out, in]; X: [n, in] (bfloat16 bits or floats).  Summed over row
    chunks of X (a sum of squares splits over samples)."""
    dW = np.asarray(W, dtype=np.float64) - np.asarray(What, dtype=np.float64)
    n = X.shape[0]
    total = 0.0
    for r0 in range(0, n, chunk):
        y = x_to_f64(X[r0:r0 + chunk]) @ dW.T
        total += float(np.sum(y * y))
    return total
