"""Parity metric shared by the GPU tests (comparison only; no layer arithmetic).

err = max over rows m of  max_n |Y_gpu[m,n] - Y_ref[m,n]| / max(max_n |Y_ref[m,n]|, tiny)

Per-row normalisation keeps rows scaled x20 (outlier tokens) from loosening the check on
ordinary rows, and avoids the undefined element-wise relative error at zero crossings.
Tolerances: 2e-2 for bf16 inputs with fp32 accumulation, 1e-4 for fp32.
"""

import numpy as np

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def row_normalised_max_err(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    if y.size == 0:
        return 0.0
    scale = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((np.abs(y - ref).max(axis=1) / scale).max())
