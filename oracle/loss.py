"""O6: the K-FAC layer loss.

KronQ abstract and README intro: under the Kronecker-factored Hessian
H ~ H_X (x) H_G the quantization loss of a weight change dW depends on both
covariances, L(dW) = vec(dW)^T (H_X (x) H_G) vec(dW) = tr(dW H_X dW^T H_G)
(column-stacking vec, symmetric factors).  Evaluated in float64 with the
undamped factors; BiIP leaves it unchanged.
"""
from __future__ import annotations

import numpy as np


def kfac_loss(dW, HX, HG) -> float:
    """tr(dW H_X dW^T H_G)."""
    dW = np.asarray(dW, dtype=np.float64)
    return float(np.sum((dW @ np.asarray(HX, dtype=np.float64)) * (np.asarray(HG, dtype=np.float64) @ dW)))


def sweep_loss_from_errors(E, HG) -> float:
    """sum_j e_j^T H_G e_j over the columns e_j of the scaled error E.

    Because dW = E U and U (H + lambda I) U^T = I, this equals
    tr(dW (H_X + lambda I) dW^T H_G) for the sweep's own factors."""
    E = np.asarray(E, dtype=np.float64)
    return float(np.sum(E * (np.asarray(HG, dtype=np.float64) @ E)))
