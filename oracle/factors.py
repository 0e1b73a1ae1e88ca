"""O1/O2: the two Kronecker factors of the layer Hessian and the traces.

KronQ README (intro): the layer Hessian is approximated as H ~ H_X (x) H_G, an
input-side factor from the activations and an output-side factor from the
output gradients.  "WaterKron and FlipFlop Hessian", Table 1, "Marginal" row:
A = E[x x^T], B = E[g g^T].  KronQ abstract, point (2): the inter-layer
sensitivity is driven by the gradient and activation Hessian traces; KronQ
README bullet "Inter-layer mixed precision": tr(H_G) * tr(H_X).

Reading taken: sums over the calibration tokens, not means.  A common scale
on all factors changes nothing downstream (damping and the BiIP rescale are
relative, and bit allocation compares sublayers with the same token count).
"""
from __future__ import annotations

import numpy as np


def factor(A) -> np.ndarray:
    """H = A^T A = sum_t a_t a_t^T in float64.

    ``A`` is (T, d); bf16/fp32 inputs are widened exactly to float64 first.
    """
    A64 = np.asarray(A, dtype=np.float64)
    return A64.T @ A64


def trace_of_factor(H) -> float:
    """tr(H) as the float64 sum of the diagonal."""
    return float(np.sum(np.diag(np.asarray(H, dtype=np.float64))))


def trace_from_rows(A) -> float:
    """tr(A^T A) = sum_t ||a_t||^2, computed straight from the tokens."""
    A64 = np.asarray(A, dtype=np.float64)
    return float(np.sum(A64 * A64))


def sensitivity(HX, HG):
    """(tr(H_X), tr(H_G), tr(H_G) * tr(H_X)) -- the KronQ sensitivity."""
    trx = trace_of_factor(HX)
    trg = trace_of_factor(HG)
    return trx, trg, trg * trx


def factor_columns(A, cols) -> np.ndarray:
    """Columns ``cols`` of H = A^T A: A^T a_j for each sampled j (float64)."""
    A64 = np.asarray(A, dtype=np.float64)
    return A64.T @ A64[:, list(cols)]
