"""Deploy-path matvec from packed codes (float64).

TEST INFRASTRUCTURE ONLY (see the package header).

KronQ README intro: quantized weights are stored packed int4/int2 and a
fused dequant + BiIP matvec unpacks them on the fly for single-token decode
(integer weights times activations).  What it computes, written as the plain
definition:

  Q[i, j]  = scale[i, g(j)] (q[i, j] - zero[i, g(j)]),  g(j) = j // group
             (one group per row when group == -1), q unpacked from the words
  W_hat    = D_o^-1 U^T Q V D_i^-1     (the inverse BiIP of Q, biip.py)
  y        = W_hat x

so that W_hat approximates the original W and y its product with the
activation x.  Pinned in tests/test_oracle_decode.py (hand-worked
dequantisation, dense rotation matrices, round trip through the pipeline).
"""
from __future__ import annotations

import numpy as np

from . import biip, pack


def dequantize(words, scales, zeros, n: int, bits: int, group: int) -> np.ndarray:
    """Q (m x n, float64) from packed words and per-group scales and zeros."""
    q = pack.unpack(words, n, bits).astype(np.float64)
    sc = np.asarray(scales, dtype=np.float64)
    zp = np.asarray(zeros, dtype=np.float64)
    g = np.zeros(n, dtype=np.int64) if group == -1 else np.arange(n) // group
    return sc[:, g] * (q - zp[:, g])


def decode_matvec(words, scales, zeros, bits: int, group: int, seed: int, mode: str, d_in, d_out,
                  x) -> np.ndarray:
    """y = D_o^-1 U^T Q V D_i^-1 x for one activation vector x (length n)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    Q = dequantize(words, scales, zeros, n, bits, group)
    W_hat = biip.biip_inverse(Q, seed, mode, d_in, d_out)
    return W_hat @ x
