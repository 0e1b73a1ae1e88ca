"""Two-sided adaptive rounding under H_X (x) H_G (float64).

TEST INFRASTRUCTURE ONLY (see the package header).

Source: the BaKron abstract ("BaKron: Efficient Quantization with
Kronecker-Factored Hessians" page): GPTQ-style rounding applied in the
vectorised weight domain with a two-sided Kronecker-factored Hessian, solved
with anti-diagonal parallelism in O(m + n) sequential steps and O(mn(m+n))
work; modular in the base quantizer and the Hessian estimator.  The abstract
gives no algorithm; the reading taken is the plain definition of GPTQ on
vec(W) under H = H_X (x) H_G:

* The loss tr(dW H_X dW^T H_G) is vec(dW)^T (H_X (x) H_G) vec(dW) (columns
  stacked).  With U_X^T U_X = (H_X + lambda_X I)^-1 and U_G likewise (both
  damped by the relative rule of the one-sided pass), the upper Cholesky
  factor of the inverse Kronecker Hessian is U = U_X (x) U_G, whose entry
  for element (i, j) -> (i', j') (row i of W is output i, column j input j)
  is U_X[j, j'] U_G[i, i'], non-zero only for j' >= j and i' >= i.
* GPTQ on vec(W) with that factor: element (i, j) is quantized to deq, its
  scaled error e = (w_ij - deq) / (U_X[j, j] U_G[i, i]) is fed back as
  w_i'j' -= e U_X[j, j'] U_G[i, i'] to every later element (i' >= i,
  j' >= j, not (i, j) itself).  An element depends only on the elements
  above-left of it, so every processing order that respects that partial
  order (row-major, column-major, anti-diagonal wavefronts) gives the same
  result; the oracle runs row-major.
* Base quantizer: the asymmetric grid of the one-sided pass per row and
  group, fixed before the sweep from the values the sweep starts from
  (static groups: a grid taken at a group start would depend on the order).

Pinned in tests/test_oracle_twosided.py.
"""
from __future__ import annotations

import numpy as np

from . import sweep


def static_grid(W, bits: int, group: int, asym: bool = True):
    """Per-row, per-group (scale, zero) from W itself (m x ngroups each)."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    ng = 1 if group == -1 else -(-n // group)
    sc = np.zeros((m, ng))
    zp = np.zeros((m, ng))
    for g in range(ng):
        c0, c1 = (0, n) if group == -1 else (g * group, min(n, (g + 1) * group))
        sc[:, g], zp[:, g] = sweep.grid_params(W[:, c0:c1], bits, asym)
    return sc, zp


def _group_of(j: int, group: int) -> int:
    return 0 if group == -1 else j // group


def two_sided_sweep(Wt, UX, UG, bits: int, group: int, asym: bool = True, order: str = "row"):
    """GPTQ on vec(W) with the factor UX (x) UG and static grids.

    order: "row" (row-major), "col" (column-major) or "anti" (anti-diagonal
    wavefronts i + j = const) -- the same result for all three.
    Returns dict(codes, Q, E, scales, zeros).
    """
    W = np.array(Wt, dtype=np.float64, copy=True)
    UX = np.asarray(UX, dtype=np.float64)
    UG = np.asarray(UG, dtype=np.float64)
    m, n = W.shape
    sc, zp = static_grid(W, bits, group, asym)
    codes = np.zeros((m, n), dtype=np.int64)
    Q = np.zeros((m, n))
    E = np.zeros((m, n))
    if order == "row":
        seq = [(i, j) for i in range(m) for j in range(n)]
    elif order == "col":
        seq = [(i, j) for j in range(n) for i in range(m)]
    elif order == "anti":
        seq = [(i, s - i) for s in range(m + n - 1) for i in range(m) if 0 <= s - i < n]
    else:
        raise ValueError(order)
    for i, j in seq:
        g = _group_of(j, group)
        q, deq = sweep.quantize(W[i:i + 1, j], sc[i:i + 1, g], zp[i:i + 1, g], bits)
        codes[i, j] = int(q[0])
        Q[i, j] = deq[0]
        e = (W[i, j] - deq[0]) / (UX[j, j] * UG[i, i])
        E[i, j] = e
        upd = e * np.outer(UG[i, i:], UX[j, j:])
        upd[0, 0] = 0.0
        W[i:, j:] -= upd
    return dict(codes=codes, Q=Q, E=E, scales=sc, zeros=zp)


def quantize_two_sided(Wt, HXt, HGt, bits: int, group: int, asym: bool = True, damp_rel: float = 0.01,
                       order: str = "row"):
    """Damping of both factors, their inverse Cholesky factors, the sweep."""
    AX, lam_x = sweep.damp(HXt, damp_rel)
    AG, lam_g = sweep.damp(HGt, damp_rel)
    UX = sweep.chol_upper_of_inverse(AX)
    UG = sweep.chol_upper_of_inverse(AG)
    res = two_sided_sweep(Wt, UX, UG, bits, group, asym, order)
    res.update(UX=UX, UG=UG, AX=AX, AG=AG)
    return res
