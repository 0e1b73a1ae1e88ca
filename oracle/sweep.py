"""O4/O5: the quantization grid, damping, the Cholesky factor of the damped
inverse and the GPTQ column sweep under the K-FAC loss.

KronQ README (intro): KronQ extends GPTQ/GPTAQ; "Reproduce from scratch":
``--w_bits --w_groupsize --w_asym`` (2/3/4 bits, per-channel or group 128);
"Mapping paper results to flags": GPTQ and RTN (``--w_rtn``) baselines.

Why H_G does not enter the column sweep: for the K-FAC Hessian H_X (x) H_G,
the best compensation of the later columns for a fixed error e_j in column j
is -(H_X^-1)[:, j] / (H_X^-1)[j, j] (x) e_j; H_G cancels.  The sweep is
therefore GPTQ's, each row rounded on its own; H_G acts through BiIP and the
loss.

Readings fixed here (the pages are silent):

* Grid (asymmetric, per row and per group, dynamic groups): at a group's
  first column, from the current error-updated values of the group's columns,
  x_min = min(0, min w), x_max = max(0, max w); x_min = x_max -> (-1, 1);
  scale = (x_max - x_min) / (2^b - 1), zero = rint(-x_min / scale);
  q = clamp(rint(w / scale) + zero, 0, 2^b - 1), deq = scale (q - zero);
  rint is round-half-to-even.  Symmetric: scale = 2 max(|x_min|, x_max) /
  (2^b - 1), zero = 2^(b-1).  group = -1 is one group per row.
* Damping: columns whose diagonal is zero get H_jj := 1 and W[:, j] := 0;
  then lambda = damp_rel * mean(diag H) is added to the diagonal.
* U = upper Cholesky factor of (H + lambda I)^-1 (U^T U = (H + lambda I)^-1),
  by the plain definition: explicit inverse, then Cholesky.
* Sweep: for j = 0..n-1: quantize column j, e_j = (w_j - deq_j) / U_jj,
  W[:, j+1:] -= e_j U[j, j+1:].  ``block`` > 1 applies the same updates
  lazily (in-block rank-1, then one block product for the later columns),
  a re-association that is exact in exact arithmetic.  gptq_sweep_rform
  takes the same decisions from R = U^-1 (the factor of H + lambda I
  itself) and the diagonal blocks of U only.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------- grid
def grid_params(wg, bits: int, asym: bool = True, dtype=np.float64):
    """Per-row (scale, zero) from the group's current values ``wg`` (rows x g).

    With ``dtype=np.float32`` every operation is a single float32 operation
    (the schedule-mirroring mode)."""
    wg = np.asarray(wg, dtype=dtype)
    maxq = dtype(2 ** bits - 1)
    zero_c = dtype(0)
    xmin = np.minimum(wg.min(axis=1), zero_c)
    xmax = np.maximum(wg.max(axis=1), zero_c)
    if not asym:
        xmax = np.maximum(np.abs(xmin), xmax)
        xmin = -xmax
    tie = xmin == xmax
    xmin = np.where(tie, dtype(-1), xmin).astype(dtype)
    xmax = np.where(tie, dtype(1), xmax).astype(dtype)
    scale = ((xmax - xmin) / maxq).astype(dtype)
    if asym:
        zero = np.rint((-xmin) / scale).astype(dtype)
    else:
        zero = np.full_like(scale, dtype(2 ** (bits - 1)))
    return scale, zero


def quantize(w, scale, zero, bits: int, dtype=np.float64):
    """(codes, dequantised values) of a column ``w`` on the row grids."""
    w = np.asarray(w, dtype=dtype)
    maxq = dtype(2 ** bits - 1)
    q = np.clip(np.rint(w / scale) + zero, dtype(0), maxq).astype(dtype)
    deq = (scale * (q - zero)).astype(dtype)
    return q, deq


def rtn(W, bits: int, group: int, asym: bool = True):
    """Round-to-nearest on the same grid, no error feedback (``--w_rtn``)."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    g = n if group == -1 else group
    codes = np.zeros((m, n), dtype=np.int64)
    Q = np.zeros((m, n))
    for j0 in range(0, n, g):
        j1 = min(n, j0 + g)
        scale, zero = grid_params(W[:, j0:j1], bits, asym)
        for j in range(j0, j1):
            q, deq = quantize(W[:, j], scale, zero, bits)
            codes[:, j] = q.astype(np.int64)
            Q[:, j] = deq
    return codes, Q


# ---------------------------------------------------------------- factor
def dead_columns(H, W):
    """GPTQ's dead-column rule: zero diagonal -> H_jj := 1, W[:, j] := 0."""
    H = np.array(H, dtype=np.float64, copy=True)
    W = np.array(W, dtype=np.float64, copy=True)
    dead = np.diag(H) == 0
    idx = np.nonzero(dead)[0]
    H[idx, idx] = 1.0
    W[:, idx] = 0.0
    return H, W, dead


def damp(H, damp_rel: float = 0.01):
    """H + lambda I with lambda = damp_rel * mean(diag H)."""
    H = np.array(H, dtype=np.float64, copy=True)
    lam = damp_rel * float(np.mean(np.diag(H)))
    H[np.diag_indices_from(H)] += lam
    return H, lam


def chol_upper_of_inverse(A):
    """Upper triangular U with U^T U = A^-1: explicit inverse, then Cholesky."""
    Ainv = np.linalg.inv(np.asarray(A, dtype=np.float64))
    Ainv = 0.5 * (Ainv + Ainv.T)
    L = np.linalg.cholesky(Ainv)
    return L.T


def chol_upper_of_inverse_f32(A):
    """The same U computed in float32 by LAPACK: the Cholesky factor of the
    index-reversed float32 matrix (A = R R^T with R upper, eliminating from
    the last index), then the float32 triangular inverse U = R^-1.

    Not a step of the method: it measures what a float32 factorisation of a
    given factor can achieve (its error grows with the factor's condition
    number), the floor against which the float32 GPU factorisation is held.
    """
    import scipy.linalg as sl

    A32 = np.asarray(A, dtype=np.float32)
    n = A32.shape[0]
    L = sl.cholesky(np.ascontiguousarray(A32[::-1, ::-1]), lower=True, check_finite=False)
    R = np.ascontiguousarray(L[::-1, ::-1])
    return sl.solve_triangular(R, np.eye(n, dtype=np.float32), lower=False, check_finite=False)


def reverse_chol_failure(A) -> int:
    """LAPACK-style info for a factorisation that eliminates from the last
    index down: 0 when A is positive definite, else 1 + the largest j whose
    trailing principal submatrix A[j:, j:] is not positive definite."""
    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    for j in range(n - 1, -1, -1):
        if np.linalg.eigvalsh(A[j:, j:]).min() <= 0.0:
            return j + 1
    return 0


# ---------------------------------------------------------------- sweeps
def _group_bounds(j, n, group, block):
    """Is column j a group start, and the group's column range."""
    if group == -1:
        return (j == 0), 0, n
    if j % group == 0:
        return True, j, min(n, j + group)
    return False, None, None


def gptq_sweep(Wt, U, bits: int, group: int, asym: bool = True, block: int = 1,
               fixed_steps=None):
    """Float64 GPTQ sweep.  Returns dict(codes, scales, zeros, Q, E, W_final).

    ``fixed_steps`` (test hook for the Babai example): per-column grid steps
    alpha_j with unbounded integers, q_j = rint(w_j / alpha_j), deq = alpha_j q.
    """
    W = np.array(Wt, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    ng = 1 if group == -1 else -(-n // group)
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, ng))
    zeros = np.zeros((m, ng))
    Q = np.zeros((m, n))
    E = np.zeros((m, n))
    scale = zero = None
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        for j in range(b0, b1):
            if fixed_steps is None:
                start, g0, g1 = _group_bounds(j, n, group, block)
                if start:
                    scale, zero = grid_params(W[:, g0:g1], bits, asym)
                    gi = 0 if group == -1 else j // group
                    scales[:, gi] = scale
                    zeros[:, gi] = zero
                q, deq = quantize(W[:, j], scale, zero, bits)
            else:
                a = float(fixed_steps[j])
                q = np.rint(W[:, j] / a)
                deq = a * q
            codes[:, j] = q.astype(np.int64)
            Q[:, j] = deq
            e = (W[:, j] - deq) / U[j, j]
            E[:, j] = e
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
        W[:, b1:] -= E[:, b0:b1] @ U[b0:b1, b1:]
    return dict(codes=codes, scales=scales, zeros=zeros, Q=Q, E=E, W_final=W)


def gptq_sweep_rform(Wt, R, bits: int, group: int, asym: bool = True, block: int = 1):
    """The sweep of gptq_sweep taken from R itself (H + lambda I = R R^T, R
    upper, so U = R^-1), with only diagonal blocks of U formed.

    With the columns split into the swept ones S and the rest T, and F =
    (W - Q)_S R_ST (W the weights before the sweep, Q the dequantised values),
    gptq_sweep's partial state is W_T - E_S U_ST = W_T + F U_TT, because
    E_S = (W - Q)_S R_SS and R_SS U_ST = -R_ST U_TT.  So:
      * column j, when its turn comes, holds w_j + F_j / R_jj (U_TT is upper,
        and its (j, j) entry is 1 / R_jj once every earlier column is in S);
      * a group G starting at column c is gridded from W_G + F_G U_GG, U_GG =
        (R_GG)^-1 the group's diagonal block of U;
      * F accumulates (w_k - deq_k) R_k,: over the swept columns k.
    The codes, grids and E_j = (w~_j - deq_j) R_jj are those of gptq_sweep
    (pinned against it in the tests).  ``block`` only batches the updates of
    F (in-block rank-1, then one product for the later columns).
    """
    W0 = np.array(Wt, dtype=np.float64, copy=True)
    R = np.asarray(R, dtype=np.float64)
    rd = np.diag(R).copy()
    m, n = W0.shape
    F = np.zeros((m, n))
    ng = 1 if group == -1 else -(-n // group)
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, ng))
    zeros = np.zeros((m, ng))
    Q = np.zeros((m, n))
    E = np.zeros((m, n))
    D = np.zeros((m, n))
    Wcur = np.zeros((m, n))
    scale = zero = None
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        for j in range(b0, b1):
            start, g0, g1 = _group_bounds(j, n, group, block)
            if start:
                UGG = np.linalg.inv(np.triu(R[g0:g1, g0:g1]))
                scale, zero = grid_params(W0[:, g0:g1] + F[:, g0:g1] @ np.triu(UGG), bits, asym)
                gi = 0 if group == -1 else j // group
                scales[:, gi] = scale
                zeros[:, gi] = zero
            w = W0[:, j] + F[:, j] / rd[j]
            Wcur[:, j] = w
            q, deq = quantize(w, scale, zero, bits)
            codes[:, j] = q.astype(np.int64)
            Q[:, j] = deq
            E[:, j] = (w - deq) * rd[j]
            D[:, j] = W0[:, j] - deq
            F[:, j + 1:b1] += np.outer(D[:, j], R[j, j + 1:b1])
        F[:, b1:] += D[:, b0:b1] @ R[b0:b1, b1:]
    return dict(codes=codes, scales=scales, zeros=zeros, Q=Q, E=E, W_final=Wcur)


def gptq_sweep_f32(Wt, U, bits: int, group: int, asym: bool = True, block: int = 128):
    """Float32 sweep in a fixed operation order (bit-exact test mode).

    Every operation is one float32 operation, multiply and subtract not
    fused.  The grid of a group (scale, zero) uses correctly rounded
    divisions; per column, the divisions by scale and by U_jj are
    multiplications by the correctly rounded reciprocals 1/scale and 1/U_jj
    (float32 throughout, so both the library and this mirror take every
    rounding decision identically).  In a block the rank-1 updates run in
    column order; after the block, acc = sum_k E[:, k] U[k, later] is
    accumulated in ascending k (one rounding per product and per add) and
    then W[:, later] = W[:, later] - acc.
    """
    f32 = np.float32
    W = np.array(Wt, dtype=f32, copy=True)
    U = np.asarray(U, dtype=f32)
    m, n = W.shape
    ng = 1 if group == -1 else -(-n // group)
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, ng), dtype=f32)
    zeros = np.zeros((m, ng), dtype=f32)
    Q = np.zeros((m, n), dtype=f32)
    E = np.zeros((m, n), dtype=f32)
    scale = zero = None
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        for j in range(b0, b1):
            start, g0, g1 = _group_bounds(j, n, group, block)
            if start:
                scale, zero = grid_params(W[:, g0:g1], bits, asym, dtype=f32)
                inv_scale = (f32(1) / scale).astype(f32)
                gi = 0 if group == -1 else j // group
                scales[:, gi] = scale
                zeros[:, gi] = zero
            maxq = f32(2 ** bits - 1)
            q = np.clip(np.rint((W[:, j] * inv_scale).astype(f32)) + zero, f32(0), maxq).astype(f32)
            deq = (scale * (q - zero)).astype(f32)
            codes[:, j] = q.astype(np.int64)
            Q[:, j] = deq
            inv_u = f32(1) / U[j, j]
            e = ((W[:, j] - deq).astype(f32) * inv_u).astype(f32)
            E[:, j] = e
            if j + 1 < b1:
                prod = (e[:, None] * U[j, j + 1:b1][None, :]).astype(f32)
                W[:, j + 1:b1] = (W[:, j + 1:b1] - prod).astype(f32)
        if b1 < n:
            acc = np.zeros((m, n - b1), dtype=f32)
            for k in range(b0, b1):
                prod = (E[:, k][:, None] * U[k, b1:][None, :]).astype(f32)
                acc = (acc + prod).astype(f32)
            W[:, b1:] = (W[:, b1:] - acc).astype(f32)
    return dict(codes=codes, scales=scales, zeros=zeros, Q=Q, E=E, W_final=W)


def quantize_factored(Wt, Ht, bits: int, group: int, asym: bool = True,
                      damp_rel: float = 0.01, block: int = 1):
    """Dead columns, damping, U, then the float64 sweep (kronq_quantize_layer)."""
    H1, W1, dead = dead_columns(Ht, Wt)
    A, lam = damp(H1, damp_rel)
    U = chol_upper_of_inverse(A)
    res = gptq_sweep(W1, U, bits, group, asym, block)
    res.update(U=U, lam=lam, dead=dead, A=A, W_in=W1)
    return res
