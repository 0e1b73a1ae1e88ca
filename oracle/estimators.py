"""Kronecker factor estimators A (x) B ~ H = E[x x^T (x) g g^T] (float64).

TEST INFRASTRUCTURE ONLY (see the package header).

Source: "WaterKron and FlipFlop Hessian" page, Table 1 ("Different Hessian
approximations") and its caption, and the abstract (minimising the
Kronecker-Hessian mismatch factor Phi is a Gaussian covariance-fitting
problem with the classical flip-flop updates).  x is an input row (length
n), g an output-gradient row (length m), E the mean over the T tokens.

  input      A = E[x x^T],                 B = I_m
  marginal   A = E[x x^T],                 B = E[g g^T]
  Frobenius  A = E[(g^T B g) x x^T],       B = E[(x^T A x) g g^T]
  FlipFlop   A = E[(g^T B^-1 g) x x^T],    B = E[(x^T A^-1 x) g g^T]

Frobenius and FlipFlop run the alternating fixed-point iteration from the
identity (caption of Table 1): A from the current B, then B from the new A,
``iters`` times.  The table prints the updates up to constant factors; the
readings taken here (each the exact minimiser of the stated target over one
factor with the other fixed):

* Frobenius targets ||H - A (x) B||_F.  For fixed B its least-squares A is
  E[(g^T B g) x x^T] / ||B||_F^2, and symmetrically for B.
* FlipFlop targets the Gaussian covariance fit: minimise
  F(A, B) = E[(x^T A^-1 x)(g^T B^-1 g)] + m log det A + n log det B
  (= tr((A (x) B)^-1 H) + log det (A (x) B)).  For fixed B its minimiser is
  E[(g^T B^-1 g) x x^T] / m, and for fixed A, E[(x^T A^-1 x) g g^T] / n.

Each step is an exact block minimisation, so the target never increases
along the iteration; that, the nearest-Kronecker-product SVD (Van Loan) and
exactly Kronecker-structured samples pin this module (tests/test_oracle_estimators.py).
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def second_moment(A):
    """E[a a^T] over the rows of A (T x d)."""
    A = _f64(A)
    return A.T @ A / A.shape[0]


def weighted_second_moment(A, w):
    """E[w_t a_t a_t^T] over the rows of A with per-row weights w."""
    A = _f64(A)
    return (A * _f64(w)[:, None]).T @ A / A.shape[0]


def quad_forms(A, M):
    """a_t^T M a_t for every row a_t of A."""
    A = _f64(A)
    return np.einsum("ti,ij,tj->t", A, _f64(M), A)


def input_factors(X, G):
    """Table 1, row "Input": (E[x x^T], I_m)."""
    return second_moment(X), np.eye(_f64(G).shape[1])


def marginal_factors(X, G):
    """Table 1, row "Marginal": (E[x x^T], E[g g^T])."""
    return second_moment(X), second_moment(G)


def frobenius(X, G, iters: int = 10):
    """Table 1, row "Frobenius": alternating least squares from the identity.

    Returns (A, B, history) with history[k] = ||H - A (x) B||_F^2 after sweep
    k + 1 (computed without forming H, from frob_objective).
    """
    X, G = _f64(X), _f64(G)
    m = G.shape[1]
    B = np.eye(m)
    hist = []
    for _ in range(iters):
        A = weighted_second_moment(X, quad_forms(G, B)) / np.sum(B * B)
        B = weighted_second_moment(G, quad_forms(X, A)) / np.sum(A * A)
        hist.append(frob_objective(X, G, A, B))
    return A, B, hist


def flipflop(X, G, iters: int = 10):
    """Table 1, row "FlipFlop": the flip-flop iteration from the identity.

    Returns (A, B, history) with history[k] = F(A, B) (flipflop_objective)
    after sweep k + 1.
    """
    X, G = _f64(X), _f64(G)
    n, m = X.shape[1], G.shape[1]
    B = np.eye(m)
    hist = []
    for _ in range(iters):
        A = weighted_second_moment(X, quad_forms(G, np.linalg.inv(B))) / m
        B = weighted_second_moment(G, quad_forms(X, np.linalg.inv(A))) / n
        hist.append(flipflop_objective(X, G, A, B))
    return A, B, hist


def kron_hessian(X, G):
    """Dense H = E[x x^T (x) g g^T] (n m x n m); tiny sizes only."""
    X, G = _f64(X), _f64(G)
    T = X.shape[0]
    H = np.zeros((X.shape[1] * G.shape[1],) * 2)
    for t in range(T):
        H += np.kron(np.outer(X[t], X[t]), np.outer(G[t], G[t]))
    return H / T


def frob_objective(X, G, A, B):
    """||H - A (x) B||_F^2 = ||H||^2 - 2 E[(x^T A x)(g^T B g)] + ||A||^2 ||B||^2.

    ||H||_F^2 = E_s E_t (x_s . x_t)^2 (g_s . g_t)^2 (T^2 terms).
    """
    X, G = _f64(X), _f64(G)
    T = X.shape[0]
    hh = np.sum(((X @ X.T) ** 2) * ((G @ G.T) ** 2)) / (T * T)
    cross = np.mean(quad_forms(X, A) * quad_forms(G, B))
    return float(hh - 2.0 * cross + np.sum(A * A) * np.sum(B * B))


def flipflop_objective(X, G, A, B):
    """F(A, B) = E[(x^T A^-1 x)(g^T B^-1 g)] + m log det A + n log det B."""
    X, G = _f64(X), _f64(G)
    n, m = X.shape[1], G.shape[1]
    sa, la = np.linalg.slogdet(_f64(A))
    sb, lb = np.linalg.slogdet(_f64(B))
    if sa <= 0 or sb <= 0:
        return float("inf")
    q = quad_forms(X, np.linalg.inv(A)) * quad_forms(G, np.linalg.inv(B))
    return float(np.mean(q) + m * la + n * lb)
