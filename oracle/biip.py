"""O3: bidirectional incoherence processing (BiIP).

KronQ abstract, point (1), and KronQ README bullet "Bidirectional incoherence
processing (BiIP)": an incoherence rotation plus a rescale applied on both the
input and the output side of W, the output side driven by the gradient
covariance H_G; it reduces the spread of weight magnitudes along both
dimensions.  README "Reproduce from scratch": ``--incoh_rotate --incoh_kernel
had --incoh_mode full --alpha 0.25``; "Mapping paper results to flags":
modes {full, no_rescale, su_only, sv_only}, alpha 0.25 for weight-only.
README "Acknowledgements": the incoherence machinery follows QuIP#.

The pages give no formula, so these readings are fixed here (and followed by
the CUDA path):

* Rescale first, then rotate.
  d_in[j]  = (H_X[j, j] / ||W[:, j]||^2) ** alpha
  d_out[i] = (H_G[i, i] / ||W[i, :]||^2) ** alpha
  both from the original W and factors; a zero diagonal or zero norm gives a
  raw value of 1; each vector is then divided by its geometric mean.
  At alpha = 1/4 this is the minimiser of tr(D^-1 H D^-1) * ||W D||_F^2
  (Cauchy-Schwarz), the diagonal rescale of the QuIP line.
  W' = D_o W D_i,  H'_X = D_i^-1 H_X D_i^-1,  H'_G = D_o^-1 H_G D_o^-1.
* Rotation V (n x n) = (Had_{2^k} / sqrt(2^k)  (x)  C_K) . diag(s_in) with
  n = 2^k K, K odd, C_K the orthonormal DCT-II of order K (C_1 = [1]); the
  output side U (m x m) is built the same way with s_out.  No Hadamard matrix
  exists for odd K, so the DCT carries the odd factor.
* Signs s_side[i] = 1 - 2 * bit63(splitmix64(2 * seed + side, i)), side 0 =
  input (V), side 1 = output (U).  splitmix64(s, i) is output i of the
  SplitMix64 generator (Steele, Lea and Flood 2014) started from state s:
  mix64(s + (i + 1) * 0x9E3779B97F4A7C15 mod 2^64).
* W~ = U W' V^T,  H~_X = V H'_X V^T,  H~_G = U H'_G U^T.
* Modes: no_rescale sets D = I; su_only keeps only the output side (U, D_o);
  sv_only keeps only the input side (V, D_i).
"""
from __future__ import annotations

import math

import numpy as np

GOLDEN_GAMMA = 0x9E3779B97F4A7C15
_MASK64 = (1 << 64) - 1

MODES = ("full", "no_rescale", "su_only", "sv_only")


# ---------------------------------------------------------------- generator
def mix64(z: int) -> int:
    """The SplitMix64 output mix (Python integers, explicit 2^64 wrap)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def splitmix64(state0: int, i: int) -> int:
    """Output number ``i`` (0-based) of SplitMix64 started at ``state0``."""
    return mix64((state0 + (i + 1) * GOLDEN_GAMMA) & _MASK64)


def signs(seed: int, side: int, n: int) -> np.ndarray:
    """Random +-1 vector of length n for ``side`` (0 input, 1 output)."""
    s0 = (2 * int(seed) + int(side)) & _MASK64
    return np.array([1.0 - 2.0 * (splitmix64(s0, i) >> 63) for i in range(n)],
                    dtype=np.float64)


# ---------------------------------------------------------------- matrices
def split_pow2_odd(n: int):
    """n = 2^k * K with K odd; returns (2^k, K)."""
    if n <= 0:
        raise ValueError("n must be positive")
    p = 1
    while n % (2 * p) == 0:
        p *= 2
    return p, n // p


def dct2_matrix(K: int) -> np.ndarray:
    """Orthonormal DCT-II: C[i, j] = sqrt(2/K) c_i cos(pi (2j+1) i / (2K)),
    c_0 = 1/sqrt(2), c_i = 1 otherwise."""
    C = np.empty((K, K), dtype=np.float64)
    for i in range(K):
        ci = math.sqrt(0.5) if i == 0 else 1.0
        for j in range(K):
            C[i, j] = math.sqrt(2.0 / K) * ci * math.cos(math.pi * (2 * j + 1) * i / (2 * K))
    return C


def hadamard(P: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order P (a power of two), unnormalised."""
    Hm = np.ones((1, 1), dtype=np.float64)
    while Hm.shape[0] < P:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    return Hm


def rotation_matrix(n: int, seed: int, side: int) -> np.ndarray:
    """Dense V = (Had_P / sqrt(P) (x) C_K) diag(s) (small n only)."""
    P, K = split_pow2_odd(n)
    core = np.kron(hadamard(P) / math.sqrt(P), dct2_matrix(K))
    return core * signs(seed, side, n)[None, :]


def rotate_rows(M, seed: int, side: int, inverse: bool = False) -> np.ndarray:
    """Apply the rotation to every row of M (r x n).

    forward:  row v -> (V v^T)^T, i.e. M V^T
    inverse:  row v -> v V,       i.e. M V      (V orthogonal: undoes forward)
    Uses the Kronecker identity (A (x) B) vec_r(Y) = vec_r(A Y B^T) for the
    row-major reshape Y[a, b] = v[a K + b].
    """
    M = np.asarray(M, dtype=np.float64)
    r, n = M.shape
    P, K = split_pow2_odd(n)
    Hn = hadamard(P) / math.sqrt(P)
    C = dct2_matrix(K)
    s = signs(seed, side, n)
    if not inverse:
        Y = (M * s[None, :]).reshape(r, P, K)
        Z = np.einsum("ac,rcb,db->rad", Hn, Y, C, optimize=True)
        return Z.reshape(r, n)
    Y = M.reshape(r, P, K)
    Z = np.einsum("ac,rcb,bd->rad", Hn, Y, C, optimize=True)  # Hn Y C (Had symmetric)
    return Z.reshape(r, n) * s[None, :]


# ---------------------------------------------------------------- rescale
def _side_flags(mode: str):
    if mode not in MODES:
        raise ValueError(f"unknown BiIP mode {mode!r}")
    use_in = mode in ("full", "no_rescale", "sv_only")
    use_out = mode in ("full", "no_rescale", "su_only")
    rescale = mode != "no_rescale"
    return use_in, use_out, rescale


def _geo_normalised(raw: np.ndarray) -> np.ndarray:
    return raw / math.exp(float(np.mean(np.log(raw))))


def rescale_vector(hdiag, wnorm2, alpha: float) -> np.ndarray:
    """(hdiag / wnorm2) ** alpha, degenerate entries 1, geometric mean 1."""
    hdiag = np.asarray(hdiag, dtype=np.float64)
    wnorm2 = np.asarray(wnorm2, dtype=np.float64)
    ok = (hdiag > 0) & (wnorm2 > 0)
    raw = np.ones_like(hdiag)
    raw[ok] = (hdiag[ok] / wnorm2[ok]) ** alpha
    return _geo_normalised(raw)


def biip_scales(W, HX, HG, alpha: float, mode: str):
    """(d_in, d_out) for the mode; a side that is off or not rescaled is 1."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    use_in, use_out, rescale = _side_flags(mode)
    d_in = np.ones(n)
    d_out = np.ones(m)
    if rescale and use_in:
        d_in = rescale_vector(np.diag(HX), np.sum(W * W, axis=0), alpha)
    if rescale and use_out:
        d_out = rescale_vector(np.diag(HG), np.sum(W * W, axis=1), alpha)
    return d_in, d_out


# ---------------------------------------------------------------- transforms
def _two_sided(M, left_seed_side, right_seed_side, seed):
    """U M V^T for the requested sides (None = identity on that side)."""
    out = np.asarray(M, dtype=np.float64)
    if right_seed_side is not None:
        out = rotate_rows(out, seed, right_seed_side)
    if left_seed_side is not None:
        out = rotate_rows(out.T, seed, left_seed_side).T
    return out


def biip_forward(W, HX, HG, seed: int, alpha: float, mode: str = "full"):
    """Return (W~, H~_X, H~_G, d_in, d_out).  ``HG`` may be None when the
    mode does not need it (sv_only)."""
    W = np.asarray(W, dtype=np.float64)
    HX = np.asarray(HX, dtype=np.float64)
    use_in, use_out, _ = _side_flags(mode)
    if HG is None and use_out and mode != "no_rescale":
        raise ValueError("H_G is required for the output side")
    HGd = np.asarray(HG, dtype=np.float64) if HG is not None else np.eye(W.shape[0])
    d_in, d_out = biip_scales(W, HX, HGd, alpha, mode)
    Wp = d_out[:, None] * W * d_in[None, :]
    HXp = HX / d_in[:, None] / d_in[None, :]
    Wt = _two_sided(Wp, 1 if use_out else None, 0 if use_in else None, seed)
    HXt = _two_sided(HXp, 0 if use_in else None, 0 if use_in else None, seed)
    HGt = None
    if HG is not None:
        HGp = HGd / d_out[:, None] / d_out[None, :]
        HGt = _two_sided(HGp, 1 if use_out else None, 1 if use_out else None, seed)
    return Wt, HXt, HGt, d_in, d_out


def biip_inverse(Wt, seed: int, mode: str, d_in, d_out) -> np.ndarray:
    """W = D_o^-1 U^T W~ V D_i^-1 (undoes biip_forward on W)."""
    use_in, use_out, _ = _side_flags(mode)
    out = np.asarray(Wt, dtype=np.float64)
    if use_in:
        out = rotate_rows(out, seed, 0, inverse=True)
    if use_out:
        out = rotate_rows(out.T, seed, 1, inverse=True).T
    return out / np.asarray(d_out, dtype=np.float64)[:, None] / np.asarray(d_in, dtype=np.float64)[None, :]
