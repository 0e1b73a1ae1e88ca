"""The blocked orders of two GPU kernels, replayed in float64 against the
oracle (no GPU).  They check the decomposition the kernels are written
from, not the kernels themselves (the GPU parity tests do that):

* two-sided rounding: 32 x 32 tiles along anti-diagonals; inside a tile,
  row r takes column t - r at step t with the cross-row sum over the rows
  above; after each anti-diagonal, P[I, later] += E[I, J] U_X[J, later]
  (row direction) and W~[later, J] -= U_G[I, later]^T P[I, J] (column
  direction).  Equal to the element-by-element sweep up to rounding order.
* the 28672-long BiIP row pass: the Hadamard index a (12 bits) held four
  bits at a time in registers (a = 256 u + 32 w + l, then u + 16 l + 512 w,
  then (l & 15) + 16 u + 256 (l >> 4) + 512 w), the exchanges through the
  padded layout 7 a + b + (a >> 4).  Equal to the oracle's row rotation, and
  the padded exchanges are free of shared-memory bank conflicts."""
import numpy as np
import pytest

from oracle import biip, sweep, twosided

TR = TC = 32


def _tiled_two_sided(W0, UX, UG, bits, group):
    m, n = W0.shape
    W = W0.copy()
    sc, zp = twosided.static_grid(W0, bits, group)
    P = np.zeros((m, n))
    E = np.zeros((m, n))
    codes = np.zeros((m, n), dtype=np.int64)
    NI, NJ = -(-m // TR), -(-n // TC)
    maxq = 2 ** bits - 1
    for s in range(NI + NJ - 1):
        tiles = [(I, s - I) for I in range(max(0, s - NJ + 1), min(NI - 1, s) + 1)]
        for I, J in tiles:
            r0, c0 = I * TR, J * TC
            rows, cols = min(TR, m - r0), min(TC, n - c0)
            X = UX[c0:c0 + cols, c0:c0 + cols]
            G = UG[r0:r0 + rows, r0:r0 + rows]
            Pm = P[r0:r0 + rows, c0:c0 + cols].copy()
            S = W[r0:r0 + rows, c0:c0 + cols] - np.triu(G).T @ Pm
            w = S.copy()
            PL = np.zeros_like(S)
            for t in range(rows + cols - 1):
                for r in range(rows):
                    c = t - r
                    if not 0 <= c < cols:
                        continue
                    x = sum(G[k, r] * PL[k, c] for k in range(r))
                    wt = w[r, c] - x
                    g = 0 if group == -1 else (c0 + c) // group
                    q = min(max(np.rint(wt / sc[r0 + r, g]) + zp[r0 + r, g], 0), maxq)
                    deq = sc[r0 + r, g] * (q - zp[r0 + r, g])
                    e1 = (wt - deq) / X[c, c]
                    W[r0 + r, c0 + c] = deq
                    codes[r0 + r, c0 + c] = q
                    E[r0 + r, c0 + c] = e1 / G[r, r]
                    PL[r, c] = (S[r, c] - x - deq) / G[r, r]
                    w[r, c + 1:] -= e1 * X[c, c + 1:]
            P[r0:r0 + rows, c0:c0 + cols] = Pm + PL
        for I, J in tiles:
            r0, c0 = I * TR, J * TC
            rows, cols = min(TR, m - r0), min(TC, n - c0)
            P[r0:r0 + rows, c0 + cols:] += E[r0:r0 + rows, c0:c0 + cols] @ UX[c0:c0 + cols, c0 + cols:]
            W[r0 + rows:, c0:c0 + cols] -= UG[r0:r0 + rows, r0 + rows:].T @ P[r0:r0 + rows, c0:c0 + cols]
    return codes, W, E


@pytest.mark.parametrize("m,n,group", [(40, 70, 32), (70, 100, 16), (33, 65, -1), (65, 40, 1)])
def test_two_sided_tile_schedule_equals_the_sweep(m, n, group):
    rng = np.random.default_rng(m * n)
    W0 = rng.normal(0, 0.02, (m, n))
    X = rng.standard_normal((3 * n, n))
    G = rng.standard_normal((3 * m, m))
    UX = sweep.chol_upper_of_inverse(sweep.damp(X.T @ X, 0.01)[0])
    UG = sweep.chol_upper_of_inverse(sweep.damp(G.T @ G, 0.01)[0])
    ref = twosided.two_sided_sweep(W0, UX, UG, 2, group)
    codes, Q, E = _tiled_two_sided(W0, UX, UG, 2, group)
    assert np.array_equal(codes, ref["codes"])
    assert np.abs(Q - ref["Q"]).max() <= 1e-12
    # (with one column per group every value starts on its own grid and E is
    # rounding noise of ~1e-15: hence the absolute floor)
    assert np.abs(E - ref["E"]).max() <= 1e-9 * np.abs(ref["E"]).max() + 1e-12


def _pad(a):
    return 7 * a + (a >> 4)


def _radix16(x):
    x = x.copy()
    h = 1
    while h < 16:
        for u in range(16):
            if u & h == 0:
                s0, s1 = x[u].copy(), x[u | h].copy()
                x[u], x[u | h] = s0 + s1, s0 - s1
        h <<= 1
    return x


def test_row_pass_28672_index_maps_equal_the_rotation():
    L, P = 28672, 4096
    seed, side = 5, 0
    rng = np.random.default_rng(0)
    x0 = rng.standard_normal(L)
    d = np.exp(0.3 * rng.standard_normal(L))
    cf = biip.signs(seed, side, L) * d
    C = biip.dct2_matrix(7)
    sm = np.zeros(L + P // 16)
    for w in range(8):                      # phase 1: a = 256 u + 32 w + l
        for l in range(32):
            x = np.zeros((16, 7))
            for u in range(16):
                a = 256 * u + 32 * w + l
                x[u] = C @ (x0[7 * a:7 * a + 7] * cf[7 * a:7 * a + 7])
            x = _radix16(x)
            for u in range(16):
                p = _pad(256 * u + 32 * w + l)
                sm[p:p + 7] = x[u]
    for w in range(8):                      # phase 2: a = u + 16 l + 512 w
        for l in range(32):
            pos = [_pad(u + 16 * l + 512 * w) for u in range(16)]
            x = _radix16(np.array([sm[p:p + 7] for p in pos]))
            for u, p in enumerate(pos):
                sm[p:p + 7] = x[u]
    out = np.zeros(L)
    for w in range(8):                      # phase 3: bits 4-7 in registers
        for l in range(32):
            a3 = (l & 15) + 256 * (l >> 4) + 512 * w
            x = _radix16(np.array([sm[_pad(a3 + 16 * u):_pad(a3 + 16 * u) + 7] for u in range(16)]))
            for u in range(16):
                out[7 * (a3 + 16 * u):7 * (a3 + 16 * u) + 7] = x[u] / 64.0
    ref = biip.rotate_rows((x0 * d)[None, :], seed, side)[0]
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()
    assert _pad(P - 1) + 6 < L + P // 16                     # the padded layout fits its buffer

    def worst_conflict(addr):
        worst = 0
        for w in range(8):
            for u in range(16):
                banks = [addr(w, l, u) % 32 for l in range(32)]
                worst = max(worst, max(banks.count(b) for b in set(banks)))
        return worst
    assert worst_conflict(lambda w, l, u: _pad(u + 16 * l + 512 * w)) == 1
    assert worst_conflict(lambda w, l, u: _pad((l & 15) + 256 * (l >> 4) + 512 * w + 16 * u)) == 1
    assert worst_conflict(lambda w, l, u: 7 * (256 * u + 32 * w + l)) == 1
