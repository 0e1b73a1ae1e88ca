"""Pins for the oracle's factors (O1/O2) and BiIP (O3)."""
import json
import math
import os

import numpy as np
import pytest
import scipy.fft

from oracle import biip, factors, loss
from synth import tiny_layer


# ------------------------------------------------------------------ O1 / O2
def test_factor_hand_worked_2x2(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "factor_2x2.json")))
    H = factors.factor(np.array(g["X"]))
    assert np.array_equal(H, np.array(g["HX"]))
    assert factors.trace_of_factor(H) == g["trace"]
    assert factors.trace_from_rows(np.array(g["X"])) == g["trace"]


def test_factor_symmetric_psd_and_trace():
    W, X, G = tiny_layer()
    for A in (X, G):
        H = factors.factor(A)
        assert np.array_equal(H, H.T)
        ev = np.linalg.eigvalsh(H)
        assert ev.min() >= -1e-12 * np.abs(ev).max()
        t1 = factors.trace_of_factor(H)
        t2 = factors.trace_from_rows(A)
        assert abs(t1 - t2) <= 1e-12 * abs(t2)
        # entry (i, j) is the inner product of columns i and j
        A64 = A.astype(np.float64)
        i, j = 3, 17
        assert math.isclose(H[i, j], math.fsum(A64[:, i] * A64[:, j]), rel_tol=1e-12)


def test_sensitivity_is_product_of_traces():
    _, X, G = tiny_layer(m=64, n=32, T=100)
    HX, HG = factors.factor(X), factors.factor(G)
    trx, trg, s = factors.sensitivity(HX, HG)
    assert math.isclose(trx, factors.trace_from_rows(X), rel_tol=1e-12)
    assert math.isclose(trg, factors.trace_from_rows(G), rel_tol=1e-12)
    assert s == trg * trx


# ------------------------------------------------------------------ generator
def test_splitmix64_published_outputs(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "splitmix64.json")))
    assert biip.splitmix64(0, 0) == int(g["seed0_first"], 16)
    got = [biip.splitmix64(1234567, i) for i in range(5)]
    assert got == [int(v) for v in g["seed1234567_first5"]]


def test_signs_are_top_bit_and_sides_differ():
    s0 = biip.signs(7, 0, 1000)
    s1 = biip.signs(7, 1, 1000)
    assert set(np.unique(s0)) <= {-1.0, 1.0}
    assert 400 < np.sum(s0 > 0) < 600          # balanced
    assert np.mean(s0 == s1) < 0.6             # independent streams per side
    for i in (0, 1, 999):
        top = biip.splitmix64(15, i) >> 63
        assert s1[i] == (-1.0 if top else 1.0)


# ------------------------------------------------------------------ matrices
@pytest.mark.parametrize("K", [1, 3, 7, 43])
def test_dct_matches_scipy_orthonormal_dct2(K):
    C = biip.dct2_matrix(K)
    x = np.random.default_rng(K).normal(size=K)
    assert np.allclose(C @ x, scipy.fft.dct(x, type=2, norm="ortho"), atol=1e-13)


@pytest.mark.parametrize("P", [1, 2, 8, 64])
def test_hadamard_matches_popcount_form(P):
    Hm = biip.hadamard(P)
    ref = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(P)] for i in range(P)])
    assert np.array_equal(Hm, ref)


@pytest.mark.parametrize("n", [1, 8, 24, 43, 56, 86, 256, 344])
def test_rotation_orthogonal(n):
    V = biip.rotation_matrix(n, seed=3, side=0)
    assert np.max(np.abs(V @ V.T - np.eye(n))) < 1e-12
    # every entry bounded by sqrt(2/n) (incoherent)
    assert np.max(np.abs(V)) <= math.sqrt(2.0 / n) + 1e-15


def test_rotation_4096_orthogonal_by_probes():
    n = 4096
    rng = np.random.default_rng(0)
    M = rng.normal(size=(16, n))
    R = biip.rotate_rows(M, seed=5, side=1)
    assert np.allclose(np.linalg.norm(R, axis=1), np.linalg.norm(M, axis=1), rtol=1e-12)
    assert np.allclose(R @ R.T, M @ M.T, rtol=0, atol=1e-9)


def test_power_of_two_rotation_is_signed_hadamard():
    n = 64
    V = biip.rotation_matrix(n, seed=11, side=0)
    Hp = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(n)] for i in range(n)]) / 8.0
    assert np.allclose(V, Hp * biip.signs(11, 0, n)[None, :], atol=1e-15)


@pytest.mark.parametrize("n", [8, 56, 86])
def test_rotate_rows_equals_dense(n):
    rng = np.random.default_rng(n)
    M = rng.normal(size=(5, n))
    V = biip.rotation_matrix(n, seed=2, side=1)
    assert np.allclose(biip.rotate_rows(M, 2, 1), M @ V.T, atol=1e-12)
    assert np.allclose(biip.rotate_rows(M, 2, 1, inverse=True), M @ V, atol=1e-12)


# ------------------------------------------------------------------ BiIP
def _layer(m=48, n=56, T=300, seed=1):
    W, X, G = tiny_layer(m=m, n=n, T=T, seed=seed)
    return W.astype(np.float64), factors.factor(X), factors.factor(G)


def test_no_rescale_preserves_frobenius_norm():
    W, HX, HG = _layer()
    Wt, HXt, HGt, din, dout = biip.biip_forward(W, HX, HG, 4, 0.25, "no_rescale")
    assert np.all(din == 1.0) and np.all(dout == 1.0)
    assert abs(np.linalg.norm(Wt) - np.linalg.norm(W)) <= 1e-12 * np.linalg.norm(W)
    assert abs(np.trace(HXt) - np.trace(HX)) <= 1e-12 * np.trace(HX)


@pytest.mark.parametrize("mode", ["full", "no_rescale", "su_only", "sv_only"])
def test_kfac_loss_invariant(mode):
    W, HX, HG = _layer(m=40, n=24)
    _, HXt, HGt, din, dout = biip.biip_forward(W, HX, HG, 9, 0.25, mode)
    dW = np.random.default_rng(2).normal(size=W.shape) * 1e-3
    use_in = mode in ("full", "no_rescale", "sv_only")
    use_out = mode in ("full", "no_rescale", "su_only")
    dWt = dout[:, None] * dW * din[None, :]
    if use_in:
        dWt = biip.rotate_rows(dWt, 9, 0)
    if use_out:
        dWt = biip.rotate_rows(dWt.T, 9, 1).T
    a = loss.kfac_loss(dW, HX, HG)
    b = loss.kfac_loss(dWt, HXt, HGt)
    assert abs(a - b) <= 1e-12 * abs(a)


@pytest.mark.parametrize("mode", ["full", "no_rescale", "su_only", "sv_only"])
def test_forward_then_inverse_is_identity(mode):
    W, HX, HG = _layer()
    Wt, _, _, din, dout = biip.biip_forward(W, HX, HG, 13, 0.25, mode)
    back = biip.biip_inverse(Wt, 13, mode, din, dout)
    assert np.max(np.abs(back - W)) <= 1e-12 * np.max(np.abs(W))


def test_mode_sides():
    W, HX, HG = _layer()
    _, HXt, HGt, din, _ = biip.biip_forward(W, HX, HG, 1, 0.25, "su_only")
    assert np.array_equal(HXt, HX) and np.all(din == 1.0)
    _, HXt, HGt, _, dout = biip.biip_forward(W, HX, HG, 1, 0.25, "sv_only")
    assert np.array_equal(HGt, HG) and np.all(dout == 1.0)


def test_quarter_power_rescale_minimises_proxy():
    # At alpha = 1/4, d minimises tr(D^-1 H D^-1) * ||W D||_F^2; random +-1%
    # perturbations of d never lower it.
    W, HX, _ = _layer(m=32, n=40, seed=5)
    din = biip.rescale_vector(np.diag(HX), np.sum(W * W, axis=0), 0.25)

    def proxy(d):
        return np.sum(np.diag(HX) / d ** 2) * np.sum((W * d[None, :]) ** 2)

    base = proxy(din)
    rng = np.random.default_rng(0)
    for _ in range(200):
        p = din * (1.0 + 0.01 * rng.uniform(-1, 1, size=din.shape))
        assert proxy(p) >= base * (1 - 1e-13)
    # and the closed form d_j^2 ∝ sqrt(H_jj) / ||W_j||
    r = din ** 2 * np.linalg.norm(W, axis=0) / np.sqrt(np.diag(HX))
    assert np.allclose(r, r[0], rtol=1e-12)
    assert abs(np.sum(np.log(din))) < 1e-10          # geometric mean 1


def test_degenerate_rescale_entries():
    d = biip.rescale_vector([0.0, 4.0, 1.0], [1.0, 0.0, 1.0], 0.25)
    # raw values (1, 1, 1) -> all one after the geometric-mean normalisation
    assert np.allclose(d, 1.0)
