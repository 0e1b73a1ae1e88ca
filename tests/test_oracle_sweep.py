"""Pins for the oracle's grid, factorisation and sweeps (O4/O5/O6)."""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import biip, factors, loss, sweep
from synth import tiny_layer


def _rtn_independent(W, bits, group):
    """Round-to-nearest written straight from the grid reading, vectorised."""
    m, n = W.shape
    g = n if group == -1 else group
    codes = np.empty((m, n), dtype=np.int64)
    maxq = 2 ** bits - 1
    for j0 in range(0, n, g):
        blk = W[:, j0:j0 + g]
        lo = np.minimum(blk.min(1), 0.0)
        hi = np.maximum(blk.max(1), 0.0)
        same = lo == hi
        lo[same], hi[same] = -1.0, 1.0
        sc = (hi - lo) / maxq
        z = np.rint(-lo / sc)
        codes[:, j0:j0 + g] = np.clip(np.rint(blk / sc[:, None]) + z[:, None], 0, maxq)
    return codes


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64), (3, -1)])
def test_identity_hessian_reduces_to_rtn(bits, group):
    W, _, _ = tiny_layer(m=64, n=256, seed=2)
    res = sweep.quantize_factored(W, np.eye(256), bits, group, damp_rel=0.01, block=128)
    assert np.array_equal(res["codes"], _rtn_independent(W.astype(np.float64), bits, group))
    codes_rtn, _ = sweep.rtn(W, bits, group)
    assert np.array_equal(res["codes"], codes_rtn)


def test_sweep_loss_identity():
    W, X, G = tiny_layer(m=48, n=64, T=512, seed=3)
    HX, HG = factors.factor(X), factors.factor(G)
    Wt, HXt, HGt, _, _ = biip.biip_forward(W, HX, HG, 0, 0.25, "full")
    res = sweep.quantize_factored(Wt, HXt, 2, 32, block=16)
    dW = res["W_in"] - res["Q"]
    a = loss.sweep_loss_from_errors(res["E"], HGt)
    b = loss.kfac_loss(dW, res["A"], HGt)
    assert abs(a - b) <= 1e-10 * abs(b)
    # dW = E U column by column
    assert np.allclose(dW, res["E"] @ res["U"], rtol=0, atol=1e-12 * np.abs(dW).max())


def test_chol_upper_of_inverse():
    rng = np.random.default_rng(0)
    B = rng.normal(size=(30, 30))
    A = B @ B.T + 30 * np.eye(30)
    U = sweep.chol_upper_of_inverse(A)
    assert np.array_equal(U, np.triu(U))
    assert np.allclose(U.T @ U @ A, np.eye(30), atol=1e-10)
    assert np.all(np.diag(U) > 0)


def test_damping_and_dead_columns():
    H = np.diag([4.0, 0.0, 2.0])
    W = np.ones((2, 3))
    H1, W1, dead = sweep.dead_columns(H, W)
    assert dead.tolist() == [False, True, False]
    assert H1[1, 1] == 1.0 and np.all(W1[:, 1] == 0)
    A, lam = sweep.damp(H1, 0.01)
    assert lam == 0.01 * (4.0 + 1.0 + 2.0) / 3.0
    assert np.allclose(np.diag(A), [4 + lam, 1 + lam, 2 + lam])


def test_reverse_chol_failure_index():
    assert sweep.reverse_chol_failure(np.eye(5)) == 0
    A = np.eye(6)
    A[1, 1] = -1.0
    A[3, 3] = 0.0
    assert sweep.reverse_chol_failure(A) == 4     # trailing minor from index 3 fails first
    B = np.array([[1.0, 2.0], [2.0, 1.0]])        # indefinite, every diagonal positive
    assert sweep.reverse_chol_failure(B) == 1


@pytest.mark.parametrize("group", [128, 64, -1])
def test_lazy_batch_equals_unbatched(group):
    W, X, _ = tiny_layer(m=64, n=384, T=2048, seed=4)
    HX = factors.factor(X)
    r1 = sweep.quantize_factored(W, HX, 3, group, block=1)
    r128 = sweep.quantize_factored(W, HX, 3, group, block=128)
    same = r1["codes"] == r128["codes"]
    # exclude near ties: values within 1e-9 of a rounding boundary
    assert np.mean(same) > 0.9999
    assert np.allclose(r1["Q"][same], r128["Q"][same], rtol=0, atol=1e-9)


def test_f32_mirror_close_to_f64():
    W, X, _ = tiny_layer(m=64, n=256, T=2048, seed=6)
    HX = factors.factor(X)
    r = sweep.quantize_factored(W, HX, 4, 128, block=128)
    f = sweep.gptq_sweep_f32(r["W_in"].astype(np.float32), r["U"].astype(np.float32), 4, 128, True, 128)
    assert np.mean(f["codes"] != r["codes"]) < 0.005
    assert f["Q"].dtype == np.float32


# ------------------------------------------------------------------ Babai
def _babai_nearest_plane(B, t):
    """Textbook nearest plane (basis columns processed last to first)."""
    n = B.shape[1]
    Bs = np.zeros_like(B)
    for i in range(n):                         # Gram-Schmidt
        v = B[:, i].copy()
        for k in range(i):
            v -= (B[:, i] @ Bs[:, k]) / (Bs[:, k] @ Bs[:, k]) * Bs[:, k]
        Bs[:, i] = v
    c = np.zeros(n)
    r = t.copy()
    for i in range(n - 1, -1, -1):
        c[i] = np.rint((r @ Bs[:, i]) / (Bs[:, i] @ Bs[:, i]))
        r = r - c[i] * B[:, i]
    return c, Bs


def test_babai_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "babai_2x2.json")))
    L = np.array(g["L"])
    HX = L.T @ L
    assert np.array_equal(HX, np.array([[5.0, 3.0], [3.0, 9.0]]))
    U = sweep.chol_upper_of_inverse(HX)               # no damping
    assert np.allclose(U, np.linalg.inv(L).T, atol=1e-14)
    assert np.allclose(U, [[0.5, -1.0 / 6.0], [0.0, 1.0 / 3.0]], atol=1e-14)
    # optimal steps: alpha_j = det(L)^(1/2) / L_jj = sqrt(det) * U_jj
    det = float(np.prod(1.0 / np.diag(U)))
    alpha = math.sqrt(det) * np.diag(U)
    page = np.array(g["alpha_opt_num"]) / math.sqrt(g["alpha_opt_den_sqrt"])
    assert np.allclose(alpha, page, atol=1e-14)
    assert abs(np.prod(alpha) - 1.0) < 1e-14                 # volume preserved
    sides = alpha / np.diag(U)                               # alpha_j L_jj
    assert np.allclose(sides, math.sqrt(6.0), atol=1e-14)    # square cells
    rng = np.random.default_rng(0)
    w = rng.normal(size=(1000, 2))
    for steps in (np.array(g["alpha_rect"]), alpha):
        res = sweep.gptq_sweep(w, U, bits=0, group=-1, block=1, fixed_steps=steps)
        # The sweep decides column 0 first: basis order (b_2, b_1) for nearest plane.
        Bb = (L * steps[None, :])[:, ::-1]
        for r in range(w.shape[0]):
            c, Bs = _babai_nearest_plane(Bb, L @ w[r])
            assert np.array_equal(res["codes"][r, ::-1], c.astype(np.int64))
            err = L @ (w[r] - res["Q"][r])
            coef = np.array([(err @ Bs[:, i]) / (Bs[:, i] @ Bs[:, i]) for i in range(2)])
            assert np.all(np.abs(coef) <= 0.5 + 1e-12)       # error in the fundamental cell
    # with square cells the mean squared error is side^2 / 12 per dimension
    res = sweep.gptq_sweep(w, U, 0, -1, block=1, fixed_steps=alpha)
    mse = np.mean(np.sum(((w - res["Q"]) @ L.T) ** 2, axis=1))
    assert abs(mse - 2 * 6.0 / 12.0) < 0.1


# ------------------------------------------------------------------ brute force
def _tiny_instance(rng):
    W = rng.normal(size=(2, 3))
    X = rng.normal(size=(8, 3)) * np.exp(rng.normal(size=3))
    Gm = rng.normal(size=(8, 2)) * np.exp(rng.normal(size=2))
    return W, factors.factor(X), factors.factor(Gm)


def test_brute_force_tiny_layer():
    rng = np.random.default_rng(1)
    bits = 2
    W, HX, HG = _tiny_instance(rng)
    scale, zero = sweep.grid_params(W, bits, True)     # grid fixed at column 0 (g = -1)
    best = np.inf
    for cand in itertools.product(range(4), repeat=6):
        q = np.array(cand, dtype=np.float64).reshape(2, 3)
        deq = scale[:, None] * (q - zero[:, None])
        dW = W - deq
        a = loss.kfac_loss(dW, HX, HG)
        vec = dW.reshape(-1, order="F")                  # column-stacking vec
        b = vec @ np.kron(HX, HG) @ vec
        assert abs(a - b) <= 1e-12 * max(abs(b), 1e-300)
        best = min(best, a)
    res = sweep.quantize_factored(W, HX, bits, -1, block=1)
    sweep_loss = loss.kfac_loss(W - res["Q"], HX, HG)
    _, Qr = sweep.rtn(W, bits, -1)
    rtn_loss = loss.kfac_loss(W - Qr, HX, HG)
    assert best <= sweep_loss * (1 + 1e-12)
    assert best <= rtn_loss * (1 + 1e-12)


def test_sweep_beats_rtn_on_average():
    rng = np.random.default_rng(7)
    s_tot = r_tot = 0.0
    violations = 0
    for _ in range(1000):
        W, HX, HG = _tiny_instance(rng)
        res = sweep.quantize_factored(W, HX, 2, -1, block=1)
        ls = loss.kfac_loss(W - res["Q"], HX, HG)
        _, Qr = sweep.rtn(W, 2, -1)
        lr = loss.kfac_loss(W - Qr, HX, HG)
        s_tot += ls
        r_tot += lr
        violations += ls > lr * (1 + 1e-12)
    assert s_tot < r_tot
    assert violations < 500
    print(f"sweep > rtn on {violations}/1000 tiny instances; mean ratio {s_tot / r_tot:.3f}")


def test_sweep_beats_rtn_on_tiny_config():
    W, X, G = tiny_layer()
    HX, HG = factors.factor(X), factors.factor(G)
    res = sweep.quantize_factored(W, HX, 4, 128, block=128)
    _, Qr = sweep.rtn(W, 4, 128)
    assert loss.kfac_loss(W - res["Q"], HX, HG) < loss.kfac_loss(W - Qr, HX, HG)


def test_symmetric_grid():
    wg = np.array([[-3.0, 1.0, 2.0], [0.5, 0.25, 0.0], [0.0, 0.0, 0.0]])
    s, z = sweep.grid_params(wg, 4, asym=False)
    assert np.allclose(s, [6.0 / 15, 1.0 / 15, 2.0 / 15])
    assert np.all(z == 8)
    s, z = sweep.grid_params(wg, 2, asym=True)
    assert np.allclose(s, [5.0 / 3, 0.5 / 3, 2.0 / 3])
    assert np.array_equal(z, [np.rint(3.0 / (5.0 / 3)), 0.0, np.rint(1.0 / (2.0 / 3))])


def test_float32_factorisation_floor():
    # the float32 LAPACK route gives the same upper factor as the float64
    # definition to float32 accuracy on a well-conditioned matrix, and its
    # error grows with the condition number
    rng = np.random.default_rng(4)
    n = 96
    X = rng.standard_normal((4 * n, n))
    A, _ = sweep.damp(X.T @ X, 0.01)
    U = sweep.chol_upper_of_inverse(A)
    U32 = sweep.chol_upper_of_inverse_f32(A)
    assert U32.dtype == np.float32
    assert np.array_equal(U32, np.triu(U32))
    assert np.linalg.norm(U32 - U) / np.linalg.norm(U) < 1e-5
    assert np.abs(U32.astype(np.float64).T @ U32.astype(np.float64) @ A - np.eye(n)).max() < 1e-4
    # an ill-conditioned factor (a large common mean, as rectified inputs give)
    Xr = np.abs(X) + 3.0
    Ar, _ = sweep.damp(Xr.T @ Xr, 0.01)
    Ur = sweep.chol_upper_of_inverse(Ar)
    Ur32 = sweep.chol_upper_of_inverse_f32(Ar)
    e_good = np.linalg.norm(U32 - U) / np.linalg.norm(U)
    e_bad = np.linalg.norm(Ur32 - Ur) / np.linalg.norm(Ur)
    assert e_bad > 3 * e_good


@pytest.mark.parametrize("bits,group,block", [(2, 128, 1), (3, 16, 128), (4, 1, 16), (2, -1, 128),
                                              (3, 64, 64)])
def test_r_form_sweep_equals_u_form(bits, group, block):
    """gptq_sweep_rform(W, R) takes GPTQ's decisions: the same codes, grids and
    scaled errors as gptq_sweep(W, U) with U the Cholesky factor of the damped
    inverse (computed by its definition) and R the factor of the damped matrix
    (LAPACK on the index-reversed matrix), float64 both."""
    m, n = 24, 300
    W, X, _ = tiny_layer(m=m, n=n, T=3 * n, seed=bits * 100 + n)
    H = X.astype(np.float64).T @ X.astype(np.float64)
    A, _ = sweep.damp(H, 0.01)
    U = sweep.chol_upper_of_inverse(A)
    R = np.linalg.cholesky(A[::-1, ::-1])[::-1, ::-1]
    assert np.allclose(R @ R.T, A, rtol=1e-10, atol=1e-8 * np.abs(A).max())
    ru = sweep.gptq_sweep(W, U, bits, group, True, block=block)
    rr = sweep.gptq_sweep_rform(W, R, bits, group, True, block=block)
    assert np.array_equal(ru["codes"], rr["codes"])
    assert np.allclose(ru["scales"], rr["scales"], rtol=1e-12, atol=0)
    assert np.allclose(ru["Q"], rr["Q"], rtol=1e-12, atol=1e-15)
    assert np.allclose(ru["E"], rr["E"], rtol=1e-7, atol=1e-9)
    # the value of each column at its turn (gptq_sweep's final W holds it)
    assert np.allclose(ru["W_final"], rr["W_final"], rtol=1e-8, atol=1e-10)


def test_r_form_sweep_slips_are_caught():
    """Two plausible slips in the R form change codes: feeding the updated
    weight instead of the weight before the sweep into the feedback, and
    gridding a group from w + F / R_jj (the diagonal of U only) instead of
    W + F U_GG."""
    m, n, bits = 24, 384, 2
    W, X, _ = tiny_layer(m=m, n=n, T=3 * n, seed=3)
    A, _ = sweep.damp(X.astype(np.float64).T @ X.astype(np.float64), 0.01)
    R = np.linalg.cholesky(A[::-1, ::-1])[::-1, ::-1]
    U = sweep.chol_upper_of_inverse(A)
    ref = sweep.gptq_sweep(W, U, bits, 128, True)
    rd = np.diag(R)
    for slip in ("updated weight", "diagonal grid"):
        W0 = W.astype(np.float64)
        F = np.zeros_like(W0)
        codes = np.zeros((m, n), dtype=np.int64)
        for j in range(n):
            if j % 128 == 0:
                cur = W0[:, j:j + 128] + F[:, j:j + 128] / rd[j:j + 128]
                if slip == "updated weight":
                    cur = W0[:, j:j + 128] + F[:, j:j + 128] @ np.linalg.inv(np.triu(R[j:j + 128, j:j + 128]))
                scale, zero = sweep.grid_params(cur, bits, True)
            w = W0[:, j] + F[:, j] / rd[j]
            q, deq = sweep.quantize(w, scale, zero, bits)
            codes[:, j] = q
            d = (w - deq) if slip == "updated weight" else (W0[:, j] - deq)
            F[:, j + 1:] += np.outer(d, R[j, j + 1:])
        assert np.mean(codes != ref["codes"]) > 0.01, slip
