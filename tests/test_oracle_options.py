"""Pins of oracle/options.py (the act-order sweep order of the KronQ recipe)."""
import numpy as np
import pytest

from oracle import options, sweep


def _layer(rng, m=8, n=32, T=256):
    X = rng.standard_normal((T, n)) * np.exp(rng.standard_normal(n))
    X += 0.5 * X[:, [0]] * rng.standard_normal(n)
    W = rng.standard_normal((m, n)) * 0.02
    return W, X.T @ X


def test_order_is_decreasing_diagonal_with_stable_ties():
    H = np.diag([1.0, 3.0, 2.0, 3.0, 0.5])
    assert list(options.act_order_permutation(H)) == [1, 3, 2, 0, 4]


@pytest.mark.parametrize("group", [8, 16, -1])
def test_already_sorted_diagonal_is_the_plain_sweep(group):
    rng = np.random.default_rng(1)
    W, H = _layer(rng)
    order = np.argsort(-np.diag(H), kind="stable")
    W, H = W[:, order], H[np.ix_(order, order)]          # diagonal now non-increasing
    a = options.quantize_act_order(W, H, 3, group, True, 0.01, 1)
    p = sweep.quantize_factored(W, H, 3, group, True, 0.01, 1)
    assert np.array_equal(a["perm"], np.arange(W.shape[1]))
    for k in ("codes", "Q", "E", "scales", "zeros"):
        assert np.array_equal(a[k], p[k]), k


@pytest.mark.parametrize("group", [8, -1])
def test_group_index_dequantises_every_column(group):
    rng = np.random.default_rng(2)
    W, H = _layer(rng)
    a = options.quantize_act_order(W, H, 2, group, True, 0.01, 1)
    for j in range(W.shape[1]):
        g = a["g_idx"][j]
        assert np.allclose(a["Q"][:, j], a["scales"][:, g] * (a["codes"][:, j] - a["zeros"][:, g]),
                           rtol=0, atol=1e-15)


def test_loss_identity_in_original_coordinates():
    """sum_j |e_j|^2 = tr(dW (H + lambda I) dW^T) with dW, E and H all in the
    original column order: the un-permutation of Q and E is consistent."""
    rng = np.random.default_rng(3)
    W, H = _layer(rng)
    a = options.quantize_act_order(W, H, 2, 16, True, 0.01, 1)
    dW = a["W_in"] - a["Q"]
    lhs = float(np.sum(a["E"] ** 2))
    rhs = float(np.trace(dW @ a["A"] @ dW.T))
    assert abs(lhs - rhs) <= 1e-10 * rhs


def test_act_order_lowers_the_loss_on_average():
    """GPTQ's finding for act-order: over 200 layers with uneven input
    channels the damped quadratic loss is lower on average (here by ~10 %)."""
    rng = np.random.default_rng(0)
    la = lp = 0.0
    for _ in range(200):
        W, H = _layer(rng)
        a = options.quantize_act_order(W, H, 2, 16, True, 0.01, 1)
        p = sweep.quantize_factored(W, H, 2, 16, True, 0.01, 1)
        la += np.trace((a["W_in"] - a["Q"]) @ a["A"] @ (a["W_in"] - a["Q"]).T)
        lp += np.trace((p["W_in"] - p["Q"]) @ p["A"] @ (p["W_in"] - p["Q"]).T)
    assert la < 0.97 * lp


def test_errors_reproduce_the_weight_change():
    """dW = E U in the sweep order: W_in - Q equals E (taken in the sweep
    order) times the upper Cholesky factor of the damped, permuted inverse."""
    rng = np.random.default_rng(4)
    W, H = _layer(rng)
    a = options.quantize_act_order(W, H, 2, 8, True, 0.01, 1)
    p = a["perm"]
    inv = np.argsort(p)
    Ap = a["A"][np.ix_(p, p)]
    Up = np.linalg.cholesky(np.linalg.inv(Ap)).T
    dW = (a["E"][:, p] @ Up)[:, inv]
    assert np.allclose(dW, a["W_in"] - a["Q"], rtol=1e-9, atol=1e-12)
