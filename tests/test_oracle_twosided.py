"""Pins of oracle/twosided.py (two-sided adaptive rounding of the BaKron
abstract): the dense vectorised GPTQ, order independence over the partial
order, the one-sided reduction, the loss identity and the average gain."""
import numpy as np
import pytest

from oracle import sweep, twosided


def _layer(rng, m=3, n=4, T=80):
    X = rng.standard_normal((T, n)) * np.exp(0.5 * rng.standard_normal(n))
    G = rng.standard_normal((T, m)) @ rng.standard_normal((m, m))
    W = rng.standard_normal((m, n)) * 0.02
    return W, X.T @ X, G.T @ G


def _dense_vec_gptq(W, AX, AG, sc, zp, bits, group):
    """GPTQ element by element on vec(W) (columns stacked, index j m + i)
    with the Cholesky factor of the dense inverse of AX (x) AG."""
    m, n = W.shape
    H = np.kron(AX, AG)
    Ud = np.linalg.cholesky(np.linalg.inv(H)).T
    w = W.T.reshape(-1).copy()
    q_out = np.zeros(m * n, dtype=np.int64)
    d_out = np.zeros(m * n)
    for k in range(m * n):
        j, i = divmod(k, m)
        g = 0 if group == -1 else j // group
        q, deq = sweep.quantize(w[k:k + 1], sc[i:i + 1, g], zp[i:i + 1, g], bits)
        q_out[k], d_out[k] = int(q[0]), deq[0]
        e = (w[k] - deq[0]) / Ud[k, k]
        w[k + 1:] -= e * Ud[k, k + 1:]
    return q_out.reshape(n, m).T, d_out.reshape(n, m).T


@pytest.mark.parametrize("group", [2, -1])
def test_equals_dense_vectorised_gptq(group):
    rng = np.random.default_rng(1)
    W, HX, HG = _layer(rng)
    r = twosided.quantize_two_sided(W, HX, HG, 2, group)
    codes, Q = _dense_vec_gptq(W, r["AX"], r["AG"], r["scales"], r["zeros"], 2, group)
    assert np.array_equal(r["codes"], codes)
    assert np.allclose(r["Q"], Q, rtol=0, atol=1e-14)


def test_every_order_of_the_partial_order_agrees():
    rng = np.random.default_rng(2)
    W, HX, HG = _layer(rng, m=5, n=7)
    res = [twosided.quantize_two_sided(W, HX, HG, 3, 4, order=o) for o in ("row", "col", "anti")]
    for r in res[1:]:
        assert np.array_equal(r["codes"], res[0]["codes"])
        assert np.allclose(r["Q"], res[0]["Q"], rtol=0, atol=1e-13)
        assert np.allclose(r["E"], res[0]["E"], rtol=1e-11, atol=1e-13)


def test_identity_output_factor_is_the_one_sided_sweep():
    """H_G = I: rows are independent and the sweep is GPTQ's along each row
    (one group per row: the one-sided grid is taken from the initial row)."""
    rng = np.random.default_rng(3)
    W, HX, _ = _layer(rng, m=4, n=6)
    r = twosided.quantize_two_sided(W, HX, np.eye(4), 2, -1)
    A, _ = sweep.damp(HX, 0.01)
    one = sweep.gptq_sweep(W, sweep.chol_upper_of_inverse(A), 2, -1)
    assert np.array_equal(r["codes"], one["codes"])
    assert np.allclose(r["Q"], one["Q"], rtol=0, atol=1e-14)
    # scaled errors differ by U_G's diagonal only
    assert np.allclose(r["E"] * np.diag(r["UG"])[:, None], one["E"], rtol=1e-12, atol=1e-14)


def test_loss_identity():
    """sum E^2 = vec(dW)^T (A_X (x) A_G) vec(dW) = tr(dW A_X dW^T A_G)."""
    rng = np.random.default_rng(4)
    W, HX, HG = _layer(rng, m=4, n=5)
    r = twosided.quantize_two_sided(W, HX, HG, 2, -1)
    dW = W - r["Q"]
    loss = float(np.trace(dW @ r["AX"] @ dW.T @ r["AG"]))
    assert abs(float(np.sum(r["E"] ** 2)) - loss) <= 1e-10 * loss


def test_two_sided_lowers_the_loss_on_average():
    """With correlated output gradients, using H_G in the rounding lowers the
    K-FAC loss on average against the one-sided sweep (~25 % here)."""
    rng = np.random.default_rng(0)
    l2 = l1 = 0.0
    for _ in range(60):
        W, HX, HG = _layer(rng, m=6, n=8, T=200)
        r = twosided.quantize_two_sided(W, HX, HG, 2, -1)
        one = sweep.gptq_sweep(W, sweep.chol_upper_of_inverse(r["AX"]), 2, -1)
        for res, acc in ((r, "2"), (one, "1")):
            dW = W - res["Q"]
            v = float(np.trace(dW @ r["AX"] @ dW.T @ r["AG"]))
            if acc == "2":
                l2 += v
            else:
                l1 += v
    assert l2 < 0.9 * l1


@pytest.mark.parametrize("group", [2, 3, -1])
def test_identity_factors_give_round_to_nearest(group):
    """H_X = H_G = I: no error feedback, so the codes are round-to-nearest on
    the static grids (the independently written RTN of the sweep module)."""
    rng = np.random.default_rng(5)
    W = rng.standard_normal((4, 7)) * 0.02
    r = twosided.quantize_two_sided(W, np.eye(7), np.eye(4), 2, group)
    codes, Q = sweep.rtn(W, 2, group)
    assert np.array_equal(r["codes"], codes)
    assert np.allclose(r["Q"], Q, rtol=0, atol=1e-15)
