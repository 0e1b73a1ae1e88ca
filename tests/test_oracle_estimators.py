"""Pins of oracle/estimators.py (Kronecker factor estimators of the
"WaterKron and FlipFlop Hessian" page, Table 1), independent of its update
formulas: the dense Kronecker definition, the nearest Kronecker product from
an SVD of the Van Loan rearrangement, exactly Kronecker-structured samples,
monotone targets, block optimality under perturbation, and the first sweep
from the identity as partial traces of the dense H (which also fixes how the
scale is split between A and B)."""
import numpy as np
import pytest

from oracle import estimators as est
from oracle import factors


def _tokens(T, n, m, seed):
    rng = np.random.default_rng(seed)
    # correlated, heavy-ish inputs and gradients that depend on the inputs,
    # so H is not a Kronecker product
    X = rng.standard_normal((T, n)) @ rng.standard_normal((n, n)) * np.exp(rng.standard_normal(n))
    G = rng.standard_normal((T, m)) * (1.0 + 0.5 * np.abs(X[:, :1]))
    return X, G


def _product_sample(p, q, n, m, seed):
    """Every pair (x_i, g_j): E[x x^T (x) g g^T] = E[x x^T] (x) E[g g^T] exactly."""
    rng = np.random.default_rng(seed)
    xs = rng.standard_normal((p, n)) @ rng.standard_normal((n, n))
    gs = rng.standard_normal((q, m)) @ rng.standard_normal((m, m))
    X = np.repeat(xs, q, axis=0)
    G = np.tile(gs, (p, 1))
    return X, G, xs.T @ xs / p, gs.T @ gs / q


def test_kron_hessian_one_token_by_hand():
    # x = (1, 2), g = (3, -1): H = x x^T (x) g g^T written out entry by entry
    H = est.kron_hessian(np.array([[1.0, 2.0]]), np.array([[3.0, -1.0]]))
    xx = [[1, 2], [2, 4]]
    gg = [[9, -3], [-3, 1]]
    want = np.array([[xx[i][j] * gg[k][l] for j in range(2) for l in range(2)]
                     for i in range(2) for k in range(2)], dtype=float)
    assert np.array_equal(H, want)


def test_objectives_equal_dense_forms():
    X, G = _tokens(40, 3, 2, 1)
    H = est.kron_hessian(X, G)
    rng = np.random.default_rng(2)
    for _ in range(5):
        Ma, Mb = rng.standard_normal((3, 3)), rng.standard_normal((2, 2))
        A, B = Ma @ Ma.T + np.eye(3), Mb @ Mb.T + np.eye(2)
        K = np.kron(A, B)
        frob = np.sum((H - K) ** 2)
        assert abs(est.frob_objective(X, G, A, B) - frob) <= 1e-10 * frob
        dense = np.trace(np.linalg.solve(K, H)) + np.linalg.slogdet(K)[1]
        assert abs(est.flipflop_objective(X, G, A, B) - dense) <= 1e-10 * abs(dense)


def test_input_and_marginal_rows():
    X, G = _tokens(50, 4, 3, 3)
    A, B = est.input_factors(X, G)
    assert np.allclose(A, factors.factor(X) / 50, rtol=1e-13) and np.array_equal(B, np.eye(3))
    A, B = est.marginal_factors(X, G)
    assert np.allclose(B, factors.factor(G) / 50, rtol=1e-13)


@pytest.mark.parametrize("fn", [est.frobenius, est.flipflop])
def test_exact_kronecker_sample_is_recovered(fn):
    X, G, Sx, Sg = _product_sample(5, 4, 3, 2, 4)
    A, B, _ = fn(X, G, iters=3)
    K, want = np.kron(A, B), np.kron(Sx, Sg)
    assert np.linalg.norm(K - want) <= 1e-11 * np.linalg.norm(want)
    A, B = est.marginal_factors(X, G)
    assert np.linalg.norm(np.kron(A, B) - want) <= 1e-11 * np.linalg.norm(want)


def test_frobenius_is_the_nearest_kronecker_product():
    n, m = 3, 2
    X, G = _tokens(60, n, m, 5)
    H = est.kron_hessian(X, G)
    # Van Loan rearrangement: R[(i, j), (k, l)] = H[i m + k, j m + l]
    R = H.reshape(n, m, n, m).transpose(0, 2, 1, 3).reshape(n * n, m * m)
    U, s, Vt = np.linalg.svd(R)
    best = np.kron(s[0] * U[:, 0].reshape(n, n), Vt[0].reshape(m, m))
    A, B, hist = est.frobenius(X, G, iters=300)
    assert np.linalg.norm(np.kron(A, B) - best) <= 1e-9 * np.linalg.norm(best)
    assert abs(hist[-1] - np.sum((H - best) ** 2)) <= 1e-9 * np.sum(H * H)


def test_targets_never_increase():
    X, G = _tokens(80, 4, 3, 6)
    _, _, hf = est.frobenius(X, G, iters=25)
    _, _, hp = est.flipflop(X, G, iters=25)
    for h in (hf, hp):
        scale = max(abs(v) for v in h)
        assert all(b <= a + 1e-12 * scale for a, b in zip(h, h[1:]))


def test_flipflop_block_optimality_and_scale():
    n, m = 4, 3
    X, G = _tokens(120, n, m, 7)
    A, B, _ = est.flipflop(X, G, iters=200)
    f0 = est.flipflop_objective(X, G, A, B)
    # stationarity of F in the scale of either factor: E[q] = n m
    q = est.quad_forms(X, np.linalg.inv(A)) * est.quad_forms(G, np.linalg.inv(B))
    assert abs(np.mean(q) - n * m) <= 1e-9 * n * m
    rng = np.random.default_rng(8)
    for c in (0.9, 1.1):
        assert est.flipflop_objective(X, G, c * A, B) > f0
        assert est.flipflop_objective(X, G, A, c * B) > f0
    for _ in range(10):
        Sa = rng.standard_normal((n, n))
        Sb = rng.standard_normal((m, m))
        eps = 1e-3
        assert est.flipflop_objective(X, G, A + eps * (Sa + Sa.T) * np.linalg.norm(A), B) > f0
        assert est.flipflop_objective(X, G, A, B + eps * (Sb + Sb.T) * np.linalg.norm(B)) > f0
    # the Kronecker scale ambiguity leaves F unchanged
    assert abs(est.flipflop_objective(X, G, 2.0 * A, B / 2.0) - f0) <= 1e-12 * abs(f0)


def test_frobenius_block_optimality():
    n, m = 4, 3
    X, G = _tokens(100, n, m, 9)
    A, B, _ = est.frobenius(X, G, iters=100)
    f0 = est.frob_objective(X, G, A, B)
    rng = np.random.default_rng(10)
    for _ in range(10):
        Sa, Sb = rng.standard_normal((n, n)), rng.standard_normal((m, m))
        assert est.frob_objective(X, G, A + 1e-3 * Sa * np.linalg.norm(A), B) >= f0
        assert est.frob_objective(X, G, A, B + 1e-3 * Sb * np.linalg.norm(B)) >= f0


def test_one_sweep_from_identity_by_partial_traces():
    """The first sweep's factors are the block minimisers, written from the
    dense H: with B = I, both targets give A = tr_B(H) / m (the partial trace
    over the output index); then Frobenius gives B = sum_ij A_ij H_(i.),(j.) /
    ||A||_F^2 and FlipFlop B = sum_ij (A^-1)_ji H_(i.),(j.) / n, where H_(i.),(j.)
    is the m x m block of H at input indices (i, j)."""
    n, m = 3, 4
    X, G = _tokens(30, n, m, 11)
    Hb = est.kron_hessian(X, G).reshape(n, m, n, m)      # Hb[i, k, j, l] = H[i m + k, j m + l]
    A1 = np.einsum("ikjk->ij", Hb) / m
    blocks = Hb.transpose(0, 2, 1, 3)                     # blocks[i, j] = H_(i.),(j.)
    Bf = np.einsum("ij,ijkl->kl", A1, blocks) / np.sum(A1 * A1)
    Bp = np.einsum("ji,ijkl->kl", np.linalg.inv(A1), blocks) / n
    A, B, _ = est.frobenius(X, G, iters=1)
    assert np.allclose(A, A1, rtol=1e-12, atol=0) and np.allclose(B, Bf, rtol=1e-11, atol=0)
    A, B, _ = est.flipflop(X, G, iters=1)
    assert np.allclose(A, A1, rtol=1e-12, atol=0) and np.allclose(B, Bp, rtol=1e-11, atol=0)
