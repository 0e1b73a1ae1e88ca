"""Pins of oracle/decode.py (the deploy path's dequant + BiIP matvec)."""
import numpy as np
import pytest

from oracle import biip, decode, pack, pipeline
from synth import tiny_layer


def test_dequantize_by_hand():
    # one row, codes 0 1 2 3 | 3 2, 2 bits, groups of 4: scales 0.5 and 2,
    # zeros 1 and 2 -> 0.5 (q - 1) for the first four, 2 (q - 2) for the rest
    words = pack.pack(np.array([[0, 1, 2, 3, 3, 2]]), 2)
    Q = decode.dequantize(words, [[0.5, 2.0]], [[1.0, 2.0]], 6, 2, 4)
    assert np.array_equal(Q, [[-0.5, 0.0, 0.5, 1.0, 2.0, 0.0]])
    # one group per row
    Q = decode.dequantize(words, [[0.25]], [[2.0]], 6, 2, -1)
    assert np.array_equal(Q, [[-0.5, -0.25, 0.0, 0.25, 0.25, 0.0]])


@pytest.mark.parametrize("mode", ["full", "no_rescale", "su_only", "sv_only"])
@pytest.mark.parametrize("m,n", [(8, 16), (12, 24)])
def test_matvec_equals_dense_rotations(mode, m, n):
    rng = np.random.default_rng(m * n)
    bits, group, seed = 4, 8, 3
    codes = rng.integers(0, 16, size=(m, n))
    words = pack.pack(codes, bits)
    ng = n // group
    sc = rng.uniform(0.01, 0.1, size=(m, ng))
    zp = rng.integers(0, 16, size=(m, ng)).astype(float)
    d_in = np.exp(rng.standard_normal(n) * 0.3)
    d_out = np.exp(rng.standard_normal(m) * 0.3)
    x = rng.standard_normal(n)
    y = decode.decode_matvec(words, sc, zp, bits, group, seed, mode, d_in, d_out, x)
    # the same product from dense rotation matrices and an explicit loop
    Q = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            Q[i, j] = sc[i, j // group] * (codes[i, j] - zp[i, j // group])
    V = biip.rotation_matrix(n, seed, 0) if mode != "su_only" else np.eye(n)
    U = biip.rotation_matrix(m, seed, 1) if mode != "sv_only" else np.eye(m)
    W_hat = np.diag(1.0 / d_out) @ U.T @ Q @ V @ np.diag(1.0 / d_in)
    assert np.allclose(y, W_hat @ x, rtol=1e-12, atol=1e-14)


def test_round_trip_through_the_pass():
    """Quantize a layer with the oracle pass, pack its codes, and decode: y
    equals the pass's own inverse-transformed dequantised weights times x."""
    W, X, G = tiny_layer()
    ref = pipeline.quantize_layer(X, G, W, bits=4, group=128, seed=0, block=128)
    words = pack.pack(ref["codes"], 4)
    m, n = W.shape
    rng = np.random.default_rng(0)
    x = rng.standard_normal(n)
    y = decode.decode_matvec(words, ref["scales"], ref["zeros"], 4, 128, 0, "full", ref["d_in"],
                             ref["d_out"], x)
    assert np.allclose(y, ref["What"] @ x, rtol=1e-10, atol=1e-12)
