"""Parity of kronq_kron_factors (Kronecker factor estimators of the
"WaterKron and FlipFlop Hessian" page, Table 1) with oracle/estimators.py
on the same bf16 tokens.

Tolerance: the weighted second moments are SYRKs of the tokens scaled by
sqrt(w_t) and rounded to bf16 (relative 2^-9 per element, so at most
2 * 2^-9 ~ 4e-3 per product before any averaging over tokens); the weights
come from a bf16 hi/lo split product (~2^-16).  4e-3 relative Frobenius
error per factor is that per-term bound, without the averaging."""
import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import estimators as est
from synth import llama_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 4e-3


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _oracle(name, Xn, Gn, iters):
    if name == "input":
        return est.input_factors(Xn, Gn)
    if name == "marginal":
        return est.marginal_factors(Xn, Gn)
    A, B, _ = (est.frobenius if name == "frobenius" else est.flipflop)(Xn, Gn, iters=iters)
    return A, B


CODES = {"input": kq.EST_INPUT, "marginal": kq.EST_MARGINAL, "frobenius": kq.EST_FROBENIUS,
         "flipflop": kq.EST_FLIPFLOP}


# (3000 tokens: one ragged chunk; 20000: two chunks.  n or m above 256 takes
# the persistent factorisation in the FlipFlop steps.)
@pytest.mark.parametrize("T,n,m", [(3000, 128, 192), (20000, 320, 256)])
@pytest.mark.parametrize("name", ["input", "marginal", "frobenius", "flipflop"])
def test_kron_factors_match_oracle(name, T, n, m):
    iters = 3
    _, X, G = llama_layer(m, n, T, seed=5, device=DEV)
    A = torch.empty(n, n, device=DEV)
    B = torch.empty(m, m, device=DEV)
    info = torch.ones(1, dtype=torch.int32, device=DEV)
    kq.kronq_kron_factors(X, G, CODES[name], iters, A, B, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    Xn = X.float().cpu().numpy().astype(np.float64)
    Gn = G.float().cpu().numpy().astype(np.float64)
    rA, rB = _oracle(name, Xn, Gn, iters)
    gA = A.cpu().numpy().astype(np.float64)
    gB = B.cpu().numpy().astype(np.float64)
    assert rel(gA, rA) < TOL, rel(gA, rA)
    assert rel(gB, rB) < TOL, rel(gB, rB)
    assert np.array_equal(gA, gA.T) and np.array_equal(gB, gB.T)
