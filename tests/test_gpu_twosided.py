"""Two-sided rounding (kronq_quantize_two_sided) against the float64 oracle.

The oracle is GPTQ on vec(W) under U_X (x) U_G, element by element in row
order; the library runs 32 x 32 tiles along anti-diagonals with float32
arithmetic.  Checked: with the oracle's factors given (the sweep alone) and
with the library's own damping and factorisations, at sizes that span
several tiles in both directions with ragged edges, groups from 1 column to
the whole row, and 2 to 4 bits; at sizes the element-by-element oracle
cannot reach, the two identities that define the result: W~ - Q =
U_G^T E U_X, and every code the rounding of the value it was taken from."""
import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import sweep, twosided

pytestmark = pytest.mark.gpu


def _factors(m, n, seed, spread=0.0):
    rng = np.random.default_rng(seed)
    W = rng.normal(0.0, 0.02, size=(m, n))
    X = rng.standard_normal((3 * n, n)) * np.exp(spread * rng.standard_normal(n))
    G = rng.standard_normal((3 * m, m)) * np.exp(spread * rng.standard_normal(m))
    return W, X.T @ X, G.T @ G


def _run(W, HX, HG, bits, group, flags=0, asym=1, damp=0.01):
    m, n = W.shape
    dev = "cuda"
    p = kq.QuantParams(bits=bits, group=group, asym=asym, damp_rel=damp, block=128, flags=flags | kq.WRITE_E)
    ng = 1 if group == -1 else -(-n // group)
    Wt = torch.tensor(np.ascontiguousarray(W, dtype=np.float32), device=dev)
    HXt = torch.tensor(np.ascontiguousarray(HX, dtype=np.float32), device=dev)
    HGt = torch.tensor(np.ascontiguousarray(HG, dtype=np.float32), device=dev)
    codes = torch.zeros(m, n, dtype=torch.uint8, device=dev)
    scales = torch.zeros(m, ng, dtype=torch.float32, device=dev)
    zeros = torch.zeros(m, ng, dtype=torch.float32, device=dev)
    E = torch.zeros(m, n, dtype=torch.float32, device=dev)
    info = torch.full((2,), -7, dtype=torch.int32, device=dev)
    kq.kronq_quantize_two_sided(Wt, HXt, HGt, p, codes, scales, zeros, info, E=E)
    torch.cuda.synchronize()
    assert kq.kronq_device_status() == 0
    out = dict(codes=codes.cpu().numpy().astype(np.int64), Q=Wt.cpu().numpy().astype(np.float64),
               E=E.cpu().numpy().astype(np.float64), scales=scales.cpu().numpy().astype(np.float64),
               zeros=zeros.cpu().numpy().astype(np.float64), info=info.cpu().numpy(),
               UX=np.triu(HXt.cpu().numpy().astype(np.float64)), UG=np.triu(HGt.cpu().numpy().astype(np.float64)))
    return out


def _compare(got, ref, m, tol_codes=0.005):
    codes_ref = ref["codes"]
    dis = float(np.mean(got["codes"] != codes_ref))
    assert dis <= tol_codes, dis
    assert np.allclose(got["scales"], ref["scales"], rtol=1e-6, atol=0)
    assert np.array_equal(got["zeros"], ref["zeros"])
    # elements up to the first disagreement in the partial order see the
    # same history: take the rows whose codes all agree and compare there
    rows = np.all(got["codes"] == codes_ref, axis=1)
    first_bad = np.argmin(rows) if not rows.all() else m
    ok = slice(0, first_bad)   # every row above the first bad row has an identical history
    if first_bad > 0:
        assert np.abs(got["Q"][ok] - ref["Q"][ok]).max() <= 1e-6 * np.abs(ref["Q"]).max()
        # normwise, with a floor for float32 rounding of w~ - deq (with one
        # column per group every w~ starts on its own grid and E is pure
        # rounding noise)
        floor = 1e-5 * np.abs(ref["Q"]).max() / (np.diag(got["UG"]).min() * np.diag(got["UX"]).min())
        scale = np.abs(ref["E"][ok]).max()
        assert np.abs(got["E"][ok] - ref["E"][ok]).max() <= 1e-3 * scale + floor
    return first_bad


CASES = [(40, 200, 2, 128, 1), (70, 300, 3, 64, 1), (33, 129, 4, -1, 1), (65, 260, 2, 1, 1),
         (96, 300, 2, 32, 1), (64, 256, 4, 128, 0), (5, 7, 2, 4, 1)]


@pytest.mark.parametrize("m,n,bits,group,asym", CASES)
def test_two_sided_sweep_matches_oracle(m, n, bits, group, asym):
    """The sweep alone: the oracle's float64 factors passed in (KRONQ_U_GIVEN)."""
    W, HX, HG = _factors(m, n, seed=m * 1000 + n)
    AX, _ = sweep.damp(HX, 0.01)
    AG, _ = sweep.damp(HG, 0.01)
    UX = sweep.chol_upper_of_inverse(AX)
    UG = sweep.chol_upper_of_inverse(AG)
    ref = twosided.two_sided_sweep(W, UX, UG, bits, group, asym=bool(asym))
    got = _run(W, UX, UG, bits, group, flags=kq.U_GIVEN, asym=asym)
    assert list(got["info"]) == [0, 0]
    assert int(got["codes"].max()) <= 2 ** bits - 1
    first_bad = _compare(got, ref, m)
    assert first_bad >= min(m, 8)


@pytest.mark.parametrize("m,n,bits,group", [(96, 300, 2, 128), (130, 520, 3, 128), (64, 1000, 2, -1)])
def test_two_sided_full_path_matches_oracle(m, n, bits, group):
    """Damping and both factorisations on the GPU, then the sweep."""
    W, HX, HG = _factors(m, n, seed=7 + m + n, spread=0.5)
    ref = twosided.quantize_two_sided(W, HX, HG, bits, group, damp_rel=0.01)
    got = _run(W, HX, HG, bits, group)
    assert list(got["info"]) == [0, 0]
    for k in ("UX", "UG"):
        err = np.linalg.norm(got[k] - ref[k]) / np.linalg.norm(ref[k])
        assert err < 1e-4, (k, err)
    _compare(got, ref, m)


def _check_identities(W, got, bits, group):
    """W~ - Q = U_G^T E U_X (the feedback), and every code rounds the value
    it was taken from, w~ = deq + e U_G[i, i] U_X[j, j] (the decision)."""
    m, n = W.shape
    UX, UG, E, Q = got["UX"], got["UG"], got["E"], got["Q"]
    lhs = W - Q
    rhs = UG.T @ E @ UX
    assert np.abs(lhs - rhs).max() <= 2e-4 * np.abs(lhs).max(), np.abs(lhs - rhs).max()
    wt = Q + E * np.outer(np.diag(UG), np.diag(UX))
    g = np.zeros(n, dtype=np.int64) if group == -1 else np.arange(n) // group
    sc = got["scales"][:, g]
    zp = got["zeros"][:, g]
    q = got["codes"].astype(np.float64)
    assert np.allclose(Q, sc * (q - zp), rtol=0, atol=1e-6 * np.abs(Q).max())
    t = wt / sc + zp - q    # within half a step, or beyond it towards a clamped end
    maxq = 2 ** bits - 1
    slack = 1e-3
    inner = (q > 0) & (q < maxq)
    assert np.all(np.abs(t[inner]) <= 0.5 + slack)
    assert np.all(t[q == 0] <= 0.5 + slack)
    assert np.all(t[q == maxq] >= -0.5 - slack)
    ref_sc, ref_zp = twosided.static_grid(W, bits, group)
    assert np.allclose(got["scales"], ref_sc, rtol=1e-6, atol=0)


@pytest.mark.parametrize("m,n,bits,group", [(512, 1024, 2, 128), (300, 1000, 3, 64), (1024, 640, 4, -1)])
def test_two_sided_identities_at_size(m, n, bits, group):
    W, HX, HG = _factors(m, n, seed=m + 3 * n)
    got = _run(W, HX, HG, bits, group)
    assert list(got["info"]) == [0, 0]
    _check_identities(W, got, bits, group)


def test_two_sided_identity_output_factor_is_one_sided_static():
    """H_G = I: U_G = I / sqrt(1 + lambda), the rows decouple and each is a
    one-sided sweep with static grids (the oracle with U_G = I)."""
    m, n, bits = 64, 384, 2
    W, HX, _ = _factors(m, n, seed=3)
    AX, _ = sweep.damp(HX, 0.01)
    UX = sweep.chol_upper_of_inverse(AX)
    ref = twosided.two_sided_sweep(W, UX, np.eye(m), bits, 128)
    got = _run(W, UX, np.eye(m), bits, 128, flags=kq.U_GIVEN)
    _compare(got, ref, m)


def test_two_sided_reports_non_pd_output_factor():
    m, n = 40, 200
    W, HX, HG = _factors(m, n, seed=5)
    HG = -np.eye(m)
    got = _run(W, HX, HG, 2, 128, damp=0.0)
    assert got["info"][0] == 0 and got["info"][1] > 0


def test_two_sided_is_deterministic():
    m, n = 200, 700
    W, HX, HG = _factors(m, n, seed=11)
    a = _run(W, HX, HG, 2, 128)
    b = _run(W, HX, HG, 2, 128)
    for k in ("codes", "Q", "E", "scales"):
        assert np.array_equal(a[k], b[k]), k
