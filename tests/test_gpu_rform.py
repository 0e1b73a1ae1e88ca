"""The sweep on the factor R itself (KRONQ_R_FORM) against the oracle.

The oracle follows the pages: U, the upper Cholesky factor of the damped
inverse of H~_X, and GPTQ's column sweep with the feedback -e_k U_kj.  The
library's R form reaches the same updates from R (H~_X + lambda I = R R^T,
U = R^-1) without inverting it: w~_j = w_j + sum_{k<j} (w_k - q_k) R_kj / R_jj.
Checked here: R against the float64 factor (held to a multiple of what a
float32 LAPACK factorisation of the same matrix achieves), codes, scales and
the scaled errors against the oracle's float64 sweep, at sizes that run the
per-step factorisation, the persistent one and the two-level blocked one, with
dead columns and with groups from 1 to 128 columns."""
import numpy as np
import pytest
import scipy.linalg as sl
import torch

import post_quantization_kronq_b200 as kq
from oracle import sweep
from post_quantization_kronq_b200.layer import LayerPass
from synth import tiny_layer

pytestmark = pytest.mark.gpu


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def to_np(t):
    return t.detach().float().cpu().numpy()


def reverse_chol(A, dtype):
    """R upper with A = R R^T (LAPACK on the index-reversed matrix)."""
    L = sl.cholesky(np.ascontiguousarray(np.asarray(A, dtype)[::-1, ::-1]), lower=True, check_finite=False)
    return np.ascontiguousarray(L[::-1, ::-1]).astype(np.float64)


def _run(W, H, bits, group, flags, E=False):
    m, n = W.shape
    f = flags | (kq.WRITE_E if E else 0)
    lp = LayerPass(m, n, bits=bits, group=group, flags=f)
    lp.HX.copy_(torch.from_numpy(H))
    lp.Wt.copy_(torch.from_numpy(W))
    Et = torch.zeros(m, n, dtype=torch.float32, device="cuda") if E else None
    kq.kronq_quantize_layer(lp.Wt, lp.HX, lp.params, lp.codes, lp.scales, lp.zeros, lp.info,
                            E=Et, ws=lp.ws_quant)
    torch.cuda.synchronize()
    assert int(lp.info.item()) == 0
    assert kq.kronq_device_status() == 0
    return lp, (to_np(Et) if E else None)


CASES = [(64, 200, 2, 128, ()), (96, 640, 3, 64, ()), (64, 1000, 4, 128, (3, 517)),
         (48, 2304, 2, 32, ()), (40, 4500, 2, 128, (4100,)), (32, 8192, 2, 128, ())]


@pytest.mark.parametrize("m,n,bits,group,dead", CASES)
def test_r_form_matches_oracle(m, n, bits, group, dead):
    W, X, _ = tiny_layer(m=m, n=n, T=3 * n, seed=n + bits)
    if dead:
        X[:, list(dead)] = 0.0
    H = (X.astype(np.float64).T @ X.astype(np.float64)).astype(np.float32)
    ref = sweep.quantize_factored(W, H, bits, group, True, 0.01, block=128)
    assert np.array_equal(np.nonzero(ref["dead"])[0], list(dead))
    lp, E = _run(W, H, bits, group, kq.R_FORM, E=True)
    # the factor: R of the damped matrix after the dead-column rule
    H1, _, _ = sweep.dead_columns(H, W)
    A, _ = sweep.damp(H1, 0.01)
    R64 = reverse_chol(A, np.float64)
    floor = rel(reverse_chol(A, np.float32), R64)
    errR = rel(np.triu(to_np(lp.HX)), R64)
    assert errR < max(1e-5, 4 * floor), (errR, floor)
    # the sweep: codes, grids and scaled errors
    codes = lp.codes.cpu().numpy().astype(np.int64)
    dis = float(np.mean(codes != ref["codes"]))
    assert dis <= 0.005, dis
    assert int(codes.max()) <= 2 ** bits - 1
    assert rel(to_np(lp.scales), ref["scales"]) < 1e-3
    # rows whose codes all agree with the oracle: the same dequantised
    # weights and the same scaled errors (a flipped code moves a row's later
    # errors, so those rows are left out)
    rows = np.all(codes == ref["codes"], axis=1)
    assert rows.sum() >= m // 4
    Q = to_np(lp.Wt)
    assert rel(Q[rows], ref["Q"][rows]) < 1e-5
    assert rel(E[rows], ref["E"][rows]) < 1e-3
    if dead:
        assert np.allclose(Q[:, list(dead)], ref["Q"][:, list(dead)], rtol=0, atol=1e-6)


@pytest.mark.parametrize("group", [1, 4, 16, 128, -1])
def test_r_form_equals_u_form(group):
    """Both forms on the same input: the same updates, so the same codes up to
    float32 rounding at a few grid boundaries."""
    m, n, bits = 128, 768, 3
    W, X, _ = tiny_layer(m=m, n=n, T=3 * n, seed=77)
    H = (X.astype(np.float64).T @ X.astype(np.float64)).astype(np.float32)
    lr, Er = _run(W, H, bits, group, kq.R_FORM, E=True)
    lu, Eu = _run(W, H, bits, group, 0, E=True)
    cr = lr.codes.cpu().numpy()
    cu = lu.codes.cpu().numpy()
    assert np.mean(cr != cu) <= 0.002
    # R and U from the same factorisation: R U = I
    R = np.triu(to_np(lr.HX)).astype(np.float64)
    U = np.triu(to_np(lu.HX)).astype(np.float64)
    assert np.abs(R @ U - np.eye(n)).max() < 1e-4
    rows = np.all(cr == cu, axis=1)
    assert rows.sum() >= m // 2
    # normwise: the two forms round differently (~1e-6 of |E| max); with one
    # column per group every value sits on its own grid and E is rounding
    # noise of ~1e-9, hence the absolute floor
    assert np.abs(Er[rows] - Eu[rows]).max() <= 1e-4 * np.abs(Eu[rows]).max() + 1e-6


def test_r_form_ill_conditioned_factor():
    """A factor with condition number ~1e6 (column scales over three decades):
    the R form's codes stay within the tolerance of the float64 sweep."""
    m, n, bits = 64, 1536, 2
    rng = np.random.default_rng(5)
    X = rng.standard_normal((2 * n, n)) * np.exp(1.2 * rng.standard_normal(n))
    H = (X.T @ X).astype(np.float32)
    W = rng.normal(0.0, 0.02, size=(m, n)).astype(np.float32)
    ref = sweep.quantize_factored(W, H, bits, 128, True, 0.01, block=128)
    lp, _ = _run(W, H, bits, 128, kq.R_FORM)
    dis = float(np.mean(lp.codes.cpu().numpy() != ref["codes"]))
    assert dis <= 0.005, dis


def test_r_factor_precision_by_region():
    """R of a well-conditioned n = 8192 factor (two 4096 blocks of the
    two-level factorisation) against float64, region by region, next to a
    float32 LAPACK factorisation of the same matrix."""
    n, h = 8192, 4096
    rng = np.random.default_rng(12)
    X = rng.standard_normal((16384, n)) * np.exp(0.5 * rng.standard_normal(n))
    A, _ = sweep.damp(X.T @ X, 0.01)
    del X
    R = reverse_chol(A, np.float64)
    floor = rel(reverse_chol(A, np.float32), R)
    lp = LayerPass(8, n, bits=2, group=128, damp_rel=0.0, flags=kq.R_FORM)   # A is damped already
    lp.HX.copy_(torch.from_numpy(A.astype(np.float32)))
    lp.Wt.zero_()
    lp.quantize()
    torch.cuda.synchronize()
    assert int(lp.info.item()) == 0
    Rg = np.triu(to_np(lp.HX))
    errs = {"total": rel(Rg, R), "trailing block": rel(Rg[h:, h:], R[h:, h:]),
            "leading block": rel(Rg[:h, :h], R[:h, :h]), "off-diagonal": rel(Rg[:h, h:], R[:h, h:])}
    print("R relative error", {k: f"{v:.2e}" for k, v in errs.items()}, f"float32 LAPACK {floor:.2e}")
    for k, v in errs.items():
        assert v < 10 * floor + 1e-6, (k, v, floor)
