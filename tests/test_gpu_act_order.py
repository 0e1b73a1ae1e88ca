"""GPU act-order pass (the KronQ recipe's --act_order, read as GPTQ's
act-order heuristic) against the float64 oracle (oracle/options.py): the
sweep order and g_idx exactly, codes within 0.5 %, every column
dequantised through g_idx, the loss identity in the original order, and
bit for bit against the float32 mirror in the ordered mode."""
import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import biip, options, sweep
from synth import tiny_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _inputs(m, n, seed, dead=()):
    W, X, _ = tiny_layer(m=m, n=n, T=4 * n, seed=seed)
    X[:, list(dead)] = 0.0
    H = X.astype(np.float64).T @ X.astype(np.float64)
    if dead:   # unrotated, so the dead channels keep exact zero rows and columns
        return np.ascontiguousarray(W, np.float32), np.ascontiguousarray(H, np.float32)
    Wt, Ht, _, _, _ = biip.biip_forward(W, H, None, seed, 0.25, "sv_only")
    return np.ascontiguousarray(Wt, np.float32), np.ascontiguousarray(Ht, np.float32)


def _run(Wt, Ht, bits, group, flags=0):
    m, n = Wt.shape
    p = kq.QuantParams(bits=bits, group=group, asym=1, damp_rel=0.01, block=128, flags=flags)
    ng = 1 if group == -1 else -(-n // group)
    Wg, Hg = torch.from_numpy(Wt).to(DEV), torch.from_numpy(Ht).to(DEV)
    codes = torch.empty(m, n, dtype=torch.uint8, device=DEV)
    sc, zp = torch.empty(m, ng, device=DEV), torch.empty(m, ng, device=DEV)
    gi = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    perm = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    info = torch.ones(1, dtype=torch.int32, device=DEV)
    E = torch.empty(m, n, device=DEV) if flags & kq.WRITE_E else None
    kq.kronq_quantize_layer_act_order(Wg, Hg, p, codes, sc, zp, gi, info, E=E, perm=perm)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    return dict(Q=Wg, U=Hg, codes=codes.cpu().numpy().astype(np.int64), scales=sc.cpu().numpy(),
                zeros=zp.cpu().numpy(), g_idx=gi.cpu().numpy(), perm=perm.cpu().numpy(),
                E=None if E is None else E.cpu().numpy())


@pytest.mark.parametrize("m,n,bits,group,dead", [
    (96, 512, 3, 64, ()), (64, 640, 2, 128, ()), (48, 384, 4, -1, ()), (40, 256, 2, 32, (5, 77, 255)),
    (32, 4500, 2, 128, ()),            # above 4096: the blocked factorisation
])
def test_act_order_matches_oracle(m, n, bits, group, dead):
    Wt, Ht = _inputs(m, n, seed=m + n, dead=dead)
    ref = options.quantize_act_order(Wt, Ht, bits, group, True, 0.01, 128)
    got = _run(Wt, Ht, bits, group, flags=kq.WRITE_E)
    assert np.array_equal(got["perm"], ref["perm"])
    assert np.array_equal(got["g_idx"], ref["g_idx"])
    assert np.mean(got["codes"] != ref["codes"]) <= 0.005
    Q = got["Q"].cpu().numpy()
    gi = got["g_idx"]
    deq = got["scales"][:, gi] * (got["codes"].astype(np.float32) - got["zeros"][:, gi])
    assert np.array_equal(Q, deq.astype(np.float32))          # every column through g_idx
    # sum |e|^2 = tr(dW A dW^T) in the original order, A the damped factor
    dW = ref["W_in"] - Q.astype(np.float64)
    lhs = float(np.sum(got["E"].astype(np.float64) ** 2))
    rhs = float(np.trace(dW @ ref["A"] @ dW.T))
    assert abs(lhs - rhs) <= 2e-3 * rhs, (lhs, rhs)
    assert abs(lhs - float(np.sum(ref["E"] ** 2))) <= 0.01 * lhs


def test_act_order_ordered_mode_bit_exact():
    # with the float32 fixed-order sweep, the GPU pass equals the float32
    # mirror run on the permuted inputs with the GPU's own factor
    m, n, bits, group = 40, 384, 3, 64
    Wt, Ht = _inputs(m, n, seed=17)
    got = _run(Wt, Ht, bits, group, flags=kq.ORDERED_FP32 | kq.WRITE_E)
    perm = got["perm"]
    U = np.triu(got["U"].cpu().numpy())
    ref = sweep.gptq_sweep_f32(Wt[:, perm], U, bits, group, True, 128)
    inv = np.argsort(perm)
    assert np.array_equal(got["codes"], ref["codes"][:, inv])
    assert np.array_equal(got["Q"].cpu().numpy(), ref["Q"][:, inv])
    assert np.array_equal(got["E"], ref["E"][:, inv])
    assert np.array_equal(got["scales"], ref["scales"]) and np.array_equal(got["zeros"], ref["zeros"])
