"""The quantize call returns the same bits when it is repeated on the same
inputs: the factor (U, or R in the R form), the codes and the dequantised
weights.  Shapes that run the per-block recursive inverse (U form at
n = 4096) and the two-level factorisation (R form at n = 28672, seven
4096-blocks), with the ill-conditioned factor of rectified inputs."""
import pytest
import torch

import post_quantization_kronq_b200 as kq
from post_quantization_kronq_b200.layer import LayerPass
from synth import llama_layer

pytestmark = pytest.mark.gpu


def _repeat(m, n, flags, runs, seed):
    dev = torch.device("cuda", 0)
    W, X, G = llama_layer(m, n, 16384, seed=seed, device=dev, w_std=0.015, rectified=True)
    lp = LayerPass(m, n, bits=2, group=128, seed=0, device=dev, flags=flags)
    lp.accumulate(X, G, chunk=16384)
    lp.transform(W)
    torch.cuda.synchronize()
    del X, G
    Wt0, H0 = lp.Wt.clone(), lp.HX.clone()
    ref = None
    differ = []
    for k in range(runs):
        lp.Wt.copy_(Wt0)
        lp.HX.copy_(H0)
        lp.quantize()
        torch.cuda.synchronize()
        assert int(lp.info.item()) == 0
        cur = (torch.triu(lp.HX).clone(), lp.codes.clone(), lp.Wt.clone())
        if ref is None:
            ref = cur
        elif not all(torch.equal(a, b) for a, b in zip(cur, ref)):
            differ.append(k)
    assert kq.kronq_device_status() == 0
    return differ


def test_u_form_n4096_repeats_exactly():
    assert _repeat(8, 4096, 0, runs=40, seed=7) == []


def test_r_form_n28672_repeats_exactly():
    assert _repeat(64, 28672, kq.R_FORM, runs=10, seed=1001) == []
