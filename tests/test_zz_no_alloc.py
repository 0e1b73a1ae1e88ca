"""kronq_quantize_layer_static -- the quantize call for callers that cannot
allocate device memory (plugins that only receive pointers from a host
runtime's pool, foreign-language callers without a CUDA allocator, paths
where cudaMalloc's device synchronisation is not allowed).  Its scratch is
the library's static device array instead of a caller workspace.

Checked through the C ABI against kronq_quantize_layer (same inputs, fresh
workspace) on two calls in a row, the second one finding the first one's
leftovers in the shared static scratch.  Both run the same deterministic
kernels, so the outputs must agree exactly (tighter than the 0.5 % / 1e-5
bars the other parity tests use).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from post_quantization_kronq_b200 import _lib

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(m, n, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    X = torch.randn(3 * n, n, generator=g, dtype=torch.float64) * torch.exp(
        torch.randn(n, generator=g, dtype=torch.float64))
    H = (X.T @ X).float().to(DEV)
    W = (torch.randn(m, n, generator=g) * 0.02).to(DEV)
    return W, H


def _outputs(m, n, p):
    ng = 1 if p.group == -1 else -(-n // p.group)
    return (torch.empty(m, n, dtype=torch.uint8, device=DEV), torch.empty(m, ng, device=DEV),
            torch.empty(m, ng, device=DEV), torch.full((1,), 7, dtype=torch.int32, device=DEV))


def _run(static, W, H, p):
    m, n = W.shape
    Wt, HX = W.clone(), H.clone()
    codes, sc, zp, info = _outputs(m, n, p)
    if static:
        kq.kronq_quantize_layer_static(Wt, HX, p, codes, sc, zp, info)
    else:
        kq.kronq_quantize_layer(Wt, HX, p, codes, sc, zp, info)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in
            dict(Wt=Wt, U=torch.triu(HX), codes=codes, scales=sc, zeros=zp, info=info).items()}


@pytest.mark.parametrize("cases", [[(512, 1024, 4, 128, 1), (300, 640, 2, 64, 2)],
                                   [(4096, 4096, 2, 128, 3), (4096, 4096, 2, 128, 3)]])
def test_static_scratch_matches_workspace_call_twice(cases):
    for (m, n, bits, group, seed) in cases:        # two calls in a row
        W, H = _case(m, n, seed)
        p = kq.QuantParams(bits=bits, group=group, asym=1, damp_rel=0.01, block=128, flags=0)
        want = _run(False, W, H, p)
        got = _run(True, W, H, p)
        assert int(got["info"][0]) == 0 and int(want["info"][0]) == 0
        for k in ("codes", "scales", "zeros", "Wt", "U"):
            assert np.array_equal(got[k], want[k]), k


def test_static_scratch_rejects_layers_beyond_its_size():
    p = kq.QuantParams(bits=2, group=128, asym=1, damp_rel=0.01, block=128, flags=0)
    assert kq.kronq_quantize_workspace_bytes(1024, 8192, p) > 64 << 20
    fake = ctypes.c_void_p(4096)   # never dereferenced: the size check comes first
    st = _lib.lib.kronq_quantize_layer_static(fake, fake, 1024, 8192, ctypes.byref(p), fake, fake,
                                              fake, None, fake, None)
    assert st == _lib.ERR_INVALID_ARG
    assert b"64 MiB" in _lib.lib.kronq_last_error()
