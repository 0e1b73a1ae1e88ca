"""Parity of kronq_decode_matvec (the deploy path's dequant + BiIP matvec
from packed codes) with oracle/decode.py on the same words, scales, zeros,
scale vectors and activations.

Tolerance: every step is float32 (the two row transforms and the matvec's
sums of up to n = 4096 products); random rounding gives a norm-relative error
near sqrt(n) 2^-24 ~ 4e-6, so 1e-4 leaves a wide margin."""
import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import decode, pack

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-4


@pytest.mark.parametrize("m,n,bits,group,mode,xdt", [
    (64, 96, 4, 32, "full", torch.float32),      # n = 32 x 3: DCT factor 3
    (40, 256, 2, 128, "no_rescale", torch.bfloat16),
    (48, 200, 2, 8, "su_only", torch.float32),   # groups smaller than a word, ragged row
    (33, 128, 4, -1, "sv_only", torch.float32),
    (4096, 4096, 2, 128, "full", torch.bfloat16),   # q_proj W2 g128
    (4096, 4096, 4, 128, "full", torch.bfloat16),
])
def test_decode_matvec_matches_oracle(m, n, bits, group, mode, xdt):
    rng = np.random.default_rng(m + n + bits)
    codes = rng.integers(0, 2 ** bits, size=(m, n))
    words = pack.pack(codes, bits)
    ng = 1 if group == -1 else -(-n // group)
    sc = rng.uniform(0.005, 0.05, size=(m, ng)).astype(np.float32)
    zp = rng.integers(0, 2 ** bits, size=(m, ng)).astype(np.float32)
    d_in = np.exp(0.3 * rng.standard_normal(n)).astype(np.float32)
    d_out = np.exp(0.3 * rng.standard_normal(m)).astype(np.float32)
    x = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).to(xdt)
    seed = 7
    ref = decode.decode_matvec(words, sc, zp, bits, group, seed, mode, d_in, d_out,
                               x.float().numpy().astype(np.float64))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
    y = torch.empty(m, device=DEV)
    kq.kronq_decode_matvec(dev(words.view(np.int32)), dev(sc), dev(zp), n, bits, group, seed, mode,
                           dev(d_in), dev(d_out), x.to(DEV), y)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < TOL, err
