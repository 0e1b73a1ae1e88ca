"""Bounded waits give up instead of hanging.

Every spin of the library (an mbarrier phase in the tensor-core kernels, a
cross-CTA step counter in the persistent factorisation) carries a wall-clock
bound after which it records KRONQ_ERR_TIMEOUT in the device status word and
returns.  Here a self-test kernel waits on a condition that nothing
satisfies, with a 2 ms bound, through the same wait functions: the status
must read TIMEOUT once (and be cleared by the read), the abort flag of the
counter wait must be raised, and the context must stay usable.
"""
import time

import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import factors

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = 5   # KRONQ_ERR_TIMEOUT


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up(which):
    assert kq.kronq_device_status() == 0
    w = torch.full((4,), -7, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    kq.kronq_wait_selftest(which, 2_000_000, w)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 2.0, elapsed            # gave up after ~2 ms, not the 4 s default
    got = w.cpu().tolist()
    assert got[2] == 1                       # the wait reported that it gave up
    assert got[0] == 0                       # nothing advanced the counter
    if which == 1:
        assert got[1] == 1                   # the counter wait raised the abort flag
    assert kq.kronq_device_status() == TIMEOUT
    assert kq.kronq_device_status() == 0     # the read cleared it
    # the context is still usable: a factor accumulation afterwards is right
    X = torch.randn(512, 256, device=DEV).bfloat16()
    H = torch.empty(256, 256, device=DEV)
    kq.kronq_accumulate_factors(X, H, zero_first=True)
    torch.cuda.synchronize()
    ref = factors.factor(X.float().cpu().numpy())
    Hn = H.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(Hn - ref) / np.linalg.norm(ref) < 1e-4
    assert kq.kronq_device_status() == 0
