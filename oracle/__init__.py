"""CPU oracle for KronQ's per-layer quantization pass.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 restatement
of what the pass computes, written from the KronQ pages (the KronQ README
mirrored on gitlite, the KronQ arXiv abstract on fugumt, the aissential.tech
and groundtruth.day summaries) and, for the worked Babai example and the
Kronecker factor definitions, the "WaterKron and FlipFlop Hessian" page.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
may import it.  It shares no code with the CUDA library and imports nothing
from it; the product path never calls it.

Modules
  factors  -- O1/O2: H_X = X^T X, H_G = G^T G, traces, sensitivity.
  biip     -- O3: bidirectional incoherence processing (rescale + rotation).
  sweep    -- O4/O5: grid, damping, Cholesky of the damped inverse, GPTQ
              column sweep (float64) and the float32 schedule-mirroring sweep.
  loss     -- O6: K-FAC layer loss tr(dW H_X dW^T H_G).
  alloc    -- O7: inter-layer bit allocation from tr(H_G) * tr(H_X).
  pack     -- int2/int4 code packing.
  pipeline -- the whole layer pass chained from the above.
  estimators -- Kronecker factor estimators (input, marginal, Frobenius,
              FlipFlop) of the "WaterKron and FlipFlop Hessian" page, Table 1.
  decode   -- the deploy path's dequant + BiIP matvec from packed codes.
  options  -- recipe options named without a definition (act-order).
  twosided -- two-sided adaptive rounding under H_X (x) H_G (BaKron abstract).

Every function is pinned by tests under ``tests/test_oracle_*.py`` against
closed forms, invariants, library special cases, brute force or the values
printed on the pages.  Parity is pinned for every function here.
"""
from . import factors, biip, sweep, loss, alloc, pack, pipeline, estimators, decode, options, twosided  # noqa: F401
