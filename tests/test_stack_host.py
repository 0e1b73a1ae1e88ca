"""Host logic of the mixed-precision stack (no GPU): the allocation from the
first pass's sensitivities and the built-in trace check."""
import pytest

from oracle import alloc
from post_quantization_kronq_b200.stack import StackPass


def _stack():
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
              (4096, 14336)]
    return StackPass(shapes, avg_bits=2.5, device="cpu"), shapes


def test_allocation_uses_the_library_rule():
    sp, shapes = _stack()
    sp.sens1 = [(1.0 + i, 2.0 + 3 * i, (1.0 + i) * (2.0 + 3 * i)) for i in range(len(shapes))]
    bits = sp.allocate()
    assert bits == list(alloc.allocate_budget([t[2] for t in sp.sens1], [m * n for m, n in shapes]))


def test_trace_check_flags_a_mismatch():
    sp, shapes = _stack()
    sp.sens1 = [(100.0, 50.0, 5000.0)] * len(shapes)
    sp.check_traces(0, (100.05, 50.0, 5002.5))          # within 1e-3
    assert sp.sens2[0][0] == 100.05
    with pytest.raises(RuntimeError):
        sp.check_traces(1, (100.2, 50.0, 5010.0))       # 2e-3 off in tr(H_X)
    with pytest.raises(RuntimeError):
        sp.check_traces(2, (100.0, 49.9, 4990.0))       # 2e-3 off in tr(H_G)
