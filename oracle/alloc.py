"""O7: inter-layer mixed precision from the trace sensitivity.

KronQ abstract, point (2), and README bullet "Inter-layer mixed precision":
per-sublayer bit allocation guided by s = tr(H_G) * tr(H_X).  README
"Mapping paper results to flags": ``--inter_layer_mp N`` upgrades the top-N
most sensitive sublayer types by +1 bit.

Budget reading (the pages give no rule for a fixed average): every sublayer
starts at ``bmin`` bits; repeatedly the sublayer with the largest expected
loss drop per stored bit, s_i (4^-b_i - 4^-(b_i+1)) / size_i, gets +1 bit,
among those whose upgrade keeps sum b_i size_i <= avg_bits * sum size_i and
b_i < bmax; ties go to the lower index.  The expected loss of a b-bit grid is
proportional to 4^-b tr(H_X) tr(H_G).  Scale/zero storage is not counted.
"""
from __future__ import annotations

import numpy as np


def expected_cost(s, bits) -> float:
    """sum_i s_i 4^-b_i -- the separable cost the allocation trades off."""
    return float(sum(float(si) * 4.0 ** (-int(b)) for si, b in zip(s, bits)))


def allocate_budget(s, sizes, avg_bits: float = 2.5, bmin: int = 2, bmax: int = 4):
    s = [float(v) for v in s]
    sizes = [int(v) for v in sizes]
    L = len(s)
    bits = [bmin] * L
    budget = avg_bits * sum(sizes)
    used = float(bmin * sum(sizes))
    while True:
        best, best_gain = -1, None
        for i in range(L):
            if bits[i] >= bmax or used + sizes[i] > budget:
                continue
            gain = s[i] * (4.0 ** (-bits[i]) - 4.0 ** (-(bits[i] + 1))) / sizes[i]
            if best_gain is None or gain > best_gain:
                best, best_gain = i, gain
        if best < 0:
            return bits
        bits[best] += 1
        used += sizes[best]


def allocate_topn_types(s, types, base_bits: int, N: int):
    """Type-level rule: the N types with the largest summed s get +1 bit."""
    names = []
    for t in types:
        if t not in names:
            names.append(t)
    tot = {t: 0.0 for t in names}
    for si, t in zip(s, types):
        tot[t] += float(si)
    order = sorted(range(len(names)), key=lambda k: (-tot[names[k]], k))
    top = {names[k] for k in order[:N]}
    return [base_bits + (1 if t in top else 0) for t in types]
