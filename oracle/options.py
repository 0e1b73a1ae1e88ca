"""Recipe options of the KronQ README named without a definition (float64).

TEST INFRASTRUCTURE ONLY (see the package header).

KronQ README, "Reproduce from scratch": the recipe passes ``--act_order``
(among ``--w_clip``, ``--use_gptaq`` and others) to the GPTQ-style sweep.  The
pages do not define it; the reading taken is GPTQ's published act-order
heuristic:

* After the dead-column rule, the columns are swept in order of decreasing
  diagonal of H~_X (a stable sort: ties keep the column order).  The sweep,
  its groups and its scales run in that order (dynamic groups of consecutive
  permuted columns); damping is unchanged (the mean diagonal does not depend
  on the order).
* Codes, Q and E come back in the original column order; column j belongs to
  group g_idx[j] = (rank of j in the sweep order) // group (0 when group is
  -1), and scales and zeros are indexed by that group.

Pinned in tests/test_oracle_options.py.
"""
from __future__ import annotations

import numpy as np

from . import sweep


def act_order_permutation(H) -> np.ndarray:
    """Sweep order: column indices by decreasing diagonal, ties by index."""
    d = np.diag(np.asarray(H, dtype=np.float64))
    return np.argsort(-d, kind="stable")


def quantize_act_order(Wt, Ht, bits: int, group: int, asym: bool = True, damp_rel: float = 0.01,
                       block: int = 1):
    """quantize_factored with the act-order sweep order.

    Returns dict(codes, Q, E (original column order), scales, zeros (per
    sweep-order group), g_idx, perm, A (damped H~_X, original order)).
    """
    H1, W1, dead = sweep.dead_columns(Ht, Wt)
    perm = act_order_permutation(H1)
    Hp = H1[np.ix_(perm, perm)]
    Ap, lam = sweep.damp(Hp, damp_rel)
    U = sweep.chol_upper_of_inverse(Ap)
    res = sweep.gptq_sweep(W1[:, perm], U, bits, group, asym, block)
    inv = np.argsort(perm)
    n = W1.shape[1]
    g_idx = np.zeros(n, dtype=np.int64) if group == -1 else inv // group
    A, _ = sweep.damp(H1, damp_rel)
    return dict(codes=res["codes"][:, inv], Q=res["Q"][:, inv], E=res["E"][:, inv],
                scales=res["scales"], zeros=res["zeros"], g_idx=g_idx, perm=perm, A=A,
                W_in=W1, dead=dead, lam=lam)
