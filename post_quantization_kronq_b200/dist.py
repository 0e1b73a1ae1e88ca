"""Multi-process plumbing for quantizing many sublayers on several GPUs.

Sublayers are independent given their calibration data (KronQ quantizes
layer by layer), so ranks split the sublayers and share nothing on the data
path.  The one exchange is the inter-layer sensitivity: bit allocation
(KronQ README, "--inter_layer_mp") needs s = tr(H_G) tr(H_X) of every
sublayer, so the ranks all-gather the (tr H_X, tr H_G, s) triples that
``kronq_sensitivity`` returned for their sublayers -- a few KB -- and then
run the same deterministic host allocation on s.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

Sens = Tuple[float, float, float]


def shard_units(n_units: int, rank: int, world: int) -> List[int]:
    """Contiguous, balanced split of unit indices 0..n_units-1 over ranks."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return list(range(start, start + count))


def gather_sensitivities(local: Dict[int, Sens], n_units: int, group=None) -> List[Sens]:
    """All-gather {unit: (tr H_X, tr H_G, s)} from every rank (the triples
    of ``kronq_sensitivity``); returns the full list ordered by unit index.
    Works with the gloo and nccl backends."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    parts: List[Dict[int, Sens]] = [None] * world  # type: ignore[list-item]
    dist.all_gather_object(parts, dict(local), group=group)
    full: Dict[int, Sens] = {}
    for p in parts:
        full.update(p)
    missing = [u for u in range(n_units) if u not in full]
    if missing:
        raise RuntimeError(f"sensitivities missing for units {missing[:8]}")
    return [tuple(full[u]) for u in range(n_units)]


def allocate_from_sensitivities(sens: Sequence[Sens], sizes: Sequence[int], avg_bits: float = 2.5,
                                bmin: int = 2, bmax: int = 4) -> List[int]:
    """Bit widths from the library's s = tr(H_G) tr(H_X) (third entry of each
    triple) via the library's host allocator."""
    from . import kronq_allocate_bits

    return kronq_allocate_bits([t[2] for t in sens], sizes, avg_bits, bmin, bmax)
