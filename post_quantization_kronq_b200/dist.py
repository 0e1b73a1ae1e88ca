"""Multi-process plumbing for quantizing many sublayers on several GPUs.

Sublayers are independent given their calibration data (KronQ quantizes
layer by layer), so ranks split the sublayers and share nothing on the data
path.  The one exchange is the inter-layer sensitivity: bit allocation
(KronQ README, "--inter_layer_mp") needs tr(H_G) tr(H_X) of every sublayer,
so the ranks all-gather their (index, trace X, trace G) triples -- a few KB --
and then run the same deterministic host allocation.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple


def shard_units(n_units: int, rank: int, world: int) -> List[int]:
    """Contiguous, balanced split of unit indices 0..n_units-1 over ranks."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return list(range(start, start + count))


def gather_traces(local: Dict[int, Tuple[float, float]], n_units: int, group=None) -> List[Tuple[float, float]]:
    """All-gather {unit: (tr_X, tr_G)} from every rank; returns the full list
    ordered by unit index.  Works with the gloo and nccl backends."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    parts: List[Dict[int, Tuple[float, float]]] = [None] * world  # type: ignore[list-item]
    dist.all_gather_object(parts, dict(local), group=group)
    full: Dict[int, Tuple[float, float]] = {}
    for p in parts:
        full.update(p)
    missing = [u for u in range(n_units) if u not in full]
    if missing:
        raise RuntimeError(f"sensitivities missing for units {missing[:8]}")
    return [full[u] for u in range(n_units)]


def allocate_from_traces(traces: Sequence[Tuple[float, float]], sizes: Sequence[int],
                         avg_bits: float = 2.5, bmin: int = 2, bmax: int = 4) -> List[int]:
    """Bit widths from s = tr(H_G) tr(H_X) via the library's host allocator."""
    from . import kronq_allocate_bits

    sens = [tx * tg for tx, tg in traces]
    return kronq_allocate_bits(sens, sizes, avg_bits, bmin, bmax)
