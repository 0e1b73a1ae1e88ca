"""A whole model's sublayers with inter-layer mixed precision.

KronQ README, "Mapping paper results to flags" (``--inter_layer_mp``) and
the bullet "Inter-layer mixed precision"; abstract point (2): bits are
allocated across sublayers by the sensitivity s = tr(H_G) tr(H_X).

Two passes over the calibration data of every sublayer:

1. traces only: tr(H_X) = sum_t |x_t|^2 and tr(H_G) = sum_t |g_t|^2 straight
   from the tokens (kronq_trace_tokens, one read of X and G, no factor is
   formed), and s from kronq_sensitivity_from_traces;
2. the bit widths from s (kronq_allocate_bits: budget rule over {bmin ..
   bmax} at an average of avg_bits), then the per-layer pass of each
   sublayer at its width (LayerPass).  Its factors give the traces again
   (kronq_sensitivity on the diagonals): they must equal the first pass's
   within a relative 1e-3 (the built-in consistency check).

Every step runs in the library; this module owns buffers and the order of
the calls.  ``data`` is a callable i -> (W, X, G) of device tensors for
sublayer i (called once per pass, so the inputs need not all be resident).
"""
from __future__ import annotations

from typing import Callable, Dict, List, Sequence, Tuple

import torch

from . import (kronq_allocate_bits, kronq_sensitivity_from_traces, kronq_trace_tokens, workspace)
from .layer import LayerPass

TRACE_RTOL = 1e-3


class StackPass:
    def __init__(self, shapes: Sequence[Tuple[int, int]], avg_bits: float = 2.5, bmin: int = 2,
                 bmax: int = 4, group: int = 128, chunk: int | None = None, seed: int = 0,
                 device="cuda"):
        self.shapes = [(int(m), int(n)) for m, n in shapes]
        self.avg_bits, self.bmin, self.bmax, self.group = avg_bits, bmin, bmax, group
        self.chunk, self.seed = chunk, seed
        self.dev = torch.device(device)
        self.traces = torch.zeros(2, dtype=torch.float64, device=self.dev)
        self.ws = workspace(256 * 1024, self.dev)
        self.sens1: List[Tuple[float, float, float]] = []
        self.bits: List[int] = []
        self.sens2: List[Tuple[float, float, float]] = []
        self._passes: Dict[Tuple[int, int, int], LayerPass] = {}

    # -------------------------------------------------------------- pass 1
    def trace_pass(self, data: Callable[[int], tuple], stream=None) -> List[Tuple[float, float, float]]:
        """(tr H_X, tr H_G, s) of every sublayer from its tokens alone."""
        self.sens1 = []
        for i in range(len(self.shapes)):
            _, X, G = data(i)
            self.sens1.append(self.trace_one(X, G, stream=stream))
        return self.sens1

    def trace_one(self, X, G, stream=None) -> Tuple[float, float, float]:
        kronq_trace_tokens(X, self.traces[0:1], zero_first=True, ws=self.ws, stream=stream)
        kronq_trace_tokens(G, self.traces[1:2], zero_first=True, ws=self.ws, stream=stream)
        return kronq_sensitivity_from_traces(self.traces, stream=stream)

    # -------------------------------------------------------------- allocation
    def allocate(self) -> List[int]:
        sizes = [m * n for m, n in self.shapes]
        self.bits = kronq_allocate_bits([t[2] for t in self.sens1], sizes, self.avg_bits, self.bmin,
                                        self.bmax)
        return self.bits

    # -------------------------------------------------------------- pass 2
    def layer_pass(self, i: int) -> LayerPass:
        m, n = self.shapes[i]
        key = (m, n, self.bits[i])
        lp = self._passes.get(key)
        if lp is None:
            lp = LayerPass(m, n, bits=self.bits[i], group=self.group, seed=self.seed, device=self.dev)
            self._passes[key] = lp
        return lp

    def quantize_one(self, i: int, W, X, G, stream=None) -> LayerPass:
        """The per-layer pass of sublayer i at its allocated width; checks its
        traces against the first pass's."""
        lp = self.layer_pass(i)
        lp.accumulate(X, G, chunk=self.chunk, stream=stream)
        sens = lp.sensitivity(stream=stream)
        lp.transform(W, stream=stream)
        lp.quantize(stream=stream)
        self.check_traces(i, sens)
        return lp

    def check_traces(self, i: int, sens) -> None:
        t1 = self.sens1[i]
        for k, name in ((0, "tr(H_X)"), (1, "tr(H_G)")):
            if abs(sens[k] - t1[k]) > TRACE_RTOL * abs(t1[k]):
                raise RuntimeError(f"sublayer {i}: {name} of the factors {sens[k]!r} differs from the "
                                   f"token pass {t1[k]!r} by more than {TRACE_RTOL}")
        while len(self.sens2) <= i:
            self.sens2.append(None)
        self.sens2[i] = sens

    def run(self, data: Callable[[int], tuple], on_layer: Callable[[int, LayerPass], None] | None = None,
            stream=None) -> List[int]:
        """Both passes; on_layer(i, layer_pass) sees each sublayer's outputs."""
        self.trace_pass(data, stream=stream)
        self.allocate()
        self.sens2 = []
        for i in range(len(self.shapes)):
            W, X, G = data(i)
            lp = self.quantize_one(i, W, X, G, stream=stream)
            if on_layer is not None:
                on_layer(i, lp)
        return self.bits
