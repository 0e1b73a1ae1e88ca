"""One KronQ layer pass chained through the C ABI with preallocated buffers.

Order (KronQ README "Reproduce from scratch", weight-only recipe): factor
accumulation (H_X from X, H_G from G, streamed in token chunks) ->
sensitivity tr(H_G) tr(H_X) -> BiIP forward -> damping, Cholesky factor of
the damped inverse and the GPTQ sweep -> int2/int4 packing.  Every step is a
library call; this class only owns the device buffers.
"""
from __future__ import annotations

import torch

from . import (QuantParams, kronq_accumulate_factors, kronq_biip_forward,
               kronq_biip_workspace_bytes, kronq_pack, kronq_quantize_layer,
               kronq_quantize_workspace_bytes, kronq_sensitivity, words_per_row, workspace)


class LayerPass:
    def __init__(self, m: int, n: int, bits: int = 4, group: int = 128, asym: bool = True,
                 damp_rel: float = 0.01, seed: int = 0, alpha: float = 0.25, mode: str = "full",
                 flags: int = 0, device="cuda"):
        self.m, self.n, self.bits, self.group = m, n, bits, group
        self.seed, self.alpha, self.mode = seed, alpha, mode
        dev = torch.device(device)
        f32 = torch.float32
        self.params = QuantParams(bits=bits, group=group, asym=1 if asym else 0,
                                  damp_rel=damp_rel, block=128, flags=flags)
        ng = 1 if group == -1 else -(-n // group)
        self.HX = torch.empty(n, n, dtype=f32, device=dev)
        self.HG = torch.empty(m, m, dtype=f32, device=dev)
        self.Wt = torch.empty(m, n, dtype=f32, device=dev)
        self.d_in = torch.empty(n, dtype=f32, device=dev)
        self.d_out = torch.empty(m, dtype=f32, device=dev)
        self.codes = torch.empty(m, n, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(m, ng, dtype=f32, device=dev)
        self.zeros = torch.empty(m, ng, dtype=f32, device=dev)
        self.info = torch.zeros(1, dtype=torch.int32, device=dev)
        self.packed = (torch.empty(m, words_per_row(n, bits), dtype=torch.int32, device=dev)
                       if bits in (2, 4) else None)
        self.ws_biip = workspace(kronq_biip_workspace_bytes(m, n), dev)
        self.ws_quant = workspace(kronq_quantize_workspace_bytes(m, n, self.params), dev)
        self.ws_small = workspace(256, dev)
        self.sens = None

    def accumulate(self, X, G, chunk: int | None = None, stream=None):
        T = X.shape[0]
        chunk = T if chunk is None else chunk
        for t0 in range(0, max(T, 1), chunk):
            t1 = min(T, t0 + chunk)
            kronq_accumulate_factors(X[t0:t1], self.HX, zero_first=(t0 == 0), stream=stream)
            kronq_accumulate_factors(G[t0:t1], self.HG, zero_first=(t0 == 0), stream=stream)

    def sensitivity(self, stream=None):
        self.sens = kronq_sensitivity(self.HX, self.HG, self.ws_small, stream=stream)
        return self.sens

    def transform(self, W, stream=None):
        kronq_biip_forward(W, self.Wt, self.HX, self.HG, self.seed, self.alpha, self.mode,
                           self.d_in, self.d_out, self.ws_biip, stream=stream)

    def quantize(self, stream=None):
        kronq_quantize_layer(self.Wt, self.HX, self.params, self.codes, self.scales, self.zeros,
                             self.info, ws=self.ws_quant, stream=stream)
        if self.packed is not None:
            kronq_pack(self.codes, self.bits, self.packed, stream=stream)

    def run(self, X, G, W, chunk: int | None = None, with_sensitivity: bool = True, stream=None):
        self.accumulate(X, G, chunk, stream=stream)
        if with_sensitivity:
            self.sensitivity(stream=stream)
        self.transform(W, stream=stream)
        self.quantize(stream=stream)
