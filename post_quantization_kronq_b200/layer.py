"""One KronQ layer pass chained through the C ABI with preallocated buffers.

Order (KronQ README "Reproduce from scratch", weight-only recipe): factor
accumulation (H_X from X, H_G from G, streamed in token chunks) ->
sensitivity tr(H_G) tr(H_X) -> BiIP forward -> damping, Cholesky factor of
the damped inverse and the GPTQ sweep -> int2/int4 packing.  Every step is a
library call; this class only owns the device buffers.
"""
from __future__ import annotations

import torch

from . import (R_FORM, QuantParams, kronq_accumulate_factors, kronq_biip_forward,
               kronq_biip_workspace_bytes, kronq_pack, kronq_quantize_layer,
               kronq_quantize_workspace_bytes, kronq_sensitivity, words_per_row, workspace)


class LayerPass:
    """flags: the kronq_quant_params flags; None picks KRONQ_R_FORM (the sweep
    on the factor R, no inverse formed; HX holds R after quantize) wherever it
    applies (groups of at most 128 columns or one per row), else 0 (HX holds
    U after quantize)."""

    def __init__(self, m: int, n: int, bits: int = 4, group: int = 128, asym: bool = True,
                 damp_rel: float = 0.01, seed: int = 0, alpha: float = 0.25, mode: str = "full",
                 flags: int | None = None, device="cuda"):
        if flags is None:
            flags = R_FORM if (group == -1 or group <= 128) else 0
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

    def run_from_host(self, hX, hG, hW, X, G, W, chunk: int = 16384, with_sensitivity: bool = True,
                      stream=None, copy_stream=None):
        """One layer pass from pinned host inputs, copies overlapped with compute.

        Token chunks of X and G (hX, hG: pinned host tensors) are copied into the
        device buffers X and G on ``copy_stream`` while the factor accumulation
        of the chunks already on the device runs on ``stream``; W's copy goes
        last on the copy stream.  Across calls, the next call's copies of X and
        G wait only for this call's last accumulation (and W's copy for this
        call's BiIP forward), so they overlap this call's BiIP and sweep.  The
        arithmetic is that of ``run(X, G, W, chunk)``: same launches, same order.
        """
        compute = torch.cuda.current_stream() if stream is None else stream
        if copy_stream is None:
            if getattr(self, "_copy_stream", None) is None:
                self._copy_stream = torch.cuda.Stream(device=X.device)
            copy_stream = self._copy_stream
        T = X.shape[0]
        prev_acc = getattr(self, "_ev_acc_done", None)
        prev_w = getattr(self, "_ev_w_done", None)
        if prev_acc is None:
            copy_stream.wait_stream(compute)
        else:
            copy_stream.wait_event(prev_acc)
        ready = []
        with torch.cuda.stream(copy_stream):
            for t0 in range(0, max(T, 1), chunk):
                t1 = min(T, t0 + chunk)
                X[t0:t1].copy_(hX[t0:t1], non_blocking=True)
                G[t0:t1].copy_(hG[t0:t1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                ready.append((t0, t1, ev))
            if prev_w is not None:
                copy_stream.wait_event(prev_w)
            W.copy_(hW, non_blocking=True)
            w_ready = torch.cuda.Event()
            w_ready.record(copy_stream)
        for t0, t1, ev in ready:
            compute.wait_event(ev)
            kronq_accumulate_factors(X[t0:t1], self.HX, zero_first=(t0 == 0), stream=compute)
            kronq_accumulate_factors(G[t0:t1], self.HG, zero_first=(t0 == 0), stream=compute)
        self._ev_acc_done = torch.cuda.Event()
        self._ev_acc_done.record(compute)
        if with_sensitivity:
            self.sensitivity(stream=compute)
        compute.wait_event(w_ready)
        self.transform(W, stream=compute)
        self._ev_w_done = torch.cuda.Event()
        self._ev_w_done.record(compute)
        self.quantize(stream=compute)
