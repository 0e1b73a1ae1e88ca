"""Seeded synthetic layer workloads shared by the CPU oracle tests, the GPU
parity tests and the benchmark.

This module only draws random numbers with the shapes and distributions of the
layers the KronQ pages quantize (Llama-2-7B and Llama-3-70B sublayers, see the
KronQ README "Model zoo" table); it holds none of the method's arithmetic.

Recipes (draw order inside one layer: W, then X, then G; inside X and G:
per-channel scales first, then values, then outlier channel indices):

* ``tiny_layer`` -- the 256x256 single-layer case: numpy ``default_rng(seed)``;
  W ~ N(0, 0.02^2); X = N(0,1) * exp(N(0,1)) per channel with 4 outlier
  channels scaled x10; G = N(0,1) * exp(N(0, 0.5^2)) per channel; all float32.
* ``llama_layer`` -- torch ``Generator(device).manual_seed(seed)``;
  W ~ N(0, w_std^2); X = Student-t(4) * exp(N(0,1)) per channel (|t| when
  ``rectified``, the down_proj input); G = N(0, 1e-4) * exp(N(0,1)) per
  channel; everything cast to bf16 at the end.  Student-t(4) is drawn as
  z / sqrt(Gamma(2,1) / 2) with Gamma(2,1) = -(ln u1 + ln u2).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["tiny_layer", "llama_layer", "LLAMA_SHAPES"]

# (m, n) = (out, in) of the sublayers the pages' models use.
LLAMA_SHAPES = {
    "llama2_7b_q_proj": (4096, 4096),
    "llama2_7b_up_proj": (11008, 4096),
    "llama2_7b_gate_proj": (11008, 4096),
    "llama2_7b_down_proj": (4096, 11008),
    "llama3_70b_gate_proj": (28672, 8192),
    "llama3_70b_up_proj": (28672, 8192),
    "llama3_70b_down_proj": (8192, 28672),
    "llama3_8b_q_proj": (4096, 4096),
    "llama3_8b_k_proj": (1024, 4096),
    "llama3_8b_v_proj": (1024, 4096),
    "llama3_8b_o_proj": (4096, 4096),
    "llama3_8b_gate_proj": (14336, 4096),
    "llama3_8b_up_proj": (14336, 4096),
    "llama3_8b_down_proj": (4096, 14336),
}


def tiny_layer(m: int = 256, n: int = 256, T: int = 2048, seed: int = 0,
               n_outliers: int = 4):
    """Return float32 numpy (W m x n, X T x n, G T x m)."""
    rng = np.random.default_rng(seed)
    W = rng.normal(0.0, 0.02, size=(m, n)).astype(np.float32)
    x_scale = np.exp(rng.normal(0.0, 1.0, size=n))
    X = rng.normal(0.0, 1.0, size=(T, n)) * x_scale[None, :]
    outl = rng.choice(n, size=min(n_outliers, n), replace=False)
    X[:, outl] *= 10.0
    g_scale = np.exp(rng.normal(0.0, 0.5, size=m))
    G = rng.normal(0.0, 1.0, size=(T, m)) * g_scale[None, :]
    return W, X.astype(np.float32), G.astype(np.float32)


def llama_layer(m: int, n: int, T: int, seed: int = 0, device="cpu",
                w_std: float = 0.02, rectified: bool = False,
                chunk_rows: int = 8192):
    """Return bf16 torch tensors (W m x n, X T x n, G T x m) on ``device``.

    Values are drawn in float32 in row chunks of ``chunk_rows`` tokens so that
    the full-size workloads (T = 131072) stay within a few GB of temporaries.
    """
    import torch

    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    bf = torch.bfloat16
    W = (torch.randn(m, n, generator=gen, device=dev) * w_std).to(bf)

    x_scale = torch.exp(torch.randn(n, generator=gen, device=dev))
    X = torch.empty(T, n, dtype=bf, device=dev)
    for r0 in range(0, T, chunk_rows):
        r1 = min(T, r0 + chunk_rows)
        z = torch.randn(r1 - r0, n, generator=gen, device=dev)
        u1 = torch.rand(r1 - r0, n, generator=gen, device=dev).clamp_min_(1e-30)
        u2 = torch.rand(r1 - r0, n, generator=gen, device=dev).clamp_min_(1e-30)
        gam = -(torch.log(u1) + torch.log(u2))
        t = z / torch.sqrt(gam * 0.5)
        if rectified:
            t = t.abs()
        X[r0:r1] = (t * x_scale[None, :]).to(bf)
        del z, u1, u2, gam, t

    g_scale = torch.exp(torch.randn(m, generator=gen, device=dev))
    G = torch.empty(T, m, dtype=bf, device=dev)
    for r0 in range(0, T, chunk_rows):
        r1 = min(T, r0 + chunk_rows)
        v = torch.randn(r1 - r0, m, generator=gen, device=dev) * math.sqrt(1e-4)
        G[r0:r1] = (v * g_scale[None, :]).to(bf)
        del v
    return W, X, G
