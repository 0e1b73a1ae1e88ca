"""The whole per-layer pass, chained from the oracle's steps.

Order (KronQ README "Reproduce from scratch" recipe, weight-only):
factors -> sensitivity -> BiIP forward -> dead columns, damping, U -> GPTQ
sweep -> (pack) ; the K-FAC loss of the result is evaluated in the original
space after the BiIP inverse.
"""
from __future__ import annotations

import numpy as np

from . import biip, factors, loss, sweep


def quantize_layer(X, G, W, bits: int, group: int, asym: bool = True,
                   damp_rel: float = 0.01, seed: int = 0, alpha: float = 0.25,
                   mode: str = "full", block: int = 128):
    HX = factors.factor(X)
    HG = factors.factor(G)
    trx, trg, s = factors.sensitivity(HX, HG)
    Wt, HXt, HGt, d_in, d_out = biip.biip_forward(W, HX, HG, seed, alpha, mode)
    res = sweep.quantize_factored(Wt, HXt, bits, group, asym, damp_rel, block)
    What = biip.biip_inverse(res["Q"], seed, mode, d_in, d_out)
    W64 = np.asarray(W, dtype=np.float64)
    L = loss.kfac_loss(W64 - What, HX, HG)
    return dict(HX=HX, HG=HG, trX=trx, trG=trg, s=s, Wt=Wt, HXt=HXt, HGt=HGt,
                d_in=d_in, d_out=d_out, What=What, loss=L, **res)
