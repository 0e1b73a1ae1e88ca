"""Inter-layer mixed precision over a Llama-3-8B-shaped block (KronQ README
"--inter_layer_mp"; abstract point (2)): the trace-only first pass, the
allocation at a 2.5-bit average over {2, 3, 4}, and the per-layer passes at
the allocated widths with the built-in trace check.  One block of the seven
sublayers at their full shapes (q/o 4096 x 4096, k/v 1024 x 4096, gate/up
14336 x 4096, down 4096 x 14336), 4096 tokens each."""
import numpy as np
import pytest
import torch

import post_quantization_kronq_b200 as kq
from oracle import alloc, factors
from post_quantization_kronq_b200.stack import StackPass
from synth import LLAMA_SHAPES, llama_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
SUBLAYERS = ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]
T = 4096


def _data(i, block=0):
    m, n = LLAMA_SHAPES["llama3_8b_" + SUBLAYERS[i]]
    return llama_layer(m, n, T, seed=1000 * block + i, device=DEV,
                       rectified=(SUBLAYERS[i] == "down_proj"))


def test_trace_tokens_matches_oracle_and_streams():
    W, X, G = llama_layer(384, 1000, 3000, seed=3, device=DEV)
    tr = torch.zeros(2, dtype=torch.float64, device=DEV)
    kq.kronq_trace_tokens(X, tr[0:1])
    for t0 in range(0, 3000, 1024):                 # streamed in chunks
        kq.kronq_trace_tokens(G[t0:t0 + 1024], tr[1:2], zero_first=(t0 == 0))
    trx, trg, s = kq.kronq_sensitivity_from_traces(tr)
    rx = factors.trace_from_rows(X.float().cpu().numpy())
    rg = factors.trace_from_rows(G.float().cpu().numpy())
    assert abs(trx - rx) <= 1e-12 * rx and abs(trg - rg) <= 1e-12 * rg
    assert s == trg * trx
    # a strided view (row stride > d) takes the scalar path
    kq.kronq_trace_tokens(X[:, :999], tr[0:1])
    r2 = factors.trace_from_rows(X[:, :999].float().cpu().numpy())
    assert abs(float(tr[0].item()) - r2) <= 1e-12 * r2


def test_llama3_8b_block_mixed_precision():
    shapes = [LLAMA_SHAPES["llama3_8b_" + s] for s in SUBLAYERS]
    sp = StackPass(shapes, avg_bits=2.5, group=128)
    sens1 = sp.trace_pass(_data)
    for i, (trx, trg, s) in enumerate(sens1):
        _, X, G = _data(i)
        rx = factors.trace_from_rows(X.float().cpu().numpy())
        rg = factors.trace_from_rows(G.float().cpu().numpy())
        assert abs(trx - rx) <= 1e-12 * rx and abs(trg - rg) <= 1e-12 * rg
    bits = sp.allocate()
    sizes = [m * n for m, n in shapes]
    assert bits == list(alloc.allocate_budget([t[2] for t in sens1], sizes, 2.5, 2, 4))
    assert all(b in (2, 3, 4) for b in bits)
    assert sum(b * z for b, z in zip(bits, sizes)) <= 2.5 * sum(sizes)
    seen = []

    def on_layer(i, lp):
        torch.cuda.synchronize()
        assert int(lp.info.item()) == 0
        codes = lp.codes
        assert int(codes.max().item()) <= 2 ** bits[i] - 1
        seen.append(i)

    sp.sens2 = []
    for i in range(len(shapes)):
        W, X, G = _data(i)
        on_layer(i, sp.quantize_one(i, W, X, G))     # raises if the traces disagree
    assert seen == list(range(7))
    for i in range(7):
        assert abs(sp.sens2[i][0] - sens1[i][0]) <= 1e-3 * sens1[i][0]
    assert kq.kronq_device_status() == 0
