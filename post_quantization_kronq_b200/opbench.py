"""Run (and time) one library call on a synthetic input of a chosen size.

    python -m post_quantization_kronq_b200.opbench accumulate --tokens 16384 --d 4096 [--reps 3]
    python -m post_quantization_kronq_b200.opbench biip --m 4096 --n 4096
    python -m post_quantization_kronq_b200.opbench biip_inverse --m 2048 --n 28672
    python -m post_quantization_kronq_b200.opbench quantize --m 4096 --n 4096 --bits 2
    python -m post_quantization_kronq_b200.opbench pack --m 8192 --n 28672 --bits 2
    python -m post_quantization_kronq_b200.opbench kronfactors --est flipflop --tokens 131072 --m 4096 --n 4096
    python -m post_quantization_kronq_b200.opbench decode --m 4096 --n 4096 --bits 2 --reps 100
    python -m post_quantization_kronq_b200.opbench twosided --m 4096 --n 4096 --bits 2 [--u-given]

Meant for profiling a single kernel family (e.g. under ncu) at a size that
is smaller than the full benchmark; prints one JSON line with the mean
CUDA-event time per call.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    import torch

    import post_quantization_kronq_b200 as kq
    from post_quantization_kronq_b200.layer import LayerPass
    from synth import llama_layer

    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["accumulate", "biip", "biip_inverse", "quantize", "pack", "kronfactors",
                                   "decode", "twosided"])
    ap.add_argument("--u-given", action="store_true",
                    help="twosided: factor once, time the sweep alone (KRONQ_U_GIVEN)")
    ap.add_argument("--est", choices=["input", "marginal", "frobenius", "flipflop"], default="flipflop")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream()
    if a.op == "accumulate":
        X = llama_layer(8, a.d, a.tokens, seed=1, device=dev)[1]
        H = torch.empty(a.d, a.d, device=dev)
        run = lambda: kq.kronq_accumulate_factors(X, H, zero_first=True)  # noqa: E731
        units = {"flops": a.tokens * a.d * (a.d + 1)}
    elif a.op == "biip_inverse":
        # two row passes over W alone (rows of n, then rows of m), no factors
        Wt = torch.randn(a.m, a.n, device=dev)
        d_in = torch.ones(a.n, device=dev)
        d_out = torch.ones(a.m, device=dev)
        ws = kq.workspace(kq.kronq_biip_workspace_bytes(a.m, a.n), dev)
        run = lambda: kq.kronq_biip_inverse(Wt, 0, "full", d_in, d_out, ws=ws)  # noqa: E731
        units = {"bytes": 16 * a.m * a.n}
    elif a.op == "decode":
        ng = -(-a.n // a.group)
        codes = torch.randint(0, 2 ** a.bits, (a.m, a.n), dtype=torch.uint8, device=dev)
        packed = torch.empty(a.m, kq.words_per_row(a.n, a.bits), dtype=torch.int32, device=dev)
        kq.kronq_pack(codes, a.bits, packed)
        sc = torch.rand(a.m, ng, device=dev) * 0.05 + 0.005
        zp = torch.randint(0, 2 ** a.bits, (a.m, ng), device=dev).float()
        d_in = torch.ones(a.n, device=dev)
        d_out = torch.ones(a.m, device=dev)
        x = torch.randn(a.n, device=dev).to(torch.bfloat16)
        y = torch.empty(a.m, device=dev)
        ws = kq.workspace(kq.kronq_decode_matvec_workspace_bytes(a.m, a.n), dev)
        run = lambda: kq.kronq_decode_matvec(packed, sc, zp, a.n, a.bits, a.group, 0, "full",  # noqa: E731
                                             d_in, d_out, x, y, ws=ws)
        units = {"bytes": packed.numel() * 4 + 2 * sc.numel() * 4 + a.n * 2 + a.m * 4}
    elif a.op == "kronfactors":
        _, X, G = llama_layer(a.m, a.n, a.tokens, seed=1, device=dev)
        A = torch.empty(a.n, a.n, device=dev)
        B = torch.empty(a.m, a.m, device=dev)
        info = torch.zeros(1, dtype=torch.int32, device=dev)
        est = {"input": kq.EST_INPUT, "marginal": kq.EST_MARGINAL, "frobenius": kq.EST_FROBENIUS,
               "flipflop": kq.EST_FLIPFLOP}[a.est]
        ws = kq.workspace(kq.kronq_kron_factors_workspace_bytes(a.tokens, a.n, a.m), dev)
        run = lambda: kq.kronq_kron_factors(X, G, est, a.iters, A, B, info, ws=ws)  # noqa: E731
        # per sweep: two weight products (2 T m^2 and 2 T n^2 flop) and two
        # SYRKs (T n (n+1) and T m (m+1))
        units = {"flops_per_sweep": 2 * a.tokens * (a.m * a.m + a.n * a.n)
                 + a.tokens * (a.n * (a.n + 1) + a.m * (a.m + 1))}
    elif a.op == "twosided":
        W, X, G = llama_layer(a.m, a.n, 2 * max(a.m, a.n), seed=1, device=dev)
        HX0 = torch.empty(a.n, a.n, device=dev)
        HG0 = torch.empty(a.m, a.m, device=dev)
        kq.kronq_accumulate_factors(X, HX0, zero_first=True)
        kq.kronq_accumulate_factors(G, HG0, zero_first=True)
        W0 = W.float().contiguous()
        ng = 1 if a.group == -1 else -(-a.n // a.group)
        Wt, HX, HG = W0.clone(), HX0.clone(), HG0.clone()
        codes = torch.empty(a.m, a.n, dtype=torch.uint8, device=dev)
        sc = torch.empty(a.m, ng, device=dev)
        zp = torch.empty(a.m, ng, device=dev)
        info = torch.zeros(2, dtype=torch.int32, device=dev)
        p = kq.QuantParams(bits=a.bits, group=a.group, asym=1, damp_rel=0.01, block=128, flags=0)
        ws = kq.workspace(kq.kronq_quantize_two_sided_workspace_bytes(a.m, a.n, p), dev)
        if a.u_given:
            kq.kronq_quantize_two_sided(Wt, HX, HG, p, codes, sc, zp, info, ws=ws)
            HX0, HG0 = HX.clone(), HG.clone()
            p = kq.QuantParams(bits=a.bits, group=a.group, asym=1, damp_rel=0.01, block=128, flags=kq.U_GIVEN)

        def run():
            Wt.copy_(W0)
            HX.copy_(HX0)
            HG.copy_(HG0)
            kq.kronq_quantize_two_sided(Wt, HX, HG, p, codes, sc, zp, info, ws=ws)
        # the feedback as two triangular products, E U_X and U_G^T (E U_X)
        units = {"weights": a.m * a.n, "flops": a.m * a.n * (a.m + a.n)}
    else:
        W, X, G = llama_layer(a.m, a.n, 2 * max(a.m, a.n), seed=1, device=dev)
        lp = LayerPass(a.m, a.n, bits=a.bits, group=a.group, device=dev)
        lp.accumulate(X, G)
        if a.op == "biip":
            HX0, HG0 = lp.HX.clone(), lp.HG.clone()

            def run():
                lp.HX.copy_(HX0)
                lp.HG.copy_(HG0)
                lp.transform(W)
            units = {"bytes": 2 * (2 + 4) * a.m * a.n + 16 * a.n * a.n + 16 * a.m * a.m}
        elif a.op == "quantize":
            lp.transform(W)
            HX0, W0 = lp.HX.clone(), lp.Wt.clone()

            def run():
                lp.HX.copy_(HX0)
                lp.Wt.copy_(W0)
                lp.quantize()
            units = {"weights": a.m * a.n}
        else:
            codes = torch.randint(0, 2 ** a.bits, (a.m, a.n), dtype=torch.uint8, device=dev)
            out = torch.empty(a.m, kq.words_per_row(a.n, a.bits), dtype=torch.int32, device=dev)
            run = lambda: kq.kronq_pack(codes, a.bits, out)  # noqa: E731
            units = {"bytes": a.m * a.n * (1 + a.bits / 8)}
    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(a.reps):
        run()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.reps
    if a.op in ("decode", "biip_inverse"):
        units["gbs"] = units["bytes"] / (ms / 1e3) / 1e9
    if a.op == "twosided":
        units["info"] = info.tolist()
        units["tflops"] = units["flops"] / (ms / 1e3) / 1e12
    if a.op == "kronfactors":
        units["info"] = int(info.item())
        units["tflops"] = units["flops_per_sweep"] * a.iters / (ms / 1e3) / 1e12
    print(json.dumps({"op": a.op, "ms_per_call": ms, "args": vars(a), **units}))
    return 0


if __name__ == "__main__":
    sys.exit(main())
