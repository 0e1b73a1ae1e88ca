"""Benchmark of KronQ's per-layer quantization pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kronq|reference]
                    [--bits 2|3|4] [--group 128] [--no-e2e] [--no-cpu-baseline]

Workload: a Llama-2-7B q_proj-shaped layer, W 4096 x 4096 bf16 ~ N(0, 0.02^2),
X and G 131072 x 4096 bf16 (X Student-t(4) with lognormal per-channel scale,
G N(0, 1e-4) with lognormal per-channel scale), 2-bit group-128 asymmetric
(the pages' headline bit width), BiIP "full", alpha 0.25, damping 0.01.

One step = the whole pass on inputs resident in HBM: H_X and H_G
accumulation, trace sensitivity, BiIP forward, damping + Cholesky factor of
the damped inverse + GPTQ sweep, int2 packing.  Metric: weights quantized
per second (m n / seconds per layer, factor accumulation included).  Each
step is timed with CUDA events on the launching stream; L2 is flushed by a
256 MB write between steps (outside the timed interval).

Under torchrun (N > 1) every rank quantizes its own layer (weak scaling, no
data-path collective); the time is the max over ranks.

``--impl reference`` times the CPU float64 oracle on this machine's host cores on
a bounded sample of the same workload and reports the same metric
(extrapolated by exact operation counts).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "weights quantized/sec per layer (incl. H_X/H_G accumulation); % of roofline"
UNIT = "weights/s"
M = N_IN = 4096
TOKENS = 131072
# dram__bytes_read.sum / dram__bytes_write.sum of one syrk_bf16_tc_kernel launch
# at T = 16384, d = 4096 (ncu, B200), used for roofline.traffic
SYRK_READ_BYTES_T16384 = 225.659136e6
E2E_CHUNK = 16384   # tokens per host->device copy chunk in the end-to-end pass
SYRK_WRITE_BYTES_D4096 = 41.663232e6
WORKLOAD = "llama2-7b q_proj 4096x4096, T=131072 tokens, W{bits} g{group} asym, BiIP full"


def _peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


def phase_rooflines(phases_ms, m: int, n: int, T: int, peaks):
    """Each timed phase's algorithmic work over the measured peak of its bound.

    accumulate_HX_HG  tensor: T n (n+1) + T m (m+1) flop (the distinct entries
                      of the two SYRKs)
    sensitivity       HBM: the two diagonals, 4 (n + m) bytes
    biip_forward      HBM: 16 m n + 16 n^2 + 16 m^2 bytes (W's norms read
                      2 m n; its two passes read 2 + 4 and write 4 + 4 bytes
                      per element; each factor takes two fp32 passes in and out)
    quantize_and_pack bound by its sequential chains (64 diagonal steps of
                      the factorisation, n column steps of the sweep); shown
                      against the tensor peak with 2 n^3 / 3 + m n^2 flop (the
                      reverse Cholesky factor and its triangular inverse, and
                      the error feedback of the sweep)
    """
    if peaks:
        tpk, hpk, src = peaks["bf16_tflops_sustained"], peaks["hbm_gbs"], "measured"
    else:
        tpk, hpk, src = 1400.0, 6650.0, "fallback"
    work = {
        "accumulate_HX_HG": ("tensor", T * n * (n + 1) + T * m * (m + 1), "TFLOP/s", tpk, 1e12),
        "sensitivity": ("hbm", 4 * (n + m), "GB/s", hpk, 1e9),
        "biip_forward": ("hbm", 16 * m * n + 16 * n * n + 16 * m * m, "GB/s", hpk, 1e9),
        "quantize_and_pack": ("latency (sequential chains)", 2 * n ** 3 / 3 + m * n * n, "TFLOP/s", tpk, 1e12),
    }
    out = {}
    for name, ms in phases_ms.items():
        if name not in work or ms <= 0:
            continue
        bound, units, unit, peak, scale = work[name]
        achieved = units / (ms / 1e3) / scale
        out[name] = {"bound": bound, "achieved": achieved, "unit": unit, "peak": peak,
                     "frac": achieved / peak, "peak_source": src}
    return out


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling during the timed region (200 ms period)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        load = [s for s in sm if s > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ----------------------------------------------------------------- CPU oracle sample
def cpu_oracle_sample(bits: int, group: int, seed: int = 0, t_sample: int = 4096, rows: int = 64):
    """Time the float64 oracle on a bounded sample of the workload and
    extrapolate to one full layer by exact operation counts.

    Sample: factor accumulation over t_sample tokens of X (scaled by
    2 * TOKENS / t_sample for H_X and H_G), the full BiIP of W and H_X
    (scaled by 3/2 for H_G), the full inverse + Cholesky of the damped
    H~_X, the non-lazy sweep of ``rows`` rows (scaled by M / rows), and the
    packing of those rows (scaled likewise)."""
    import numpy as np

    from oracle import biip, factors, pack, sweep
    from synth import llama_layer

    W, X, G = llama_layer(M, N_IN, t_sample, seed=seed, device="cpu")
    Xn = X.float().numpy()
    Wn = W.float().numpy().astype(np.float64)
    t = {}
    t0 = time.perf_counter()
    HX = factors.factor(Xn)
    t["factors"] = (time.perf_counter() - t0) * (2 * TOKENS / t_sample)
    HG = HX.copy()  # same size; its values do not change the cost of what follows
    t0 = time.perf_counter()
    Wt, HXt, _, din, dout = biip.biip_forward(Wn, HX, None, seed, 0.25, "sv_only")
    Wt = biip.rotate_rows(Wt.T, seed, 1).T
    t["biip"] = (time.perf_counter() - t0) * 1.5
    t0 = time.perf_counter()
    H1, W1, _ = sweep.dead_columns(HXt, Wt)
    A, _ = sweep.damp(H1, 0.01)
    U = sweep.chol_upper_of_inverse(A)
    t["factorisation"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    res = sweep.gptq_sweep(W1[:rows], U, bits, group, True, block=1)
    if bits in (2, 4):
        pack.pack(res["codes"], bits)
    t["sweep"] = (time.perf_counter() - t0) * (M / rows)
    total = sum(t.values())
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    sample = (f"oracle (numpy float64) on {t_sample} tokens for the factors, full BiIP and "
              f"factorisation, {rows} rows for the sweep; extrapolated to the full layer by "
              f"operation counts")
    return {"value": M * N_IN / total, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": sample, "seconds_per_layer": total,
            "phases_s": {k: round(v, 3) for k, v in t.items()}}


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(args.bits, args.group, seed=i, t_sample=2048, rows=32)
        if i >= args.warmup:
            vals.append(r["seconds_per_layer"])
        last = r
    spl = statistics.mean(vals)
    value = M * N_IN / spl
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": spl * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD.format(bits=args.bits, group=args.group),
                       "m": M, "n": N_IN, "tokens": TOKENS, "bits": args.bits, "group": args.group},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm
def run_kronq(args):
    import torch

    import post_quantization_kronq_b200 as kq
    from post_quantization_kronq_b200.layer import LayerPass
    from synth import llama_layer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    stream = torch.cuda.current_stream()
    bits, group = args.bits, args.group
    W, X, G = llama_layer(M, N_IN, TOKENS, seed=1000 + rank, device=dev)
    lp = LayerPass(M, N_IN, bits=bits, group=group, seed=rank, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(rec=None):
        if rec is not None:
            rec[0].record(stream)
        lp.accumulate(X, G)
        if rec is not None:
            rec[1].record(stream)
        lp.sensitivity()
        if rec is not None:
            rec[2].record(stream)
        lp.transform(W)
        if rec is not None:
            rec[3].record(stream)
        lp.quantize()
        if rec is not None:
            rec[4].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert int(lp.info.item()) == 0, "factorisation reported a non-positive pivot"

    recs = [[ev() for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    launches0 = kq.kronq_launch_count()
    for k in range(args.steps):
        flush.zero_()
        torch.cuda.nvtx.range_push("kronq_timed_step")
        step(recs[k])
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    launches = kq.kronq_launch_count() - launches0
    barrier()
    clocks = sampler.stop()
    step_ms = [r[0].elapsed_time(r[4]) for r in recs]
    acc_ms = [r[0].elapsed_time(r[1]) for r in recs]
    phases = {
        "accumulate_HX_HG": statistics.mean(acc_ms),
        "sensitivity": statistics.mean(r[1].elapsed_time(r[2]) for r in recs),
        "biip_forward": statistics.mean(r[2].elapsed_time(r[3]) for r in recs),
        "quantize_and_pack": statistics.mean(r[3].elapsed_time(r[4]) for r in recs),
    }
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * M * N_IN * args.steps / (total_ms / 1e3)

    # Roofline of the dominant kernel: the tcgen05 SYRK (two launches per step,
    # one per factor, both d = 4096).  Algorithmic flops per launch: T d (d + 1).
    syrk_launch_ms = statistics.mean(acc_ms) / 2.0
    flops = TOKENS * N_IN * (N_IN + 1)
    achieved = flops / (syrk_launch_ms / 1e3) / 1e12
    peaks = _peaks()
    if peaks:
        peak, peak_src = peaks["bf16_tflops_sustained"], "measured (sustained bf16, MEASURED_PEAKS.json)"
    else:
        peak, peak_src = 1400.0, "fallback (sustained)"
    # DRAM traffic per launch, from one ncu capture of the same kernel at
    # T = 16384, d = 4096 (dram__bytes_read.sum 225.66 MB, dram__bytes_write.sum
    # 41.66 MB): the token reads grow in proportion to T, the H write does not.
    traffic = SYRK_READ_BYTES_T16384 * (TOKENS / 16384) + SYRK_WRITE_BYTES_D4096
    roofline = {"bound": "tensor", "kernel": "syrk_bf16_tc_kernel", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "traffic_source": "ncu capture at T=16384 (d=4096), reads scaled by T/16384",
                "peak_source": peak_src,
                "flops_per_launch": flops, "launch_ms": syrk_launch_ms}

    # End to end through the public API: inputs copied from pinned host memory
    # every step, packed codes, scales and zeros copied back.
    e2e = None
    if not args.no_e2e:
        hX = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
        hG = torch.empty(G.shape, dtype=G.dtype, pin_memory=True)
        hW = torch.empty(W.shape, dtype=W.dtype, pin_memory=True)
        hX.copy_(X)
        hG.copy_(G)
        hW.copy_(W)
        outs = [lp.packed if lp.packed is not None else lp.codes, lp.scales, lp.zeros]
        houts = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        h2d = sum(t.numel() * t.element_size() for t in (hX, hG, hW))
        d2h = sum(t.numel() * t.element_size() for t in houts)

        def e2e_step():
            # token chunks of X and G copied on a second stream while the
            # factor accumulation of the earlier chunks runs
            lp.run_from_host(hX, hG, hW, X, G, W, chunk=E2E_CHUNK, stream=stream)
            for h, o in zip(houts, outs):
                h.copy_(o, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e_steps = max(2, min(args.steps, 5))
        barrier()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1)
        if dist is not None:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": world * M * N_IN * e_steps / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "pipeline": f"X, G copied in {E2E_CHUNK}-token chunks on a second stream, "
                           "overlapping the factor accumulation and the previous step's sweep"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_sample(bits, group)
        cpu = {k: c[k] for k in ("value", "unit", "cores", "kind", "sample")}
        cpu["phases_s"] = c["phases_s"]

    if dist is not None:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD.format(bits=bits, group=group), "m": M, "n": N_IN,
                   "tokens": TOKENS, "bits": bits, "group": group, "accumulate": "f32",
                   "l2": "flushed between steps (256 MB write, outside the timed interval)",
                   "parallelism": f"dp{world} (one layer per GPU)"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": launches,
        "phases_ms": {k: round(v, 4) for k, v in phases.items()},
        "phase_roofline": phase_rooflines(phases, M, N_IN, TOKENS, peaks),
        "sensitivity": list(lp.sens) if lp.sens else None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kronq", "reference"], default="kronq")
    ap.add_argument("--bits", type=int, default=2, choices=[2, 3, 4])
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.impl == "reference":
        return run_reference(args)
    return run_kronq(args)


if __name__ == "__main__":
    sys.exit(main())
