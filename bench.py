"""Benchmark of KronQ's per-layer quantization pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kronq|reference]
                    [--workload llama3_70b_mlp|llama2_7b_q_proj] [--bits 2|3|4]
                    [--no-e2e] [--no-cpu-baseline] [--no-also]

Default workload: the two layer shapes of a Llama-3-70B MLP block,
gate_proj W 28672 x 8192 and down_proj W 8192 x 28672, bf16 ~ N(0, 0.015^2),
each with its own X and G of 262144 tokens (128 sequences x 2048) bf16 (X
Student-t(4) with lognormal per-channel scale, |t| for the down_proj input;
G N(0, 1e-4) with lognormal per-channel scale), the factors accumulated in
16 chunks of 16384 tokens; 2-bit group-128 asymmetric (the pages' headline
2-bit Llama-3-70B), BiIP "full", alpha 0.25, damping 0.01.  Beside it (key
"also"): a Llama-2-7B q_proj-shaped layer (4096 x 4096, T = 131072) at W2
and W4, and the Llama-3-8B-shaped stack (224 sublayers) with inter-layer
mixed precision, timed once after the rest.

One step = the whole pass over every layer of the workload on inputs
resident in HBM: H_X and H_G accumulation, trace sensitivity, BiIP forward,
damping + Cholesky factor of the damped inverse + GPTQ sweep, int2/int4
packing.  Metric: weights quantized per second (sum of m n over the step's
layers / seconds per step, factor accumulation included).  Each phase is
timed with CUDA events on the launching stream; L2 is flushed by a 256 MB
write between steps (outside the timed interval).

Under torchrun (N > 1) every rank quantizes its own copy of the workload
(weak scaling, no data-path collective); the time is the max over ranks.

``--impl reference`` times the CPU float64 oracle on this machine's host cores on
a bounded sample of the same workload and reports the same metric
(extrapolated by exact operation counts).
"""
from __future__ import annotations

import argparse
import json
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

# name -> description, tokens, chunk (None: one call), bits, group, w_std,
# layers [(sublayer, m, n, rectified X)]
WORKLOADS = {
    "llama3_70b_mlp": dict(
        desc="llama3-70b MLP gate_proj 28672x8192 + down_proj 8192x28672, T=262144 tokens "
             "(16 chunks of 16384), W{bits} g{group} asym, BiIP full",
        tokens=262144, chunk=16384, bits=2, group=128, w_std=0.015,
        layers=[("gate_proj", 28672, 8192, False), ("down_proj", 8192, 28672, True)]),
    "llama2_7b_q_proj": dict(
        desc="llama2-7b q_proj 4096x4096, T=131072 tokens, W{bits} g{group} asym, BiIP full",
        tokens=131072, chunk=None, bits=2, group=128, w_std=0.02,
        layers=[("q_proj", 4096, 4096, False)]),
}

# dram__bytes_read.sum + dram__bytes_write.sum of one factor-accumulation
# launch (syrk_pair_kernel, ncu on a B200), keyed by (d, tokens per
# launch); shapes not captured give traffic null.  (28672, 8192): the mean
# of the two launches of a 16384-token chunk.
SYRK_TRAFFIC = {
    (28672, 8192): (6687214336 + 3252186624 + 9249690880 + 3250075648) // 2,
    (8192, 16384): 1161290496 + 251058688,
}
# The library's launch rule for the factor accumulation: from d = 16384 on,
# a call's tokens go in launches of at most 8192.
SYRK_SPLIT_MIN_D, SYRK_SPLIT_T = 16384, 8192


def syrk_launches(d: int, tokens: int):
    """(launches, tokens per launch) of one accumulation call."""
    if d >= SYRK_SPLIT_MIN_D and tokens > SYRK_SPLIT_T:
        return -(-tokens // SYRK_SPLIT_T), SYRK_SPLIT_T
    return 1, tokens


def _peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


def choose_peak(peaks, clocks):
    """The bf16 tensor peak that applies to kernels timed inside this run:
    the burst figure, unless the clocks sampled during the timed region show
    the power cap (sw_power_cap, or a median SM clock below 93 % of the
    maximum), when the sustained figure applies."""
    if not peaks:
        return 1590.0, 6650.0, "fallback (burst)"
    capped = False
    if clocks:
        if "sw_power_cap" in (clocks.get("reasons") or []):
            capped = True
        sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
        if sm and mx and sm < 0.93 * mx:
            capped = True
    if capped:
        return peaks["bf16_tflops_sustained"], peaks["hbm_gbs"], "measured sustained (power-capped clocks)"
    return peaks["bf16_tflops"], peaks["hbm_gbs"], "measured burst (clocks not capped)"


def phase_work(layers, T: int):
    """Algorithmic work of each timed phase summed over the layers (m, n):

    accumulate_HX_HG  tensor: T n (n+1) + T m (m+1) flop (the distinct
                      entries of the two SYRKs)
    sensitivity       HBM: the two diagonals, 4 (n + m) bytes
    biip_forward      HBM: 16 m n + 16 n^2 + 16 m^2 bytes (W's norms read
                      2 m n; its two passes read 2 + 4 and write 4 + 4 bytes
                      per element; each factor takes two fp32 passes in and out)
    quantize_and_pack bound by its sequential chains (the diagonal steps of
                      the factorisation, n column steps of the sweep); shown
                      against the tensor peak with n^3 / 3 + m n^2 flop (the
                      reverse Cholesky factor R, and the error feedback of the
                      sweep, which the R form takes from R: no inverse)
    """
    w = {"accumulate_HX_HG": 0, "sensitivity": 0, "biip_forward": 0, "quantize_and_pack": 0}
    for m, n in layers:
        w["accumulate_HX_HG"] += T * n * (n + 1) + T * m * (m + 1)
        w["sensitivity"] += 4 * (n + m)
        w["biip_forward"] += 16 * m * n + 16 * n * n + 16 * m * m
        w["quantize_and_pack"] += n ** 3 / 3 + m * n * n
    return w


def phase_rooflines(phases_ms, layers, T: int, tpk: float, hpk: float, src: str):
    """Each timed phase's algorithmic work over the peak of its bound."""
    kinds = {
        "accumulate_HX_HG": ("tensor", "TFLOP/s", tpk, 1e12),
        "sensitivity": ("hbm", "GB/s", hpk, 1e9),
        "biip_forward": ("hbm", "GB/s", hpk, 1e9),
        "quantize_and_pack": ("latency (sequential chains)", "TFLOP/s", tpk, 1e12),
    }
    work = phase_work(layers, T)
    out = {}
    for name, ms in phases_ms.items():
        if name not in kinds or ms <= 0:
            continue
        bound, unit, peak, scale = kinds[name]
        achieved = work[name] / (ms / 1e3) / scale
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
def cpu_oracle_sample(wl: dict, bits: int, group: int, seed: int = 0, t_s: int = 1024,
                      d_s: int = 2048, rows_s: int = 64, sweep_rows: int = 16):
    """Time the float64 oracle on a bounded sample of every layer of the
    workload and extrapolate to the full layers by exact operation counts.

    Per layer (m, n; T tokens):
      factors   H = A^T A of t_s tokens x min(d, d_s) channels of X and of
                G, scaled by (T / t_s) (d / d_s)^2 (cost T d^2)
      BiIP      the oracle's row rotation of rows_s rows of each length, scaled
                by the rows of the two-sided transforms of W (m rows of n,
                n of m), H_X (2 n of n) and H_G (2 m of m)
      factor U  dead columns, damping, inverse and Cholesky at min(n, d_s),
                scaled by (n / n_s)^3
      sweep     the non-lazy float64 sweep of sweep_rows rows with that U and
                the packing of their codes, scaled by (m / sweep_rows)(n / n_s)^2
    """
    import numpy as np

    from oracle import biip, factors, pack, sweep
    from synth import llama_layer

    T = wl["tokens"]
    t = {"factors": 0.0, "biip": 0.0, "factorisation": 0.0, "sweep": 0.0}
    weights = 0
    for li, (_, m, n, rect) in enumerate(wl["layers"]):
        weights += m * n
        ns, ms_ = min(n, d_s), min(m, d_s)
        W, X, G = llama_layer(ms_, ns, t_s, seed=seed + li, device="cpu", w_std=wl["w_std"],
                              rectified=rect)
        Xn = X.float().numpy()
        Gn = G.float().numpy()
        t0 = time.perf_counter()
        HX = factors.factor(Xn)
        t["factors"] += (time.perf_counter() - t0) * (T / t_s) * (n / ns) ** 2
        t0 = time.perf_counter()
        factors.factor(Gn)
        t["factors"] += (time.perf_counter() - t0) * (T / t_s) * (m / ms_) ** 2
        rng = np.random.default_rng(seed)
        for L, nrows in ((n, m + 2 * n), (m, n + 2 * m)):
            R = rng.standard_normal((rows_s, L))
            t0 = time.perf_counter()
            biip.rotate_rows(R, seed, 0)
            t["biip"] += (time.perf_counter() - t0) * (nrows / rows_s)
        Wn = W.float().numpy().astype(np.float64)
        Wt = biip.rotate_rows(Wn, seed, 0)
        HXt = biip.rotate_rows(biip.rotate_rows(HX, seed, 0).T, seed, 0).T
        t0 = time.perf_counter()
        H1, W1, _ = sweep.dead_columns(HXt, Wt)
        A, _ = sweep.damp(H1, 0.01)
        U = sweep.chol_upper_of_inverse(A)
        t["factorisation"] += (time.perf_counter() - t0) * (n / ns) ** 3
        t0 = time.perf_counter()
        res = sweep.gptq_sweep(W1[:sweep_rows], U, bits, group, True, block=1)
        if bits in (2, 4):
            pack.pack(res["codes"], bits)
        t["sweep"] += (time.perf_counter() - t0) * (m / sweep_rows) * (n / ns) ** 2
    total = sum(t.values())
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    sample = (f"oracle (numpy float64) per layer: factors of {t_s} tokens x {d_s} channels, row "
              f"rotations of {rows_s} rows, U at n = {d_s}, sweep of {sweep_rows} rows at n = {d_s}; "
              f"extrapolated to the full layers by operation counts")
    return {"value": weights / total, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": sample, "seconds_per_step": total,
            "phases_s": {k: round(v, 3) for k, v in t.items()}}


def _workload(args):
    wl = dict(WORKLOADS[args.workload])
    if args.bits is not None:
        wl["bits"] = args.bits
    if args.group is not None:
        wl["group"] = args.group
    return wl


def _config(wl, name, world):
    return {"workload": wl["desc"].format(bits=wl["bits"], group=wl["group"]), "name": name,
            "layers": [{"sublayer": s, "m": m, "n": n} for s, m, n, _ in wl["layers"]],
            "tokens": wl["tokens"], "chunk": wl["chunk"], "bits": wl["bits"], "group": wl["group"],
            "accumulate": "f32",
            "l2": "flushed between steps (256 MB write, outside the timed interval); inputs larger than L2",
            "parallelism": f"dp{world} (each rank its own copy of the workload)"}


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    wl = _workload(args)
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(wl, wl["bits"], wl["group"], seed=i, t_s=512, d_s=1024, rows_s=32,
                              sweep_rows=8)
        if i >= args.warmup:
            vals.append(r["seconds_per_step"])
        last = r
    sps = statistics.mean(vals)
    weights = sum(m * n for _, m, n, _ in wl["layers"])
    value = weights / sps
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(wl, args.workload, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm
def _make_layers(wl, dev, rank):
    from post_quantization_kronq_b200.layer import LayerPass
    from synth import llama_layer

    out = []
    for li, (name, m, n, rect) in enumerate(wl["layers"]):
        W, X, G = llama_layer(m, n, wl["tokens"], seed=1000 + 10 * rank + li, device=dev,
                              w_std=wl["w_std"], rectified=rect)
        lp = LayerPass(m, n, bits=wl["bits"], group=wl["group"], seed=rank + li, device=dev)
        out.append((name, W, X, G, lp))
    return out


def _time_steps(layers, chunk, steps, warmup, stream, flush, sampler=None, barrier=None):
    """Runs warmup + steps passes over all layers; returns per-step phase
    times (ms) summed over the layers, and the launches in the timed steps."""
    import torch

    import post_quantization_kronq_b200 as kq

    names = ["accumulate_HX_HG", "sensitivity", "biip_forward", "quantize_and_pack"]

    def step(recs=None):
        for li, (_, W, X, G, lp) in enumerate(layers):
            r = recs[li] if recs else None
            if r:
                r[0].record(stream)
            lp.accumulate(X, G, chunk=chunk)
            if r:
                r[1].record(stream)
            lp.sensitivity()
            if r:
                r[2].record(stream)
            lp.transform(W)
            if r:
                r[3].record(stream)
            lp.quantize()
            if r:
                r[4].record(stream)

    for w in range(warmup):
        flush.zero_()
        step()
        torch.cuda.synchronize()
        for name, _, _, _, lp in layers:
            info = int(lp.info.item())
            assert info == 0, (f"factorisation of {name} reported a non-positive pivot (info {info}) in "
                               f"warm-up step {w}; device status {kq.kronq_device_status()}")
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    recs = [[[ev() for _ in range(5)] for _ in layers] for _ in range(steps)]
    if sampler:
        sampler.start()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    l0 = kq.kronq_launch_count()
    for k in range(steps):
        flush.zero_()
        step(recs[k])
    torch.cuda.synchronize()
    launches = kq.kronq_launch_count() - l0
    if barrier:
        barrier()
    clocks = sampler.stop() if sampler else None
    per_step = []
    for k in range(steps):
        ph = {nm: 0.0 for nm in names}
        for r in recs[k]:
            for i, nm in enumerate(names):
                ph[nm] += r[i].elapsed_time(r[i + 1])
        per_step.append(ph)
    return per_step, launches, clocks


STACK_SUBLAYERS = ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]


def stack_bench(dev, blocks: int = 32, tokens: int = 65536, avg_bits: float = 2.5):
    """The Llama-3-8B-shaped stack (blocks x 7 sublayers, T tokens each) through
    StackPass: the trace-only first pass, the budget allocation over {2, 3, 4}
    at avg_bits, and the per-layer passes at the allocated widths (with the
    built-in trace check).  Only the library calls are timed (CUDA events);
    the synthetic inputs are drawn between them, once per pass."""
    import torch

    from post_quantization_kronq_b200.stack import StackPass
    from synth import LLAMA_SHAPES, llama_layer

    names = [(b, s) for b in range(blocks) for s in STACK_SUBLAYERS]
    shapes = [LLAMA_SHAPES["llama3_8b_" + s] for _, s in names]

    def data(i):
        b, sname = names[i]
        m, n = shapes[i]
        return llama_layer(m, n, tokens, seed=1000 * b + STACK_SUBLAYERS.index(sname), device=dev,
                           rectified=(sname == "down_proj"))

    stream = torch.cuda.current_stream()
    sp = StackPass(shapes, avg_bits=avg_bits, group=128, device=dev)
    t_trace = t_layers = 0.0
    sp.sens1 = []
    for i in range(len(shapes)):
        _, X, G = data(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        sp.sens1.append(sp.trace_one(X, G))
        e1.record(stream)
        torch.cuda.synchronize()
        t_trace += e0.elapsed_time(e1)
        del X, G
    h0 = time.perf_counter()
    bits = sp.allocate()
    t_alloc = (time.perf_counter() - h0) * 1e3
    sp.sens2 = []
    for i in range(len(shapes)):
        W, X, G = data(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lp = sp.quantize_one(i, W, X, G)
        e1.record(stream)
        torch.cuda.synchronize()
        assert int(lp.info.item()) == 0
        t_layers += e0.elapsed_time(e1)
        del W, X, G
    weights = sum(m * n for m, n in shapes)
    total_ms = t_trace + t_alloc + t_layers
    hist = {b: sum(1 for x in bits if x == b) for b in (2, 3, 4)}
    avg = sum(b * m * n for b, (m, n) in zip(bits, shapes)) / weights
    return {"workload": f"llama3-8b stack {blocks} blocks x 7 sublayers, T={tokens} tokens each, "
                        f"inter-layer mixed precision over {{2,3,4}} bits at {avg_bits} average, g128",
            "seconds": total_ms / 1e3, "value": weights / (total_ms / 1e3), "unit": UNIT,
            "phases_ms": {"trace_pass": round(t_trace, 2), "allocation": round(t_alloc, 3),
                          "layer_passes": round(t_layers, 2)},
            "bits_histogram": hist, "average_bits": avg, "trace_check": "passed (1e-3)"}


def run_kronq(args):
    import torch

    import post_quantization_kronq_b200 as kq

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
    wl = _workload(args)
    T, chunk = wl["tokens"], wl["chunk"]
    layers = _make_layers(wl, dev, rank)
    shapes = [(m, n) for _, m, n, _ in wl["layers"]]
    weights = sum(m * n for m, n in shapes)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    per_step, launches, clocks = _time_steps(layers, chunk, args.steps, args.warmup, stream, flush,
                                             ClockSampler(local), barrier)
    step_ms = [sum(p.values()) for p in per_step]
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * weights * args.steps / (total_ms / 1e3)
    phases = {nm: statistics.mean(p[nm] for p in per_step) for nm in per_step[0]}

    peaks = _peaks()
    tpk, hpk, src = choose_peak(peaks, clocks)
    # Roofline of the dominant kernel: the tcgen05 SYRK.  The accumulation
    # phase is SYRK launches only (two factors per layer, one call per token
    # chunk, split into launches by the library's rule); algorithmic flops
    # T d (d + 1) per factor.
    acc_ms = phases["accumulate_HX_HG"]
    flops = sum(T * n * (n + 1) + T * m * (m + 1) for m, n in shapes)
    calls = 1 if chunk is None else -(-T // chunk)
    per_call = T if chunk is None else chunk
    shapes_l = []   # (d, tokens per launch, launches per step)
    for m, n in shapes:
        for d in (n, m):
            k, tl = syrk_launches(d, per_call)
            shapes_l.append((d, tl, k * calls))
    nl = sum(c for _, _, c in shapes_l)
    achieved = flops / (acc_ms / 1e3) / 1e12
    traffic = None
    if all((d, tl) in SYRK_TRAFFIC for d, tl, _ in shapes_l):
        traffic = sum(SYRK_TRAFFIC[(d, tl)] * c for d, tl, c in shapes_l) / nl
    kname = "syrk_pair_kernel" if min(min(m, n) for m, n in shapes) >= 2048 else "syrk_bf16_tc_kernel"
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": tpk,
                "unit": "TFLOP/s", "frac": achieved / tpk, "traffic": traffic,
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean per launch "
                                  "over the step's launch shapes" if traffic else None,
                "peak_source": src, "launches_per_step": nl,
                "flops_per_launch_mean": flops / nl, "launch_ms_mean": acc_ms / nl}
    if peaks:
        roofline["frac_of_burst"] = achieved / peaks["bf16_tflops"]
        roofline["frac_of_sustained"] = achieved / peaks["bf16_tflops_sustained"]

    # The packing kernel on its own (HBM-bound: m n (1 + b/8) bytes per
    # layer), timed with CUDA events over repeated calls on the step's codes
    # (larger than L2).
    kernel_rooflines = {}
    pk_ms = pk_bytes = 0.0
    for _, _, _, _, lp in layers:
        if lp.packed is None:
            continue
        kq.kronq_pack(lp.codes, lp.bits, lp.packed, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record(stream)
        for _ in range(reps):
            kq.kronq_pack(lp.codes, lp.bits, lp.packed, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        pk_ms += e0.elapsed_time(e1) / reps
        pk_bytes += lp.m * lp.n * (1 + lp.bits / 8)
    if pk_ms > 0:
        gbs = pk_bytes / (pk_ms / 1e3) / 1e9
        kernel_rooflines["pack_kernel"] = {"bound": "hbm", "achieved": gbs, "peak": hpk, "unit": "GB/s",
                                           "frac": gbs / hpk, "bytes_per_step": pk_bytes,
                                           "ms_per_step": pk_ms,
                                           "peak_source": "measured hbm_gbs" if peaks else "fallback"}

    # End to end through the public API: inputs copied from pinned host memory
    # every step, packed codes, scales and zeros copied back.
    e2e = None
    if not args.no_e2e:
        host = []
        h2d = d2h = 0
        for _, W, X, G, lp in layers:
            hX = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
            hG = torch.empty(G.shape, dtype=G.dtype, pin_memory=True)
            hW = torch.empty(W.shape, dtype=W.dtype, pin_memory=True)
            hX.copy_(X)
            hG.copy_(G)
            hW.copy_(W)
            outs = [lp.packed if lp.packed is not None else lp.codes, lp.scales, lp.zeros]
            houts = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
            h2d += sum(t.numel() * t.element_size() for t in (hX, hG, hW))
            d2h += sum(t.numel() * t.element_size() for t in houts)
            host.append((hX, hG, hW, outs, houts))

        def e2e_step():
            # token chunks of X and G copied on each layer's copy stream while
            # the factor accumulation of the earlier chunks runs
            for (_, W, X, G, lp), (hX, hG, hW, outs, houts) in zip(layers, host):
                lp.run_from_host(hX, hG, hW, X, G, W, chunk=chunk or 16384, stream=stream)
                for h, o in zip(houts, outs):
                    h.copy_(o, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e_steps = max(2, min(args.steps, 5))
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
        e2e = {"value": world * weights * e_steps / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "pipeline": "X, G copied in 16384-token chunks on a second stream per layer, "
                           "overlapping the factor accumulation and the other layers' passes"}
        del host

    sens = [lp.sens for _, _, _, _, lp in layers]
    del layers
    torch.cuda.empty_cache()

    also = None
    if not args.no_also and args.workload != "llama2_7b_q_proj":
        also = {}
        for b in (2, 4):
            wq = dict(WORKLOADS["llama2_7b_q_proj"])
            wq["bits"] = b
            lq = _make_layers(wq, dev, rank)
            ps, ln, _ = _time_steps(lq, wq["chunk"], args.steps, args.warmup, stream, flush)
            tms = sum(sum(p.values()) for p in ps)
            if dist is not None:
                t = torch.tensor([tms], dtype=torch.float64, device=dev)
                dist.all_reduce(t, op=dist.ReduceOp.MAX)
                tms = float(t.item())
            ph = {nm: statistics.mean(p[nm] for p in ps) for nm in ps[0]}
            fl = wq["tokens"] * 4096 * 4097 * 2
            also[f"llama2_7b_q_proj_w{b}"] = {
                "workload": wq["desc"].format(bits=b, group=wq["group"]),
                "value": world * 4096 * 4096 * args.steps / (tms / 1e3), "unit": UNIT,
                "ms_per_step": tms / args.steps, "gpu_launches": ln,
                "phases_ms": {k: round(v, 4) for k, v in ph.items()},
                "syrk_tflops": fl / (ph["accumulate_HX_HG"] / 1e3) / 1e12,
                "phase_roofline": phase_rooflines(ph, [(4096, 4096)], wq["tokens"], tpk, hpk, src)}
            del lq
            torch.cuda.empty_cache()

    if also is not None and not args.no_stack:
        also["llama3_8b_stack"] = stack_bench(dev)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_sample(wl, wl["bits"], wl["group"])
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
        "config": _config(wl, args.workload, world),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": launches,
        "phases_ms": {k: round(v, 4) for k, v in phases.items()},
        "phase_roofline": phase_rooflines(phases, shapes, T, tpk, hpk, src),
        "kernel_roofline": kernel_rooflines,
        "sensitivity": sens, "also": also,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kronq", "reference"], default="kronq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3_70b_mlp")
    ap.add_argument("--bits", type=int, default=None, choices=[2, 3, 4])
    ap.add_argument("--group", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.impl == "reference":
        return run_reference(args)
    return run_kronq(args)


if __name__ == "__main__":
    sys.exit(main())
