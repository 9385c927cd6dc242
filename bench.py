#!/usr/bin/env python
"""Benchmark of the sparse MoE layer forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
                    [--experts bf16|e4m3|fp4|w4a16|w4a4] [--ep W]

A step is one moe_forward over one batch: router, top-K, softmax, dispatch,
gather, GEMM1 (w1/w3 + SwiGLU), GEMM2 (w2), combine.  The default workload is
the largest single-GPU one, the skewed-routing Mixtral-shape prefill layer
(T=16384, d=4096, ffn=14336, n=8, K=2, bf16; about 44% of the routed rows on
expert 0), whose grouped GEMMs are bound by the bf16 tensor cores; --config
picks another of the five (tiny_fp32, decode, prefill, skew_prefill,
many_expert).  Inputs are seeded synthetic data resident in HBM before the
timed region; the expert weights (>= 1.2 GB) are larger than the 126 MB L2,
so no flush is needed between steps (tiny_fp32 flushes L2 with a 256 MB write).

`value` is tokens/s over all ranks (replicas: each rank runs the same
workload on its own GPU; no collective on the data path), timed with CUDA
events on the launching stream, max over ranks.  `e2e` is the same metric
through the C ABI with every step's activations copied from pinned host memory
and its y / topk_idx / topk_w copied back inside the timed region; the copies
run on two copy streams with double buffers, overlapping the neighbouring
steps' layers.  `roofline`
reports the dominant kernel, timed by the library's per-stage CUDA events over
a second run of the same K steps (events between the kernels would serialise
their programmatic dependent launches in the headline run).  `cpu_baseline` times the fp64 oracle on a bounded
sample of the same workload on this host's cores.

--experts e4m3 times moe_forward_e4m3 instead: the same layer with FP8 (E4M3)
expert weights (per-column scales, quantised once before the timed region)
and per-row E4M3 activations; --experts fp4 times moe_forward_fp4: 4-bit
(E2M1) expert weights with E4M3 scales per 16 rows and bf16 activations (bf16
handle and workloads only); --experts w4a16 times moe_forward_w4a16: the same
layer on weights packed once by moe_pack_weights_w4a16, which the GEMMs decode
straight into tensor memory; --experts w4a4 times moe_forward_w4a4: the same
4-bit weights with 4-bit activations on the block-scaled tensor cores (d and
ffn multiples of 256).

--ep W times one expert-parallel step with W ranks emulated on this GPU (n/W
experts per rank, the tokens split over the ranks; the exchange is the
kernels' own stores and loads, here into this GPU's memory).

--impl reference runs the oracle (the reference arm: a plain fp64 CPU layer) on the
host, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_desc(cfg, experts="bf16"):
    return "%s: T=%d, d=%d, ffn=%d, n=%d, K=%d, %s%s%s" % (
        cfg.name, cfg.T, cfg.d, cfg.ffn, cfg.n, cfg.K, cfg.dtype, ", skewed router" if cfg.skew else "",
        {"e4m3": ", E4M3 experts", "fp4": ", 4-bit (E2M1) experts",
         "w4a16": ", 4-bit (E2M1) experts decoded into tensor memory",
         "w4a4": ", 4-bit (E2M1) experts and activations"}.get(experts, ""))


# --------------------------------------------------------------------------
# algorithmic work per launch: what each stage must read, write and compute
# --------------------------------------------------------------------------

def touched_experts(idx: np.ndarray, n: int) -> np.ndarray:
    return np.bincount(idx.ravel(), minlength=n)


def algorithmic(cfg, counts, experts="bf16"):
    """Bytes and FLOPs each stage must move / do, from the routing of the step.
    E4M3 experts: one byte per weight plus its column's fp32 scale; the gemm2
    stage also holds the hidden-row quantisation (bf16 H read, codes written)."""
    es = 2 if cfg.dtype == "bf16" else 4
    T, d, F, n, K = cfg.T, cfg.d, cfg.ffn, cfg.n, cfg.K
    R = T * K
    used = int((counts > 0).sum())
    if experts in ("fp4", "w4a16"):
        # codes 0.5 B + block scale 1/16 B per weight; gather, H and O in bf16
        w13 = used * 2 * (d * F // 2 + d * F // 16 + 4)
        w2 = used * (F * d // 2 + F * d // 16 + 4)
        gemm1_bytes = w13 + R * d * es + R * F * es
        gemm2_bytes = w2 + R * F * es + R * d * es
    elif experts == "w4a4":
        # weights as fp4; A operands as 4-bit codes + scales; the gemm2 stage
        # also holds the hidden-row quantisation (bf16 H read, codes written)
        w13 = used * 2 * (d * F // 2 + d * F // 16 + 4)
        w2 = used * (F * d // 2 + F * d // 16 + 4)
        hq = R * F * es + R * (F // 2 + F // 16 + 4)
        gemm1_bytes = w13 + R * (d // 2 + d // 16 + 4) + R * F * es
        gemm2_bytes = hq + w2 + R * (F // 2 + F // 16 + 4) + R * d * es
    elif experts == "e4m3":
        w13 = used * 2 * (d * F + F * 4)
        w2 = used * (F * d + d * 4)
        gemm1_bytes = w13 + R * (d + 4) + R * F * 2
        gemm2_bytes = (R * F * 2 + R * (F + 4)) + w2 + R * (F + 4) + R * d * es
    else:
        w13 = used * 2 * d * F * es
        w2 = used * F * d * es
        gemm1_bytes = w13 + R * d * es + R * F * es           # weights + Xp read + H write
        gemm2_bytes = w2 + R * F * es + R * d * es             # weights + H read + O write
    gemm1_flops = 4.0 * R * d * F
    gemm2_flops = 2.0 * R * F * d
    return {
        "gemm1": {"bytes": gemm1_bytes, "flops": gemm1_flops},
        "gemm2": {"bytes": gemm2_bytes, "flops": gemm2_flops},
        "layer_bytes": w13 + w2 + T * d * es * 2 + d * n * 4,
        "active_flops": 6.0 * R * d * F + 2.0 * T * d * n,
        "experts_touched": used,
    }


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel, config):
    """dram read+write bytes per launch from a committed ncu summary, if that
    summary was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    default_file = {"_w4a4": "gemm_w4a4.cu", "_w4a16": "gemm_w4a16.cu", "_fp4": "gemm_fp4.cu"}.get(
        config[config.rfind("_"):], "gemm_tc.cu")
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 5 and parts[0] == "traffic" and parts[1] == kernel and parts[2] == config:
                # an optional file=<name> names the kernel's source (else by the config)
                src_file = next((t[5:] for t in parts[5:] if t.startswith("file=")), default_file)
                sha = source_sha(os.path.join(ROOT, "sparse_mixture_experts_24_b200", "csrc", src_file))
                if parts[4] == "src_sha=" + sha:
                    return float(parts[3])
    return None


# --------------------------------------------------------------------------
# replicas: each rank runs the whole workload on its own GPU and its own batch
# --------------------------------------------------------------------------

def replica_seed(rank: int) -> int:
    return rank


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank timing over all ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(T: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processed T tokens per step."""
    return T * world / (ms_per_step * 1e-3)


# --------------------------------------------------------------------------
# clocks sampled during the timed region (NVML)
# --------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:  # the CUDA device's own NVML handle (indices differ under CUDA_VISIBLE_DEVICES)
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self._reasons_fn(self.h)
                for k, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the workload
# --------------------------------------------------------------------------

def oracle_tokens_per_s(cfg, L, budget_s=12.0, experts="bf16"):
    """The oracle on the first tokens of the workload, repeated until about
    budget_s of host time (a bounded sample of the same layer).  E4M3 experts:
    the oracle's router and E4M3 layer, on codes it quantised beforehand
    (untimed)."""
    import oracle
    threads = oracle.num_threads()
    if experts == "e4m3":
        q = [a for w in ("w1", "w3", "w2") for a in oracle.quantize_weights_e4m3(L[w])]

        def layer(xs):
            i, g, _ = oracle.router(xs, L["W_g"], cfg.K)
            oracle.forward_e4m3(xs, i, g, *q)
    elif experts in ("fp4", "w4a16", "w4a4"):
        q4 = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
        fwd = oracle.forward_w4a4 if experts == "w4a4" else oracle.forward_fp4

        def layer(xs):
            i, g, _ = oracle.router(xs, L["W_g"], cfg.K)
            fwd(xs, i, g, *q4)
    else:
        def layer(xs):
            oracle.moe_forward(xs, L["W_g"], L["w1"], L["w3"], L["w2"], cfg.K)
    t0 = time.perf_counter()
    layer(L["x"][:1])
    one = max(time.perf_counter() - t0, 1e-6)
    # tokens per repetition: enough to keep every thread busy, within budget
    s = int(max(1, min(cfg.T, max(threads, budget_s * threads / one / 4))))
    done, reps = 0, 0
    t0 = time.perf_counter()
    while True:
        layer(L["x"][:s])
        done += s
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    return done / el, s, reps, min(threads, s), el


# --------------------------------------------------------------------------
# reference arm: the oracle on the host
# --------------------------------------------------------------------------

def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    L = mi.make_layer(cfg, seed=0)
    threads = oracle.num_threads()
    # per-step sample sized so that warmup + steps finish in about two minutes
    t0 = time.perf_counter()
    oracle.moe_forward(L["x"][:1], L["W_g"], L["w1"], L["w3"], L["w2"], cfg.K)
    one = max(time.perf_counter() - t0, 1e-6)
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    s = int(max(1, min(cfg.T, per_step_budget * max(1, threads) / one)))
    for i in range(args.warmup):
        oracle.moe_forward(L["x"][:s], L["W_g"], L["w1"], L["w3"], L["w2"], cfg.K)
    t0 = time.perf_counter()
    for i in range(args.steps):
        lo = (i * s) % max(1, cfg.T - s + 1)
        oracle.moe_forward(L["x"][lo:lo + s], L["W_g"], L["w1"], L["w3"], L["w2"], cfg.K)
    el = time.perf_counter() - t0
    v = s * args.steps / el
    line = {
        "impl": "reference", "metric": "MoE-layer tokens/s", "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "sample_tokens_per_step": s},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": min(threads, s), "kind": "oracle",
                         "sample": "%d of %d tokens per step, full layer (router + %d experts each)"
                                   % (s, cfg.T, cfg.K)},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def run_ep(args, cfg):
    """--ep W: one expert-parallel layer step of W ranks emulated on this GPU
    (the workload's T tokens split over the ranks, n/W experts each; every
    phase runs for all ranks before the next, as the barriers order them
    across GPUs).  The exchange is the kernels' peer stores and loads, here
    into this GPU's memory, so the number measures the kernels, not NVLink."""
    import torch
    import sparse_mixture_experts_24_b200 as m
    from sparse_mixture_experts_24_b200.ep import EmulatedExpertParallel
    W = args.ep
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 or args.gpus != 1:
        raise SystemExit("--ep emulates its ranks on one GPU: run it with --gpus 1")
    if cfg.dtype != "bf16" or args.experts != "bf16" or W < 1 or cfg.n % W:
        raise SystemExit("--ep needs a bf16 workload with bf16 experts and W dividing n")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L = mi.make_layer(cfg, seed=replica_seed(0))

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.to(dev)

    x, Wg, w1, w3, w2 = (to_dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2"))
    T, n, K = cfg.T, cfg.n, cfg.K
    bounds = [T * r // W for r in range(W + 1)]
    xs = [x[bounds[r]:bounds[r + 1]] for r in range(W)]
    nl = n // W
    weights = [tuple(t[q * nl:(q + 1) * nl] for t in (w1, w3, w2)) for q in range(W)]
    ep = EmulatedExpertParallel(n, K, cfg.d, cfg.ffn, W, T * K)
    ys = [torch.empty_like(xr) for xr in xs]
    stream = torch.cuda.current_stream(dev)

    def step(mark=None):
        return ep.forward(xs, Wg, weights, ys, mark=mark)

    for _ in range(args.warmup):
        _, idxs, _ = step()
    ep.sync_status()
    counts = touched_experts(torch.cat(idxs).cpu().numpy(), n)

    sampler = ClockSampler(dev.index)
    torch.cuda.synchronize(dev)
    launches0 = ep.launch_count()
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    launches = ep.launch_count() - launches0
    ms = ev0.elapsed_time(ev1) / args.steps
    ep.sync_status()

    # the same steps with an event after each phase
    names = ("route", "dispatch", "experts", "combine")
    acc = [0.0] * 4
    for _ in range(args.steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        evs[0].record(stream)
        step(mark=lambda i: evs[i + 1].record(stream))
        torch.cuda.synchronize(dev)
        for i in range(4):
            acc[i] += evs[i].elapsed_time(evs[i + 1])
    phase_ms = {k: a / args.steps for k, a in zip(names, acc)}

    # end to end: x from pinned host memory in, y back, every step
    xh = x.cpu().pin_memory()
    yh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    xd = torch.empty_like(x)
    xds = [xd[bounds[r]:bounds[r + 1]] for r in range(W)]
    yd = torch.empty_like(x)
    yds = [yd[bounds[r]:bounds[r + 1]] for r in range(W)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        xd.copy_(xh, non_blocking=True)
        ep.forward(xds, Wg, weights, yds)
        yh.copy_(yd, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ems = e0.elapsed_time(e1) / args.steps
    same = bool(torch.equal(yh, torch.cat(ys).cpu()))

    peaks, peak_src = load_peaks()
    work = algorithmic(cfg, counts, "bf16")
    flops = work["gemm1"]["flops"] + work["gemm2"]["flops"]
    nbytes = work["gemm1"]["bytes"] + work["gemm2"]["bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    t_exp = phase_ms["experts"] * 1e-3
    if flops / nbytes < ridge:
        ach = nbytes / t_exp / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "algorithmic_per_launch": nbytes}
    else:
        pk = peaks["bf16_tflops_sustained"] if ms * args.steps > 1000 else peaks["bf16_tflops"]
        ach = flops / t_exp / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                "algorithmic_per_launch": flops}
    roof.update({"kernel": "experts phase of all ranks (plan + GEMM1 + GEMM2 per rank)",
                 "peak_source": peak_src, "launch_ms": phase_ms["experts"], "traffic": None})
    cpu = None
    if not args.no_cpu_baseline:
        v, smp, reps, cores, el = oracle_tokens_per_s(cfg, L)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": "first %d of %d tokens x %d repetitions, full layer in fp64 (%.1f s)" % (smp, T, reps, el)}
    line = {
        "metric": "MoE-layer tokens/s", "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(cfg) + "; expert-parallel, %d ranks emulated on one GPU" % W,
                   "global_batch_tokens": T, "parallelism": "ep%d emulated on 1 GPU" % W,
                   "l2": "no flush: %.2f GB of expert weights per step > 126 MB L2" % (work["layer_bytes"] / 1e9)},
        "phase_ms_per_step": {k: round(v, 5) for k, v in phase_ms.items()},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": T / (ems * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": x.numel() * 2,
                "d2h_bytes_per_step": x.numel() * 2, "outputs_match_device_run": same},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line))
    ep.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="skew_prefill", choices=sorted(mi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", default="bf16", choices=["bf16", "e4m3", "fp4", "w4a16", "w4a4"])
    ap.add_argument("--ep", type=int, default=0,
                    help="expert parallelism with this many ranks, emulated on one GPU")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = mi.CONFIGS[args.config]
    if args.ep:
        return run_ep(args, cfg)
    if args.experts != "bf16" and cfg.dtype != "bf16":
        ap.error("--experts %s needs a bf16 workload" % args.experts)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import sparse_mixture_experts_24_b200 as m

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)

    L = mi.make_layer(cfg, seed=replica_seed(rank))  # each replica gets its own seeded batch
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.to(dev)

    x, Wg, w1, w3, w2 = (to_dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2"))
    T = cfg.T
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, cfg.dtype)
    layer.reserve(T)
    y = torch.empty_like(x)
    idx = torch.empty((T, cfg.K), dtype=torch.int32, device=dev)
    gw = torch.empty((T, cfg.K), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if cfg.name == "tiny_fp32" else None
    e4m3 = args.experts == "e4m3"
    fp4 = args.experts == "fp4"
    w4a16 = args.experts == "w4a16"
    w4a4 = args.experts == "w4a4"
    if e4m3 or fp4 or w4a16 or w4a4:
        # quantised once, outside the timed region; the bf16 copies are freed
        quant = m.quantize_weights_e4m3 if e4m3 else m.quantize_weights_fp4
        if w4a4:
            # the gate/up pair pack of w1 and w3, then w2
            q = list(m.pack_weights_w4a4(*m.quantize_weights_fp4(w1), pair=m.quantize_weights_fp4(w3)))
            q += list(m.pack_weights_w4a4(*m.quantize_weights_fp4(w2)))
        elif w4a16:
            q = list(m.pack_weights_w4a16(*m.quantize_weights_fp4(w1), pair=m.quantize_weights_fp4(w3)))
            q += list(m.pack_weights_w4a16(*m.quantize_weights_fp4(w2)))
        else:
            q = [t for w in (w1, w3, w2) for t in quant(w)]
        torch.cuda.synchronize(dev)
        del w1, w3, w2
        torch.cuda.empty_cache()

    def forward(xin, yout=None, iout=None, wout=None):
        yout = y if yout is None else yout
        iout = idx if iout is None else iout
        wout = gw if wout is None else wout
        if e4m3:
            m.moe_forward_e4m3(layer.h, T, xin, Wg, *q, yout, iout, wout, stream)
        elif fp4:
            m.moe_forward_fp4(layer.h, T, xin, Wg, *q, yout, iout, wout, stream)
        elif w4a16:
            m.moe_forward_w4a16(layer.h, T, xin, Wg, *q, yout, iout, wout, stream)
        elif w4a4:
            m.moe_forward_w4a4(layer.h, T, xin, Wg, *q, yout, iout, wout, stream)
        else:
            m.moe_forward(layer.h, T, xin, Wg, w1, w3, w2, yout, iout, wout, stream)

    def step():
        if flush is not None:
            flush.fill_(1)
        forward(x)

    for _ in range(args.warmup):
        step()
    layer.sync_status(stream)
    counts = touched_experts(idx.cpu().numpy(), cfg.n)

    # ---- device-timed region (no per-stage events: they would sit between
    # the layer's kernels and serialise their programmatic dependent launches)
    sampler = ClockSampler(dev.index)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = m.moe_launch_count(layer.h)
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    launches = m.moe_launch_count(layer.h) - launches0
    if dist:
        dist.barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    layer.sync_status(stream)
    ms = max_over_ranks(ms, dist, dev)
    value = tokens_per_s(T, world, ms)

    # ---- the same K steps again with the library's per-stage CUDA events,
    # which time each kernel (the roofline's launch duration)
    torch.cuda.synchronize(dev)
    m.moe_trace_begin(layer.h, args.steps)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize(dev)
    stage_ms, traced = m.moe_trace_end(layer.h)
    layer.sync_status(stream)

    # ---- end to end: pinned host activations in, y / routing out ----
    # Every step copies its x from pinned host memory and its y, topk_idx and
    # topk_w back.  The copies run on their own streams with two buffer sets,
    # so step i+1's upload and step i's download overlap step i's layer (a
    # copy engine per direction); events keep each buffer's uses in order.
    xh = x.cpu().pin_memory()
    NB = 2
    xd = [torch.empty_like(x) for _ in range(NB)]
    yd = [torch.empty_like(y) for _ in range(NB)]
    idd = [torch.empty_like(idx) for _ in range(NB)]
    gwd = [torch.empty_like(gw) for _ in range(NB)]
    yh = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(NB)]
    ih = [torch.empty(idx.shape, dtype=idx.dtype).pin_memory() for _ in range(NB)]
    wh = [torch.empty(gw.shape, dtype=gw.dtype).pin_memory() for _ in range(NB)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(NB)]
    ev_layer = [torch.cuda.Event() for _ in range(NB)]
    ev_down = [torch.cuda.Event() for _ in range(NB)]
    step_no = [0]

    def e2e_step():
        b = step_no[0] % NB
        step_no[0] += 1
        s_up.wait_event(ev_layer[b])          # the layer two steps back has read xd[b]
        with torch.cuda.stream(s_up):
            xd[b].copy_(xh, non_blocking=True)
        ev_up[b].record(s_up)
        stream.wait_event(ev_up[b])
        stream.wait_event(ev_down[b])         # yd[b] etc. were read back two steps ago
        if flush is not None:
            flush.fill_(1)
        forward(xd[b], yd[b], idd[b], gwd[b])
        ev_layer[b].record(stream)
        s_down.wait_event(ev_layer[b])
        with torch.cuda.stream(s_down):
            yh[b].copy_(yd[b], non_blocking=True)
            ih[b].copy_(idd[b], non_blocking=True)
            wh[b].copy_(gwd[b], non_blocking=True)
        ev_down[b].record(s_down)

    for _ in range(args.warmup):
        e2e_step()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_up.wait_event(e0)
    s_down.wait_event(e0)
    for _ in range(args.steps):
        e2e_step()
    for b in range(NB):
        stream.wait_event(ev_down[b])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ems = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
    e2e_value = tokens_per_s(T, world, ems)
    # the copied-back outputs of the last step equal the device-timed run's
    # (same input, deterministic kernels)
    last = (step_no[0] - 1) % NB
    e2e_same = bool(torch.equal(yh[last], y.cpu()) and torch.equal(ih[last], idx.cpu()))
    h2d = x.numel() * x.element_size()
    d2h = y.numel() * y.element_size() + idx.numel() * 4 + gw.numel() * 4

    # ---- roofline of the dominant kernel ----
    peaks, peak_src = load_peaks()
    work = algorithmic(cfg, counts, args.experts)
    per_launch = {k: v / max(1, traced) for k, v in stage_ms.items()}
    dom = max(("gemm1", "gemm2"), key=lambda k: per_launch[k])
    dom_ms = per_launch[dom]
    if cfg.dtype == "f32":
        roof = None
    else:
        intensity = work[dom]["flops"] / work[dom]["bytes"]
        ratio = 2.0 if e4m3 else (4.0 if w4a4 else 1.0)   # dense fp8 / fp4 rate over bf16 (4.5, 9 vs 2.25 PF)
        ridge = peaks["bf16_tflops"] * ratio * 1e12 / (peaks["hbm_gbs"] * 1e9)
        if intensity < ridge:
            ach = work[dom]["bytes"] / (dom_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"]}
        else:
            timed_s = ms * args.steps * 1e-3
            pk = peaks["bf16_tflops_sustained"] if timed_s > 1.0 else peaks["bf16_tflops"]
            pk *= ratio
            ach = work[dom]["flops"] / (dom_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                    "peak_kind": "sustained" if timed_s > 1.0 else "burst"}
        roof["kernel"] = dom
        roof["peak_source"] = peak_src
        roof["algorithmic_per_launch"] = work[dom]["bytes"] if roof["bound"] == "hbm" else work[dom]["flops"]
        roof["launch_ms"] = dom_ms
        roof["traffic"] = recorded_traffic(dom, cfg.name + {"e4m3": "_e4m3", "fp4": "_fp4", "w4a16": "_w4a16",
                                                           "w4a4": "_w4a4"}.get(
            args.experts, ""))

    # ---- CPU baseline (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, s, reps, cores, el = oracle_tokens_per_s(cfg, L, experts=args.experts)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": "first %d of %d tokens x %d repetitions, full layer in fp64%s (%.1f s)"
                         % (s, cfg.T, reps, {"e4m3": ", E4M3 experts", "fp4": ", 4-bit experts",
                                             "w4a16": ", 4-bit experts",
                                             "w4a4": ", 4-bit experts and activations"}.get(args.experts, ""),
                            el)}

    if rank == 0:
        layer_ms = ms
        line = {
            "metric": "MoE-layer tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if e4m3 else ("e2m1 weights, bf16" if (fp4 or w4a16) else ("e2m1" if w4a4 else cfg.dtype)),
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg, args.experts), "global_batch_tokens": T * world,
                       "parallelism": "replicas%d" % world if world > 1 else "single",
                       "l2": "256 MB flush per step" if flush is not None else
                             "no flush: %.2f GB of expert weights per step > 126 MB L2"
                             % (work["layer_bytes"] / 1e9)},
            "active_tflops": work["active_flops"] / (layer_ms * 1e-3) / 1e12,
            "hbm_gbs_over_bytes_touched": work["layer_bytes"] / (layer_ms * 1e-3) / 1e9,
            "stage_ms_per_step": {k: round(v, 5) for k, v in per_launch.items()},
            "experts_touched": work["experts_touched"],
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "outputs_match_device_run": e2e_same},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        print(json.dumps(line))
    layer.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
