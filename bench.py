#!/usr/bin/env python
"""Benchmark of the routed-expert MoE decode layer on B200.

Metric: MoE-layer decode tokens/s, with the effective expert-weight HBM GB/s
(and its fraction of HBM peak) for the full-size 4-bit top-4 layer: hidden 4096,
expert intermediate 1024, 512 routed experts + 1 shared, 1000 tokens with
independent seeded activations.  One step = the 1000 tokens, each a single-token
fmoe_layer_forward call (one fused kernel launch), the 1000 launches replayed
from one CUDA graph.  Weights (3.64 GB) are resident in HBM; the L2 is flushed
between steps.

The default single-GPU run adds sub-records for the layer stacks (24 layers of
4-bit, 60 layers of 2-bit, 16 layers of batched top-10 decode), each with its own
roofline, clocks and CPU-oracle sample.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--config NAME]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (the layer has no exchange step): value = tokens of all
ranks / max over ranks of the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_NOMINAL_GBS = 8000.0
METRIC = "MoE-layer decode tokens/s; expert-weight HBM GB/s (% of ~8 TB/s), 4-bit K=4"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fmoe", choices=["fmoe", "reference"])
    ap.add_argument("--config", default="layer4096")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--cpu-sample", type=int, default=6,
                    help="tokens timed once for the CPU oracle baseline of the GPU arm")
    ap.add_argument("--sub-steps", type=int, default=3, help="timed steps of each stack sub-record")
    ap.add_argument("--no-sub", action="store_true", help="skip the stack sub-records of the default run")
    ap.add_argument("--ref-tokens", type=int, default=1,
                    help="tokens per step of the reference arm (the CPU oracle)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["gdn", "tier"], default=None,
                    help="run one sub-record's workload alone and print it as the line")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


KERNEL_SOURCES = ("fmoe_layer.cuh", "fmoe_device.cuh", "fmoe_topk.cuh")


def kernel_source_digest(texts) -> str:
    """sha256 of the layer kernel's sources with comments and whitespace removed (a
    change to a comment does not change the kernel the counters were taken from)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for t in texts:
        t = re.sub(r"/\*.*?\*/", " ", t, flags=re.S)
        t = re.sub(r"//[^\n]*", " ", t)
        h.update(" ".join(t.split()).encode())
    return h.hexdigest()


def profiled_traffic(key: str = "traffic_bytes_per_launch", summary: str = "fmoe_layer_kernel_layer4096.md",
                     sources=None):
    """DRAM bytes per launch of a kernel (`key`) from a committed ncu summary, if the
    kernel's sources (default: the layer kernel's) are the ones that were profiled
    (else None)."""
    texts = []
    for f in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_dequant_expert_softmax_b200", "csrc", f)) as fh:
            texts.append(fh.read())
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    want, traffic = None, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line.startswith("kernel_source_digest:"):
                want = line.split(":", 1)[1].strip()
            elif line.startswith(key + ":"):
                traffic = int(line.split(":", 1)[1].strip())
    return traffic if want == kernel_source_digest(texts) else None


def max_over_ranks(value: float, world: int, device="cuda") -> float:
    """The largest of every rank's `value` (the timed region of a multi-rank run is the
    slowest rank's); every rank must call it, in the same order."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (slowest_ms / 1e3)


def layer_bytes(shape):
    """Algorithmic bytes of one single-token layer forward."""
    import fmoe_synth as synth
    rb = synth.record_bytes(shape.hidden, shape.inter, shape.bits)
    experts = (shape.top_k + shape.has_shared) * rb
    router = shape.n_experts * shape.hidden * 4 + (shape.hidden * 4 if shape.has_shared else 0)
    io = 3 * shape.hidden * 2
    return experts, router + io


def cpu_oracle_rates(shape, n_tokens: int, block: bool = False, seed: int = 0, t0: int = 0, single: bool = True):
    """The fp64 oracle (as it stands) on n_tokens tokens of the workload, timed twice:
    with the BLAS thread pool limited to one thread, and with its default size (all
    host cores).  block=True times pre-norm blocks (RMSNorm + layer), the unit of the
    stacks.  Expert records are regenerated before each token's timed forward, which
    then runs from the packed bytes (the decode of the records is timed).  Returns
    {"single": tokens/s, "all": tokens/s, "threads_all": BLAS threads, "cores": nproc}."""
    import fmoe_synth as synth
    import oracle
    olay = oracle.synthetic_layer(seed, 0, shape, lazy=True)
    tokens = []
    cache = {}
    for t in range(n_tokens):
        x = oracle.bf16_to_f64(synth.gen_x_token(seed, t0 + t, shape.hidden))
        xin = oracle.bf16_to_f64(oracle.rmsnorm_bf16(x)) if block else x
        idx, _, _, _ = olay.route(xin)
        for e in list(idx) + ([shape.n_experts] if shape.has_shared else []):
            if int(e) not in cache:
                cache[int(e)] = synth.gen_record(seed, 0, int(e), shape.hidden, shape.inter, shape.bits)
        tokens.append(x)

    def timed():
        total = 0.0
        for x in tokens:
            olay._cache = {}
            olay._records = lambda e, _r=cache: _r[e]
            t_start = time.perf_counter()
            if block:
                oracle.block_forward(olay, x)
            else:
                olay.forward(x)
            total += time.perf_counter() - t_start
        return n_tokens / total

    threads_all, one = 1, None
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        threads_all = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        if single:
            with threadpool_limits(limits=1):
                one = timed()
    except ImportError:  # without threadpoolctl only the default pool is timed
        pass
    return {"single": one, "all": timed(), "threads_all": threads_all, "cores": os.cpu_count()}


def cpu_baseline_line(rates, unit_scale: float, unit: str, sample: str):
    """The bench line's cpu_baseline object: the all-core rate is the value (times
    unit_scale, e.g. 1/L for an L-layer stack), the single-thread one beside it."""
    return {"value": rates["all"] * unit_scale, "unit": unit, "cores": rates["cores"], "kind": "oracle",
            "threads": rates["threads_all"],
            "single_thread_value": None if rates["single"] is None else rates["single"] * unit_scale,
            "sample": sample}


def run_reference(args, rank):
    """The reference arm: the fp64 CPU oracle, timed on the host cores."""
    import fmoe_synth as synth
    if rank != 0:
        return
    shape = synth.CONFIGS[args.config]["shape"]
    per_step = max(1, args.ref_tokens)
    t_all = 0.0
    tok = 0
    threads = 1
    for i in range(args.steps):
        rates = cpu_oracle_rates(shape, per_step, t0=i * per_step, single=False)
        threads = rates["threads_all"]
        t_all += per_step / rates["all"]
        tok += per_step
    value = tok / t_all
    desc = f"{per_step} tokens of the {shape.hidden}x{shape.inter} layer"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t_all / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.config}: single-token decode, hidden {shape.hidden}, "
                                   f"inter {shape.inter}, {shape.n_experts}+{shape.has_shared} experts, "
                                   f"top-{shape.top_k}, {shape.bits}-bit",
                       "tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": os.cpu_count(), "threads": threads,
                             "kind": "oracle", "sample": f"{per_step} tokens per step ({desc})"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_stack(args, world, rank, config, steps, warmup, cpu_tokens):
    """A layer stack (pre-norm blocks) decoding its token set through the captured
    graph: token after token (batch 1) or in steps of `batch` tokens on the batched
    path.  One step = every token of the set through every layer.  Returns the bench
    line (rank 0; None elsewhere)."""
    import torch
    import torch.distributed as dist

    import fmoe_synth as synth
    from bit_dequant_expert_softmax_b200 import fmoe
    from fmoe_synth.torch_layer import make_device_layer, make_device_x

    cfg_d = synth.CONFIGS[config]
    shape, NL, B = cfg_d["shape"], cfg_d["layers"], cfg_d["batch"]
    tokens = args.tokens or cfg_d["tokens"]
    H = shape.hidden
    cfg = fmoe.fmoe_config(H, shape.inter, shape.n_experts, shape.top_k, shape.bits, shape.has_shared,
                           shape.router_bias)
    layers = []
    for l in range(NL):
        w = make_device_layer(shape, 0, l)
        L = fmoe.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
        if B > 1:
            L.attach_batch(B)
        layers.append(L)
    stack = fmoe.Stack(layers, 1e-6)
    h0 = make_device_x(0, rank * tokens, tokens, H)
    h = h0.clone()
    graph = stack.graph(h, batch=B)
    stream = torch.cuda.Stream()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(max(3, warmup)):
            h.copy_(h0)
            graph.launch(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    with torch.cuda.stream(stream):
        for i in range(steps):
            h.copy_(h0)           # every step decodes the same token set
            flush.fill_(i & 0xFF)  # L2 flush (outside the timed events)
            starts[i].record(stream)
            graph.launch(stream)
            ends[i].record(stream)
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    errs = [L.error() for L in layers]
    if any(errs):
        raise RuntimeError(f"device-side error bits {errs} during the benchmark")
    # end to end: the token set from pinned host memory, the result back
    hh = h0.cpu().pin_memory()
    ho = torch.empty_like(hh).pin_memory()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with torch.cuda.stream(stream):
        e_s.record(stream)
        for i in range(steps):
            h.copy_(hh, non_blocking=True)
            graph.launch(stream)
            ho.copy_(h, non_blocking=True)
        e_e.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), world)

    rb = synth.record_bytes(H, shape.inter, shape.bits)
    router_b = shape.n_experts * H * 4 + (H * 4 if shape.has_shared else 0)
    if B > 1:
        # distinct routed experts per layer-step, counted on the first step's routing
        hs = h0[:B].clone()
        uniq = []
        for L in layers:
            n = torch.empty_like(hs)
            fmoe.fmoe_rmsnorm(hs, n, B, H, 1e-6)
            idx, _, _ = L.route_batched(n)
            uniq.append(int(torch.unique(idx).numel()))
            L.block_batched(hs, h_out=hs)
        mean_u = sum(uniq) / len(uniq)
        step_bytes = (tokens / B) * NL * ((mean_u + shape.has_shared) * rb + router_b)
        expert_bytes = (tokens / B) * NL * (mean_u + shape.has_shared) * rb
    else:
        mean_u = None
        step_bytes = tokens * NL * ((shape.top_k + shape.has_shared) * rb + router_b)
        expert_bytes = tokens * NL * (shape.top_k + shape.has_shared) * rb
    peak, peak_kind = measured_peaks()
    step_s = total_ms / 1e3 / steps
    achieved = step_bytes / step_s / 1e9
    value = job_rate(tokens * steps, world, total_ms)
    graph.close()
    stack.close()
    for L in layers:
        L.close()
    del layers, graph, stack
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    cpu = None
    if world == 1 and cpu_tokens > 0:
        rates = cpu_oracle_rates(shape, cpu_tokens, block=True)
        cpu = cpu_baseline_line(rates, 1.0 / NL, "tokens/s",
                                f"{cpu_tokens} pre-norm blocks of layer 0 (fp64 numpy oracle), one token each; "
                                f"rate through all {NL} layers = block rate / {NL}")
    launches_per_layer = 1 if B == 1 else 6
    return {"metric": f"{NL}-layer stack decode tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": max(3, warmup), "ms_per_step": total_ms / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": f"{config}: {NL} pre-norm layers, hidden {H}, inter {shape.inter}, "
                                   f"{shape.n_experts}+{shape.has_shared} experts, top-{shape.top_k}, "
                                   f"{shape.bits}-bit, {tokens} tokens "
                                   + ("one at a time" if B == 1 else f"in steps of {B} grouped by expert"),
                       "tokens_per_step": tokens, "l2": "flushed between steps (512 MiB write)",
                       "parallelism": f"replicas x{world}"},
            "e2e": {"value": job_rate(tokens * steps, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": hh.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2},
            "gpu_launches": steps * NL * (tokens if B == 1 else -(-tokens // B) * launches_per_layer),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": None, "peak_kind": peak_kind,
                         "kernel": "whole step (all kernels)", "bytes_per_step": step_bytes,
                         "expert_gbs": round(expert_bytes / step_s / 1e9, 1),
                         "expert_frac_of_8tbs": round(expert_bytes / step_s / 1e9 / HBM_NOMINAL_GBS, 4),
                         "us_per_layer_token": round(step_s * 1e6 / (NL * tokens), 3),
                         "mean_distinct_experts_per_layer_step": mean_u},
            "cpu_baseline": cpu, "clocks": clocks,
            "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)}}


def bench_layer(args, world, rank, config):
    """The single-layer workload: every token one fmoe_layer_forward call, the calls
    of a step replayed from one CUDA graph.  Returns the bench line (rank 0)."""
    import torch
    import torch.distributed as dist

    import fmoe_synth as synth
    from bit_dequant_expert_softmax_b200 import fmoe
    from fmoe_synth.torch_layer import make_device_layer, make_device_x

    shape = synth.CONFIGS[config]["shape"]
    tokens = args.tokens or synth.CONFIGS[config]["tokens"]
    H = shape.hidden

    w = make_device_layer(shape, 0, 0)
    cfg = fmoe.fmoe_config(H, shape.inter, shape.n_experts, shape.top_k, shape.bits, shape.has_shared,
                           shape.router_bias)
    L = fmoe.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    x = make_device_x(0, rank * tokens, tokens, H)
    y = torch.empty_like(x)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def run_tokens(s):
        for t in range(tokens):
            fmoe.fmoe_layer_forward(L.handle, x[t:t + 1], x[t:t + 1], 1, y[t:t + 1], stream=s)

    with torch.cuda.stream(stream):
        run_tokens(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run_tokens(stream)
    torch.cuda.synchronize()

    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # L2 flush between steps (outside the timed events)
            starts[i].record(stream)
            graph.replay()
            ends[i].record(stream)
    barrier()
    clocks = sampler.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    total_ms = max_over_ranks(total_ms, world)
    err = L.error()
    if err:
        raise RuntimeError(f"device-side error bits {err:#x} during the benchmark")

    # end to end through the C ABI from pinned host buffers
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    barrier()
    with torch.cuda.stream(stream):
        e_s.record(stream)
        for i in range(args.steps):
            x.copy_(xh, non_blocking=True)
            graph.replay()
            yh.copy_(y, non_blocking=True)
        e_e.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), world)
    del graph
    L.close()
    del w, x, y, flush
    torch.cuda.empty_cache()

    value = job_rate(tokens * args.steps, world, total_ms)
    e2e_value = job_rate(tokens * args.steps, world, e2e_ms)
    expert_b, other_b = layer_bytes(shape)
    launch_s = (total_ms / 1e3) / (tokens * args.steps)
    peak, peak_kind = measured_peaks()
    achieved = (expert_b + other_b) / launch_s / 1e9
    expert_gbs = expert_b / launch_s / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic(),
            "traffic_warm": profiled_traffic("traffic_warm_bytes_per_launch"),
            "traffic_note": "traffic: DRAM read+write bytes of one cold-L2 launch (ncu flushes L2); "
                            "traffic_warm: per launch over consecutive launches without flushing, as in "
                            "the timed loop (the router and the shared expert can stay in L2 there)",
            "peak_kind": peak_kind, "kernel": f"fmoe_layer_kernel<{shape.bits}>",
            "bytes_per_launch": expert_b + other_b, "expert_bytes_per_launch": expert_b,
            "expert_gbs": round(expert_gbs, 1), "expert_frac_of_8tbs": round(expert_gbs / HBM_NOMINAL_GBS, 4),
            "expert_frac_of_measured": round(expert_gbs / peak, 4), "avg_launch_us": round(launch_s * 1e6, 3)}
    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rates = cpu_oracle_rates(shape, args.cpu_sample)
        cpu = cpu_baseline_line(rates, 1.0, "tokens/s",
                                f"{args.cpu_sample} tokens of the {H}x{shape.inter} layer (fp64 numpy oracle, "
                                f"expert records decoded in the timed forward)")
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": f"{config}: single-token decode, hidden {H}, inter {shape.inter}, "
                                   f"{shape.n_experts}+{shape.has_shared} experts, top-{shape.top_k}, "
                                   f"{shape.bits}-bit group-64",
                       "weights": f"{shape.bits}-bit codes, bf16 scale/bias per 64-group, HBM-resident",
                       "tokens_per_step": tokens, "l2": "flushed between steps (512 MiB write)",
                       "parallelism": f"replicas x{world}"},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": xh.numel() * 2,
                    "d2h_bytes_per_step": yh.numel() * 2},
            "gpu_launches": tokens * args.steps,
            "roofline": roof, "cpu_baseline": cpu, "clocks": clocks,
            "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)}}


def bench_tier(args, rank, slots: int = 64, tokens: int = 200):
    """The full-size layer with its routed experts in pinned host memory behind an HBM
    cache of `slots` records: single-token calls, each routing on the GPU, reading the
    routing back, copying the missing records host -> device and running the experts.
    Reports tokens/s, the host -> device GB/s of the expert copies and the cache hit
    rate (rank 0, one GPU)."""
    import torch

    import fmoe_synth as synth
    from bit_dequant_expert_softmax_b200 import fmoe
    from fmoe_synth.torch_layer import make_device_layer, make_device_x

    shape = synth.CONFIGS["layer4096"]["shape"]
    H, E = shape.hidden, shape.n_experts
    w = make_device_layer(shape, 0, 0)
    cfg = fmoe.fmoe_config(H, shape.inter, E, shape.top_k, shape.bits, shape.has_shared, shape.router_bias)
    rb = fmoe.fmoe_record_bytes(H, shape.inter, shape.bits)
    host = w.experts[:E * rb].cpu().pin_memory()
    shared = w.experts[E * rb:(E + 1) * rb].clone()
    router, rbias, gs = w.router, w.router_bias, w.shared_gate
    del w
    torch.cuda.empty_cache()
    tier = fmoe.Tier(cfg, host, shared, router, rbias, gs, slots, 1)
    x = make_device_x(0, 0, tokens, H)
    y = torch.empty_like(x)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for t in range(min(32, tokens)):  # warm the cache and the kernels
            tier.forward(x[t:t + 1], y=y[t:t + 1], stream=stream)
    torch.cuda.synchronize()
    s0 = tier.stats()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for t in range(tokens):
            tier.forward(x[t:t + 1], y=y[t:t + 1], stream=stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = a.elapsed_time(b)
    s1 = tier.stats()
    err = tier.error()
    tier.close()
    del tier, host, shared, x, y
    torch.cuda.empty_cache()
    if err:
        raise RuntimeError(f"device-side error bits {err:#x} in the tier benchmark")
    hits, misses = s1["hits"] - s0["hits"], s1["misses"] - s0["misses"]
    if rank != 0:
        return None
    return {"metric": "host-memory expert tier: MoE-layer decode tokens/s", "value": tokens / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": 1, "warmup": 32, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"layer4096 with its {E} routed expert records in pinned host memory, "
                                   f"an HBM cache of {slots} records (LRU), {tokens} single-token calls",
                       "tokens_per_step": tokens},
            "tier": {"h2d_gbs": round((s1["bytes_h2d"] - s0["bytes_h2d"]) / (ms / 1e3) / 1e9, 2),
                     "hit_rate": round(hits / max(1, hits + misses), 4), "hits": hits, "misses": misses,
                     "record_bytes": rb},
            "gpu_launches": 2 * tokens, "clocks": clocks}


def bench_gdn(args, rank, layers: int = 45, heads: int = 64, dk: int = 128, dv: int = 128, steps: int = 50):
    """GatedDeltaNet steps (the linear-attention layers beside the MoE: 45 of the 60
    layers of the pages' model, 64 heads of 128 x 128 fp32 state each): one token through
    all layers per step from a CUDA graph; the states (189 MB) exceed L2.  Roofline: the
    state is read and written once per layer (8.39 MB)."""
    import numpy as np
    import torch

    from bit_dequant_expert_softmax_b200 import fmoe

    rng = np.random.default_rng(0)
    S = torch.from_numpy((0.1 * rng.standard_normal((layers, heads, dv, dk))).astype(np.float32)).cuda()
    q = torch.nn.functional.normalize(torch.from_numpy(rng.standard_normal((layers, heads, dk)).astype(np.float32)),
                                      dim=-1).cuda()
    k = torch.nn.functional.normalize(torch.from_numpy(rng.standard_normal((layers, heads, dk)).astype(np.float32)),
                                      dim=-1).cuda()
    v = torch.from_numpy(rng.standard_normal((layers, heads, dv)).astype(np.float32)).cuda()
    alpha = torch.from_numpy(rng.uniform(0.5, 1.0, (layers, heads)).astype(np.float32)).cuda()
    beta = torch.from_numpy(rng.uniform(0.0, 1.0, (layers, heads)).astype(np.float32)).cuda()
    o = torch.empty(layers, heads, dv, dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def token():
        for l in range(layers):
            fmoe.fmoe_gdn_step(S[l], q[l], k[l], v[l], alpha[l], beta[l], o[l], stream=stream)

    with torch.cuda.stream(stream):
        token()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        token()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = a.elapsed_time(b)
    del g, S, q, k, v, alpha, beta, o
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    per_launch_bytes = heads * dv * dk * 4 * 2 + heads * (2 * dk + 2 * dv + 2) * 4
    launch_s = ms / 1e3 / (steps * layers)
    peak, peak_kind = measured_peaks()
    achieved = per_launch_bytes / launch_s / 1e9
    return {"metric": f"GatedDeltaNet step, {layers} layers x {heads} heads x {dv}x{dk} state: tokens/s",
            "value": steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": 3,
            "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"gdn: {layers} layers, {heads} heads, state {dv}x{dk} fp32 ({layers * heads * dv * dk * 4 / 1e6:.0f} MB), "
                                   "one token per step through all layers (CUDA graph)"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": profiled_traffic(summary="gdn_step_kernel_gdn45.md", sources=("fmoe_gdn.cuh",)),
                         "peak_kind": peak_kind,
                         "kernel": "gdn_step_kernel", "bytes_per_launch": per_launch_bytes,
                         "avg_launch_us": round(launch_s * 1e6, 3)},
            "gpu_launches": steps * layers, "clocks": clocks}


SUB_CONFIGS = ("stack24_4bit", "stack60_2bit", "stack16_batched")


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import datetime

    import torch
    import torch.distributed as dist

    import fmoe_synth as synth

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    cfg = synth.CONFIGS[args.config]
    if args.only and world == 1:
        line = bench_gdn(args, rank) if args.only == "gdn" else bench_tier(args, rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if cfg["layers"] > 1 or cfg["batch"] > 1:
        line = bench_stack(args, world, rank, args.config, args.steps, args.warmup,
                           0 if args.no_cpu_baseline else 2)
    else:
        line = bench_layer(args, world, rank, args.config)
        # the stacks ride along as sub-records of the default single-GPU run
        if world == 1 and args.config == "layer4096" and not args.no_sub and args.tokens is None:
            line["sub_records"] = [bench_stack(args, world, rank, c, args.sub_steps, 3,
                                               0 if args.no_cpu_baseline else 2) for c in SUB_CONFIGS]
            line["sub_records"].append(bench_tier(args, rank))
            line["sub_records"].append(bench_gdn(args, rank))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
