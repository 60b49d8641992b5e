#!/usr/bin/env python
"""Benchmark of the routed-expert MoE decode layer on B200.

Metric: MoE-layer decode tokens/s, with the effective expert-weight HBM GB/s
(and its fraction of HBM peak) for the full-size 4-bit top-4 layer: hidden 4096,
expert intermediate 1024, 512 routed experts + 1 shared, 1000 tokens with
independent seeded activations.  One step = the 1000 tokens, each a single-token
fmoe_layer_forward call (one fused kernel launch), the 1000 launches replayed
from one CUDA graph.  Weights (3.64 GB) are resident in HBM; the L2 is flushed
between steps.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

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
    ap.add_argument("--cpu-sample", type=int, default=10,
                    help="tokens timed once for the CPU oracle baseline of the GPU arm")
    ap.add_argument("--ref-tokens", type=int, default=1,
                    help="tokens per step of the reference arm (the CPU oracle)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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


def profiled_traffic():
    """DRAM bytes per launch of the layer kernel from the committed ncu summary, if
    the kernel source is the one that was profiled (else None)."""
    texts = []
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_dequant_expert_softmax_b200", "csrc", f)) as fh:
            texts.append(fh.read())
    path = os.path.join(ROOT, "profiles", "fmoe_layer_kernel_layer4096.md")
    if not os.path.exists(path):
        return None
    want, traffic = None, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line.startswith("kernel_source_digest:"):
                want = line.split(":", 1)[1].strip()
            elif line.startswith("traffic_bytes_per_launch:"):
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


def cpu_oracle_rate(shape, n_tokens: int, seed: int = 0):
    """The fp64 oracle (as it stands) on n_tokens tokens of the workload: returns
    (tokens/s, threads used, description).  Expert records are regenerated before
    each token's timed forward, which is then run from the packed bytes."""
    import numpy as np

    import fmoe_synth as synth
    import oracle
    olay = oracle.synthetic_layer(seed, 0, shape, lazy=True)
    total = 0.0
    for t in range(n_tokens):
        x = oracle.bf16_to_f64(synth.gen_x_token(seed, t, shape.hidden))
        idx, _, _, _ = olay.route(x)
        recs = {int(e): synth.gen_record(seed, 0, int(e), shape.hidden, shape.inter, shape.bits)
                for e in list(idx) + [shape.n_experts]}
        olay._cache = {}
        olay._records = lambda e, _r=recs: _r[e]
        t0 = time.perf_counter()
        olay.forward(x)
        total += time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        threads = 1
    return n_tokens / total, threads, f"{n_tokens} tokens of the {shape.hidden}x{shape.inter} layer"


def run_reference(args, rank):
    """The reference arm: the fp64 CPU oracle, timed on the host cores."""
    import fmoe_synth as synth
    if rank != 0:
        return
    shape = synth.CONFIGS[args.config]["shape"]
    per_step = max(1, args.ref_tokens)
    for _ in range(args.warmup and 1):
        cpu_oracle_rate(shape, 1)
    t_all = 0.0
    tok = 0
    threads, desc = 1, ""
    for _ in range(args.steps):
        rate, threads, desc = cpu_oracle_rate(shape, per_step)
        t_all += per_step / rate
        tok += per_step
    value = tok / t_all
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t_all / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.config}: single-token decode, hidden {shape.hidden}, "
                                   f"inter {shape.inter}, {shape.n_experts}+{shape.has_shared} experts, "
                                   f"top-{shape.top_k}, {shape.bits}-bit",
                       "tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{per_step} tokens per step ({desc})"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_stack(args, world, rank):
    """A layer stack (pre-norm blocks) decoding its token set through the captured
    graph: token after token (batch 1) or in steps of `batch` tokens on the batched
    path.  One step = every token of the set through every layer."""
    import torch
    import torch.distributed as dist

    import fmoe_synth as synth
    from bit_dequant_expert_softmax_b200 import fmoe
    from fmoe_synth.torch_layer import make_device_layer, make_device_x

    cfg_d = synth.CONFIGS[args.config]
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
        for _ in range(max(3, args.warmup)):
            h.copy_(h0)
            graph.launch(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
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
        for i in range(args.steps):
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
    step_s = total_ms / 1e3 / args.steps
    achieved = step_bytes / step_s / 1e9
    value = job_rate(tokens * args.steps, world, total_ms)
    if rank == 0:
        launches_per_layer = 1 if B == 1 else 6
        line = {"metric": f"{NL}-layer stack decode tokens/s", "value": value, "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": {"workload": f"{args.config}: {NL} pre-norm layers, hidden {H}, inter {shape.inter}, "
                                       f"{shape.n_experts}+{shape.has_shared} experts, top-{shape.top_k}, "
                                       f"{shape.bits}-bit, {tokens} tokens "
                                       + ("one at a time" if B == 1 else f"in steps of {B} grouped by expert"),
                           "tokens_per_step": tokens, "l2": "flushed between steps (512 MiB write)",
                           "parallelism": f"replicas x{world}"},
                "e2e": {"value": job_rate(tokens * args.steps, world, e2e_ms), "unit": "tokens/s",
                        "h2d_bytes_per_step": hh.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2},
                "gpu_launches": args.steps * NL * (tokens if B == 1 else -(-tokens // B) * launches_per_layer),
                "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                             "frac": round(achieved / peak, 4), "traffic": None, "peak_kind": peak_kind,
                             "kernel": "whole step (all kernels)", "bytes_per_step": step_bytes,
                             "expert_gbs": round(expert_bytes / step_s / 1e9, 1),
                             "mean_distinct_experts_per_layer_step": mean_u},
                "cpu_baseline": None, "clocks": clocks,
                "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)}}
        print(json.dumps(line), flush=True)
    graph.close()
    stack.close()
    for L in layers:
        L.close()


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
    from bit_dequant_expert_softmax_b200 import fmoe
    from fmoe_synth.torch_layer import make_device_layer, make_device_x

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if synth.CONFIGS[args.config]["layers"] > 1 or synth.CONFIGS[args.config]["batch"] > 1:
        bench_stack(args, world, rank)
        if world > 1:
            dist.destroy_process_group()
        return
    shape = synth.CONFIGS[args.config]["shape"]
    tokens = args.tokens or synth.CONFIGS[args.config]["tokens"]
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

    value = job_rate(tokens * args.steps, world, total_ms)
    e2e_value = job_rate(tokens * args.steps, world, e2e_ms)
    expert_b, other_b = layer_bytes(shape)
    launch_s = (total_ms / 1e3) / (tokens * args.steps)
    peak, peak_kind = measured_peaks()
    achieved = (expert_b + other_b) / launch_s / 1e9
    expert_gbs = expert_b / launch_s / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic(),
            "peak_kind": peak_kind, "kernel": "fmoe_layer_kernel<4>",
            "bytes_per_launch": expert_b + other_b, "expert_bytes_per_launch": expert_b,
            "expert_gbs": round(expert_gbs, 1), "expert_frac_of_8tbs": round(expert_gbs / HBM_NOMINAL_GBS, 4),
            "expert_frac_of_measured": round(expert_gbs / peak, 4), "avg_launch_us": round(launch_s * 1e6, 3)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, desc = cpu_oracle_rate(shape, args.cpu_sample)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{args.cpu_sample} tokens ({desc}), fp64 numpy oracle"}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": {"workload": f"{args.config}: single-token decode, hidden {H}, inter {shape.inter}, "
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
        print(json.dumps(line), flush=True)
    del graph
    L.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
