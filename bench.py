#!/usr/bin/env python
"""Benchmark of the quantized MoE expert block on B200.

Default workload: batch-1 decode through 48 stacked MoE layers (H=2048, E=256 experts, top-8,
I=512, int4 group-64 affine experts), one step = one decode token through all 48 layers
(router top-k, gate/up, SiLU-GLU, down and combine per layer), replayed as one CUDA graph of
48 decode-megakernel launches. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Multi-GPU (torchrun): replicas only -- every rank runs its own copy of the workload, no
data-path collective; torch.distributed is used for the start barrier and the max-over-ranks
time only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "decode_t1_l48_h2048_e256_k8_i512_int4"
PREFILL_WORKLOAD = "prefill_t4096_l8_h2048_e256_k8_i512_int4"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill measurement of the default run")
    ap.add_argument("--layers", type=int, default=0,
                    help="stack only this many layers of the workload (smaller case for profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------------------ helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(profile_file, sources):
    """dram bytes per launch from a committed ncu summary, if its kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", profile_file)
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("source_sha256") != source_hash(sources):
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device="cuda"):
    """The largest of the ranks' values (device times: the job takes as long as its slowest rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------ CPU oracle

def oracle_decode_sample(w, steps, layers, threads=None):
    """Times the fp64 oracle on `steps` decode steps x `layers` layers of workload w.
    Returns (seconds of oracle compute, tokens processed, threads used)."""
    import oracle
    import synth
    o = oracle.get()
    if threads:
        o.set_threads(threads)
    wr = {l: synth.router_weights(w, l) for l in range(layers)}
    bias = {l: synth.router_bias(w, l) for l in range(layers)}
    bits = {l: synth.expert_bits(w, l) for l in range(layers)}
    total = 0.0
    for s in range(steps):
        for l in range(layers):
            x = synth.hidden(w, s, l)
            t0 = time.perf_counter()
            logits = o.router_logits(x, wr[l], bias[l])
            idx, ww = o.topk(logits, w.k)
            total += time.perf_counter() - t0
            experts = [None] * w.E
            for e in np.unique(idx):
                experts[int(e)] = synth.expert_tensors(w, l, int(e), int(bits[l][int(e)]))
            t0 = time.perf_counter()
            o.combine(x, experts, w.H, w.I, idx, ww)
            total += time.perf_counter() - t0
    return total, steps * w.T, o.threads()


def metric_name(w):
    return ("decode" if w.mode == "decode" else "prefill") + " tokens/s (MoE expert block, all layers)"


def base_config(w, world):
    """The workload keys of the config object, the same on both arms."""
    return {"workload": w.name, "tokens_per_step": w.T, "layers": w.layers, "H": w.H, "E": w.E, "k": w.k,
            "I": w.I, "weights": "mixed 4/6/8-bit" if w.mixed_bits else f"int{w.bits} group-64 affine",
            "parallelism": f"replicas x{world}"}


def run_reference(args, w):
    """--impl reference: the fp64 oracle on the host cores, one step = one decode token through
    `layers_per_step` layers of the workload (a bounded sample), rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    layers = min(w.layers, 8) if w.mode == "decode" else 1
    times = []
    threads = 0
    for i in range(args.warmup + args.steps):
        t, tokens, threads = oracle_decode_sample(w, 1, layers)
        if i >= args.warmup:
            times.append(t)
    per_step = statistics.mean(times)
    # tokens/s of the full workload: one token needs all w.layers layers
    value = w.T / (per_step * w.layers / layers)
    sample = (f"{args.steps} steps, each 1 token through {layers} of {w.layers} layers (fp64; tokens are "
              f"independent in this block), scaled to all layers")
    line = {
        "impl": "reference", "metric": metric_name(w), "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * w.layers / layers * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": base_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ ours

def build_layers(w):
    import torch
    import synth
    import synth.device as sd
    import quantized_moe_router_b200 as qm
    from quantized_moe_router_b200.runner import LayerWeights
    layers = []
    active_bytes = []
    for l in range(w.layers):
        bits = synth.expert_bits(w, l)
        wr = sd.router_weights(w, l)
        b = synth.router_bias(w, l)
        bias = None if b is None else torch.from_numpy(b).cuda()
        experts = [sd.expert_tensors(w, l, e, int(bits[e])) for e in range(w.E)]
        packed = qm.pack_layer(experts, w.H, w.I)
        torch.cuda.synchronize()
        del experts
        layers.append(LayerWeights(wr, bias, packed))
        active_bytes.append(bits)
    return layers, active_bytes


def expert_bytes(H, I, bits):
    return 3 * I * H // 1024 * {4: 576, 6: 832, 8: 1088}[int(bits)]


def run_ours(args, w):
    import torch
    import synth.device as sd
    from quantized_moe_router_b200.runner import DecodeStack
    rank, world, local = dist_setup(args.gpus)
    if w.mode == "prefill":
        res = run_prefill(args, w, world, rank)
        res.pop("workload")
        line = {"metric": res.pop("metric"), "value": res.pop("value"), "unit": res.pop("unit"), "n_gpus": world,
                "steps": res.pop("steps"), "warmup": max(args.warmup, 3), "ms_per_step": res.pop("ms_per_step"),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": dict(base_config(w, world),
                               l2="no flush: each layer streams the weights of all its experts (> 126 MB L2)"),
                "gpu_launches": res["steps_launches"], **{k: v for k, v in res.items() if k != "steps_launches"}}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    assert w.mode == "decode", "bench.py times the decode and prefill workloads"
    layers, bits = build_layers(w)
    stack = DecodeStack(layers, w.T, w.H, w.I, w.E, w.k)
    nsteps = args.warmup + args.steps
    xs = torch.empty((min(nsteps, w.steps), w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    for s in range(xs.shape[0]):
        for l in range(w.layers):
            sd.hidden(w, s, l, out=xs[s, l])
    stack.capture()
    torch.cuda.synchronize()

    def step(i):
        stack.x_in.copy_(xs[i % xs.shape[0]], non_blocking=True)
        stack.replay()

    # ---------------- device-resident timing
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    st = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(st)
        for i in range(args.steps):
            step(args.warmup + i)
        ev1.record(st)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    barrier(world)
    ms = max_over_ranks(ms, world)
    # selections of the last step -> unique experts per layer (for the byte count)
    idx = stack.idx.cpu().numpy()
    uniq_bytes = []
    for l in range(w.layers):
        u = np.unique(idx[l])
        uniq_bytes.append(sum(expert_bytes(w.H, w.I, bits[l][e]) for e in u))
    expert_b = float(np.mean(uniq_bytes))
    router_b = w.E * w.H * 4 + (w.E * 4 if w.zipf else 0)
    io_b = 2 * w.T * w.H * 2
    layer_bytes = expert_b + router_b + io_b

    # ---------------- kernel-only: graph replays without the x copy
    torch.cuda.synchronize()
    ek0, ek1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ek0.record(st)
    for i in range(args.steps):
        stack.replay()
    ek1.record(st)
    torch.cuda.synchronize()
    kern_ms = ek0.elapsed_time(ek1) / (args.steps * w.layers)

    hbm, bf16, peak_src = measured_peaks()
    achieved = layer_bytes / (kern_ms * 1e-3) / 1e9
    traffic = recorded_traffic("decode_megakernel_decode_t1_l48_h2048.txt",
                               ["quantized_moe_router_b200/csrc/moe_decode.cu",
                                "quantized_moe_router_b200/csrc/moe_internal.cuh",
                                "quantized_moe_router_b200/csrc/moe_topk.cuh"])

    # ---------------- end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        xh = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16).pin_memory()
        oh = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16).pin_memory()
        xh.copy_(xs[0].cpu())
        for i in range(args.warmup):
            stack.x_in.copy_(xh, non_blocking=True)
            stack.replay()
            oh.copy_(stack.out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ee0.record(st)
        for i in range(args.steps):
            stack.x_in.copy_(xh, non_blocking=True)
            stack.replay()
            oh.copy_(stack.out, non_blocking=True)
        ee1.record(st)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), world)
        nbytes = w.layers * w.T * w.H * 2
        e2e = {"value": world * w.T * args.steps / (e2e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes}

    line = {
        "metric": metric_name(w),
        "value": world * w.T * args.steps / (ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(base_config(w, world),
                       l2="no flush: each step streams ~%.0f MB of expert weights (> 126 MB L2); %.1f GB resident"
                          % (expert_b * w.layers / 1e6, sum(lw.packed.numel() for lw in layers) / 1e9)),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": traffic, "peak_source": peak_src,
                     "bytes_per_launch": layer_bytes, "kernel_ms_per_launch": kern_ms,
                     "expert_bytes_per_launch": expert_b,
                     "expert_bytes_frac_of_8TBs": expert_b / (kern_ms * 1e-3) / 8e12},
        "gpu_launches": args.steps * w.layers,
        "clocks": clk.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if not args.no_prefill:
        del layers, stack, xs
        torch.cuda.empty_cache()
        import synth
        pre = run_prefill(args, synth.WORKLOADS[PREFILL_WORKLOAD], world, rank)
        pre["gpu_launches"] = pre.pop("steps_launches")
        line["prefill"] = pre
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t, tokens, threads = oracle_decode_sample(w, 1, w.layers)
        line["cpu_baseline"] = {"value": tokens / t, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"1 decode token through all {w.layers} layers (fp64 oracle)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ prefill

def prefill_flops(w):
    """Expert-GEMM flops of one prefill layer: gate, up and down for every (token, expert) pair."""
    return 2.0 * w.T * w.k * 3 * w.I * w.H


def oracle_prefill_sample(w, ntok):
    """Times the fp64 oracle on the first `ntok` tokens of layer 0 of prefill workload w.
    Returns (seconds, tokens, threads)."""
    import oracle
    import synth
    o = oracle.get()
    wr = synth.router_weights(w, 0)
    x = synth.hidden(w, 0, 0)[:ntok]
    bits = synth.expert_bits(w, 0)
    t0 = time.perf_counter()
    logits = o.router_logits(x, wr, None)
    idx, ww = o.topk(logits, w.k)
    t_route = time.perf_counter() - t0
    experts = [None] * w.E
    for e in np.unique(idx):
        experts[int(e)] = synth.expert_tensors(w, 0, int(e), int(bits[int(e)]))
    t0 = time.perf_counter()
    o.combine(x, experts, w.H, w.I, idx, ww)
    return t_route + time.perf_counter() - t0, ntok, o.threads()


def run_prefill(args, w, world, rank):
    """One step = all w.T tokens through w.layers prefill layers (route + bucket + grouped GEMMs +
    combine per layer), fresh x per layer. Returns the measurement as a dict."""
    import torch
    import synth.device as sd
    import quantized_moe_router_b200 as qm
    layers, _ = build_layers(w)
    xs = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    for l in range(w.layers):
        sd.hidden(w, 0, l, out=xs[l])
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_PREFILL)
    out = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream()

    def step(ev=None):
        for l, lw in enumerate(layers):
            qm.prefill_route(xs[l], lw.wr, lw.bias, w.I, w.E, w.k, ws)
            if ev:
                ev[l][0].record(st)
            qm.prefill_experts(xs[l], lw.packed, w.I, w.E, w.k, ws, out=out[l])
            if ev:
                ev[l][1].record(st)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    nsteps = max(1, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(w.layers)]
           for _ in range(nsteps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(st)
        for i in range(nsteps):
            step(evs[i])
        e1.record(st)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    gemm_ms = float(np.mean([ev[0].elapsed_time(ev[1]) for evl in evs for ev in evl]))
    assert qm.device_status(ws) == qm.MOE_OK
    _, bf16, peak_src = measured_peaks()
    achieved = prefill_flops(w) / (gemm_ms * 1e-3) / 1e12
    res = {
        "workload": w.name, "metric": metric_name(w),
        "value": world * w.T * nsteps / (ms * 1e-3), "unit": "tokens/s", "steps": nsteps,
        "ms_per_step": ms / nsteps, "ms_per_layer": ms / nsteps / w.layers,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                     "frac": achieved / bf16,
                     "traffic": recorded_traffic("prefill_tc_grouped_prefill_t4096_h2048.txt",
                                                 ["quantized_moe_router_b200/csrc/moe_prefill_tc.cu",
                                                  "quantized_moe_router_b200/csrc/moe_prefill.cu",
                                                  "quantized_moe_router_b200/csrc/moe_internal.cuh"])
                     if w.name == "prefill_t4096_l8_h2048_e256_k8_i512_int4" else None,
                     "peak_source": peak_src,
                     "flops_per_launch": prefill_flops(w),
                     "kernel": "expert phase (moe_prefill_experts: grouped gate/up + down GEMMs, combine)",
                     "kernel_ms_per_launch": gemm_ms},
        "clocks": clk.summary(),
        # route, 3 bucketing kernels, N-tile scan, gate/up GEMM, down GEMM, bf16 conversion per layer
        "steps_launches": nsteps * w.layers * 8,
    }
    del layers
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t, tokens, threads = oracle_prefill_sample(w, 16)
        res["cpu_baseline"] = {"value": tokens / (t * w.layers), "unit": "tokens/s", "cores": threads,
                               "kind": "oracle",
                               "sample": f"16 tokens of layer 0 (fp64 oracle), scaled to {w.layers} layers"}
    return res


def main():
    args = parse()
    import synth
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layers=min(args.layers, w.layers))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
