#!/usr/bin/env python
"""Benchmark of the quantized MoE expert block on B200.

One bench step is one pass of a workload's whole recipe through the expert block:

* decode workloads: every decode step of the recipe through every layer (for the default,
  256 batch-1 decode tokens through 48 stacked MoE layers, H=2048, E=256 experts, top-8,
  I=512, int4 group-64 affine experts), replayed as one CUDA graph of steps x layers
  decode-megakernel launches, fresh hidden states per (step, layer);
* the single-layer workload: one decode call, timed alone with L2 flushed before it;
* the prefill workload: 4096 tokens through 8 layers (route, bucketing, grouped GEMMs,
  combine per layer).

The default run times the 48-layer decode workload (the line's headline) and nests the
other four workloads under "configs", each with its throughput, roofline, end-to-end
figure, near-tie counts and CPU (fp64 oracle) baselines. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--only] [--layers L] [--seq S]

Multi-GPU (torchrun): replicas only -- every rank runs its own copy of the workload, no
data-path collective; torch.distributed is used for the barriers and the max-over-ranks time.
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
SINGLE_WORKLOAD = "moe_t1_h1024_e32_k4_i256_int4"
PREFILL_WORKLOAD = "prefill_t4096_l8_h2048_e256_k8_i512_int4"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TIE = 1e-4          # near-tie band of the top-k comparison (logit gap)
L2_FLUSH_BYTES = 512 << 20
# kernels of one prefill layer: route, three bucketing kernels, N-tile scan, x exponents, x gather,
# gate/up GEMM, h rescale, down GEMM, bf16 conversion
PREFILL_LAUNCHES_PER_LAYER = 11

DECODE_SOURCES = ["quantized_moe_router_b200/csrc/moe_decode.cu",
                  "quantized_moe_router_b200/csrc/moe_internal.cuh",
                  "quantized_moe_router_b200/csrc/moe_topk.cuh"]
PREFILL_SOURCES = ["quantized_moe_router_b200/csrc/moe_prefill_tc.cu",
                   "quantized_moe_router_b200/csrc/moe_prefill.cu",
                   "quantized_moe_router_b200/csrc/moe_internal.cuh",
                   "quantized_moe_router_b200/csrc/moe_tc.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--only", action="store_true", help="time only --workload (no nested configs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-ties", action="store_true", help="skip the near-tie count against the oracle")
    ap.add_argument("--layers", type=int, default=0,
                    help="stack only this many layers of the workload (smaller case for profiling)")
    ap.add_argument("--next", action="store_true",
                    help="with --only: also time the next rows (quantiser, streamed decode, mixed prefill)")
    ap.add_argument("--seq", type=int, default=0,
                    help="decode steps per bench step (default: the workload's own count)")
    return ap.parse_args()


# ------------------------------------------------------------------------------ helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS),
                d.get("bf16_tflops_sustained"), "measured")
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, None, "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(profile_file, sources):
    """DRAM bytes per launch from a committed ncu summary, if its kernel sources are unchanged."""
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


def nvml_handle(nv, cuda_index):
    """NVML handle of CUDA device `cuda_index`, following CUDA_VISIBLE_DEVICES (indices or UUIDs)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ent = [v.strip() for v in vis.split(",") if v.strip()][cuda_index]
        if ent.isdigit():
            return nv.nvmlDeviceGetHandleByIndex(int(ent))
        return nv.nvmlDeviceGetHandleByUUID(ent if ent.startswith("GPU-") or ent.startswith("MIG-") else ent)
    return nv.nvmlDeviceGetHandleByIndex(cuda_index)


class ClockSampler:
    """SM clock and throttle-reason samples during a timed region, read through NVML every
    few milliseconds (nvidia-smi's own source), so that short regions still get samples."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, interval_s: float = 0.004):
        self.gpu, self.interval = gpu_index, interval_s
        self.samples = []
        self._stop = threading.Event()
        self._t = None
        self._nv = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = nvml_handle(pynvml, self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:  # noqa: BLE001 - no NVML: the line reports no samples
            self._nv = None
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((sm, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.interval)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvml"}
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml",
                "interval_ms": self.interval * 1e3}


def dist_setup():
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


def expert_bytes(H, I, bits):
    """Packed bytes of one expert (codes + fp16 scale and zero) at a code width."""
    return 3 * I * H // 1024 * {4: 576, 6: 832, 8: 1088}[int(bits)]


def metric_name(w):
    return ("decode" if w.mode == "decode" else "prefill") + " tokens/s (MoE expert block, all layers)"


def base_config(w, world, seq=None):
    """The workload keys of the config object, the same on both arms."""
    c = {"workload": w.name, "tokens_per_call": w.T, "layers": w.layers, "H": w.H, "E": w.E, "k": w.k,
         "I": w.I, "weights": "mixed 4/6/8-bit" if w.mixed_bits else f"int{w.bits} group-64 affine",
         "parallelism": f"replicas x{world}"}
    if w.mode == "decode":
        c["decode_steps_per_bench_step"] = seq if seq else w.steps
    return c


# ------------------------------------------------------------------------------ CPU oracle

def oracle_decode_sample(w, ntok, layers, threads):
    """Times the fp64 oracle on the first `ntok` tokens of step 0 through `layers` layers of
    workload w with `threads` threads. Returns (seconds, tokens, threads used)."""
    import oracle
    import synth
    o = oracle.get()
    o.set_threads(threads)
    try:
        total = 0.0
        for l in range(layers):
            wr = synth.router_weights(w, l)
            bias = synth.router_bias(w, l)
            bits = synth.expert_bits(w, l)
            x = synth.hidden(w, 0, l, T=ntok)
            t0 = time.perf_counter()
            logits = o.router_logits(x, wr, bias)
            idx, ww = o.topk(logits, w.k)
            total += time.perf_counter() - t0
            experts = [None] * w.E
            for e in np.unique(idx):
                experts[int(e)] = synth.expert_tensors(w, l, int(e), int(bits[int(e)]))
            t0 = time.perf_counter()
            o.combine(x, experts, w.H, w.I, idx, ww)
            total += time.perf_counter() - t0
        return total, ntok, o.threads()
    finally:
        o.set_threads(os.cpu_count() or 1)


# bounded CPU samples per workload (tokens of step 0, layers), all cores and one core
CPU_SAMPLES = {
    SINGLE_WORKLOAD: ((1, 1), (1, 1)),
    DEFAULT_WORKLOAD: ((1, 8), (1, 2)),
    "decode_t1_l16_h4096_e512_k10_i1024_int4": ((1, 4), (1, 1)),
    "decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1": ((16, 2), (4, 1)),
    PREFILL_WORKLOAD: ((16, 1), (4, 1)),
}


def cpu_baselines(w):
    """The oracle timed on bounded samples of workload w: all host cores and one core, scaled
    to the workload's tokens/s (a token needs every layer)."""
    import oracle
    allc = oracle.get().threads()
    res = {}
    for key, (ntok, nl), thr in (("cpu_baseline", CPU_SAMPLES[w.name][0], allc),
                                 ("cpu_baseline_1core", CPU_SAMPLES[w.name][1], 1)):
        nl = min(nl, w.layers)
        t, tokens, used = oracle_decode_sample(w, ntok, nl, thr)
        res[key] = {"value": tokens / (t * w.layers / nl), "unit": "tokens/s", "cores": used, "kind": "oracle",
                    "sample": f"{tokens} token(s) of step 0 through {nl} of {w.layers} layers (fp64 oracle, "
                              f"{used} thread(s)), scaled to all layers"}
    return res


def run_reference(args, w):
    """--impl reference: the fp64 oracle on the host cores, each step one token through
    min(layers, 8) layers of the workload (a bounded sample), rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    layers = min(w.layers, 8)
    ntok = 1 if w.mode == "decode" and w.T == 1 else 4
    times = []
    threads = 0
    for i in range(args.warmup + args.steps):
        t, tokens, threads = oracle_decode_sample(w, ntok, layers, oracle.get().threads())
        if i >= args.warmup:
            times.append(t)
    per_tok = statistics.mean(times) / ntok
    value = 1.0 / (per_tok * w.layers / layers)
    sample = (f"{args.steps} steps, each {ntok} token(s) through {layers} of {w.layers} layers (fp64; tokens "
              f"are independent in this block), scaled to all layers")
    line = {
        "impl": "reference", "metric": metric_name(w), "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times) * w.layers / layers * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": base_config(w, args.gpus, getattr(args, "seq", 0) or None),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ near-ties

def tie_stats(o, x_bits, wr, bias, k, gpu_idx, gpu_w):
    """Routing of a batch of calls against the oracle's fp64 logits.

    x_bits [n, H] bf16 bits, gpu_idx / gpu_w [n, k]. Counts near-ties (oracle gap between the
    k-th and (k+1)-th logit <= TIE, where another set is allowed), sets that differ outside the
    band (must be 0), order swaps among logits within TIE, order mismatches outside it (must be
    0) and the largest routing-weight difference."""
    logits = o.router_logits(x_bits, wr, bias)
    n, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")
    ref = order[:, :k]
    lk = np.take_along_axis(logits, ref[:, -1:], 1)[:, 0]
    lk1 = np.take_along_axis(logits, order[:, k:k + 1], 1)[:, 0] if k < E else np.full(n, -np.inf)
    tied = (lk - lk1) <= TIE
    g = np.asarray(gpu_idx, np.int64)
    same_set = np.all(np.sort(g, 1) == np.sort(ref, 1), axis=1)
    lg = np.take_along_axis(logits, g, 1)
    same_order = np.all(g == ref, axis=1)
    swaps_ok = np.all(np.abs(lg - np.take_along_axis(logits, ref, 1)) <= TIE, axis=1)
    ww = np.exp(lg - lg.max(1, keepdims=True))
    ww /= ww.sum(1, keepdims=True)
    return {"tokens": int(n), "near_ties": int(np.sum(tied)),
            "near_tie_set_changes": int(np.sum(tied & ~same_set)),
            "set_mismatch_outside_band": int(np.sum(~tied & ~same_set)),
            "order_swaps": int(np.sum(same_set & ~same_order & swaps_ok)),
            "order_mismatch_outside_band": int(np.sum(same_set & ~same_order & ~swaps_ok)),
            "max_weight_diff": float(np.max(np.abs(np.asarray(gpu_w, np.float64) - ww))) if n else 0.0}


def merge_ties(parts):
    out = {}
    for p in parts:
        for key, v in p.items():
            out[key] = max(out.get(key, 0.0), v) if key == "max_weight_diff" else out.get(key, 0) + v
    return out


def bf16_np(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


# ------------------------------------------------------------------------------ ours: decode

def build_layers(w):
    import torch
    import synth
    import synth.device as sd
    import quantized_moe_router_b200 as qm
    from quantized_moe_router_b200.runner import LayerWeights
    layers, bits = [], []
    for l in range(w.layers):
        b = synth.expert_bits(w, l)
        wr = sd.router_weights(w, l)
        bb = synth.router_bias(w, l)
        bias = None if bb is None else torch.from_numpy(bb).cuda()
        experts = [sd.expert_tensors(w, l, e, int(b[e])) for e in range(w.E)]
        packed = qm.pack_layer(experts, w.H, w.I)
        torch.cuda.synchronize()
        del experts
        layers.append(LayerWeights(wr, bias, packed))
        bits.append(b)
    return layers, bits


def decode_leg(args, w, world, rank):
    """One decode workload: returns the measurement dict (rank 0's view)."""
    import torch
    import synth
    import synth.device as sd
    from quantized_moe_router_b200.runner import DecodeRun
    S = min(args.seq, w.steps) if args.seq else w.steps
    layers, bits = build_layers(w)
    x = torch.empty((S, w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    for s in range(S):
        for l in range(w.layers):
            sd.hidden(w, s, l, out=x[s, l])
    run = DecodeRun(layers, x, w.I, w.E, w.k)
    run.capture()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    W = max(args.warmup, 3)
    for _ in range(W):
        run.replay()
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(st)
        for _ in range(args.steps):
            run.replay()
        ev1.record(st)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    barrier(world)
    ms = max_over_ranks(ms, world)
    tokens_per_step = S * w.T
    per_launch_ms = ms / (args.steps * run.launches)

    # bytes: per call, the unique experts its tokens selected (+ router rows, x and out)
    idx = run.idx.cpu().numpy()
    wts = run.wts.cpu().numpy()
    eb = np.zeros((S, w.layers))
    for l in range(w.layers):
        per = np.array([expert_bytes(w.H, w.I, b) for b in bits[l]], np.float64)
        for s in range(S):
            eb[s, l] = per[np.unique(idx[s, l])].sum()
    expert_b = float(eb.mean())
    router_b = w.E * w.H * 4 + (w.E * 4 if w.zipf else 0)
    layer_bytes = expert_b + router_b + 2 * w.T * w.H * 2
    hbm, _, _, peak_src = measured_peaks()
    achieved = layer_bytes / (per_launch_ms * 1e-3) / 1e9
    prof = {DEFAULT_WORKLOAD: "decode_megakernel_decode_t1_l48_h2048.txt",
            "decode_t1_l16_h4096_e512_k10_i1024_int4": "decode_megakernel_decode_t1_l16_h4096.txt",
            "decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1": "decode_megakernel_decode_t16_l24_h2048.txt"}
    res = {
        "metric": metric_name(w), "value": world * tokens_per_step * args.steps / (ms * 1e-3), "unit": "tokens/s",
        "steps": args.steps, "warmup": W, "ms_per_step": ms / args.steps, "tokens_per_step": tokens_per_step,
        "config": dict(base_config(w, world, S),
                       l2="no flush: each bench step streams ~%.1f GB of expert weights (> 126 MB L2); %.1f GB "
                          "resident" % (expert_b * S * w.layers / 1e9,
                                        sum(lw.packed.numel() for lw in layers) / 1e9)),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": recorded_traffic(prof.get(w.name, ""), DECODE_SOURCES), "peak_source": peak_src,
                     "kernel": "decode megakernel (moe_expert_forward_decode), one launch per layer call",
                     "bytes_per_launch": layer_bytes, "expert_bytes_per_launch": expert_b,
                     "kernel_us_per_launch": per_launch_ms * 1e3,
                     "expert_bytes_frac": expert_b / (per_launch_ms * 1e-3) / 1e9 / hbm,
                     "expert_bytes_frac_of_8TBs": expert_b / (per_launch_ms * 1e-3) / 8e12},
        "gpu_launches": args.steps * run.launches,
        "clocks": clk.summary(),
    }

    # near-ties over every call of the bench step (host fp64 oracle, rank 0)
    if rank == 0 and not args.no_ties:
        import oracle
        o = oracle.get()
        xb = bf16_np(x).reshape(S, w.layers, w.T, w.H)
        parts = []
        for l in range(w.layers):
            wr = run.layers[l].wr.cpu().numpy()
            bias = synth.router_bias(w, l)
            parts.append(tie_stats(o, xb[:, l].reshape(S * w.T, w.H), wr, bias, w.k,
                                   idx[:, l].reshape(S * w.T, w.k), wts[:, l].reshape(S * w.T, w.k)))
        res["routing"] = dict(merge_ties(parts), calls=S * w.layers, band=TIE)

    # end to end: pinned host x -> device, the graph, device -> host out, every step; the host
    # batches alternate so that consecutive steps read different hidden states
    if not args.no_e2e:
        nb = 2
        xh = torch.empty((nb,) + tuple(x.shape), dtype=torch.bfloat16).pin_memory()
        oh = torch.empty(tuple(x.shape), dtype=torch.bfloat16).pin_memory()
        xh[0].copy_(x.cpu())
        # the second batch: every call's hidden states moved to the next call
        xh[1].copy_(torch.roll(x.reshape(S * w.layers, w.T, w.H), 1, 0).reshape(x.shape).cpu())
        for i in range(W):
            x.copy_(xh[i % nb], non_blocking=True)
            run.replay()
            oh.copy_(run.out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ee0.record(st)
        for i in range(args.steps):
            x.copy_(xh[i % nb], non_blocking=True)
            run.replay()
            oh.copy_(run.out, non_blocking=True)
        ee1.record(st)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), world)
        nbytes = x.numel() * 2
        res["e2e"] = {"value": world * tokens_per_step * args.steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                      "inputs": f"{nb} pinned host batches alternating per step"}
        del xh, oh
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res.update(cpu_baselines(w))
    del run, layers, x
    torch.cuda.empty_cache()
    return res


def single_leg(args, w, world, rank):
    """The single-layer, single-token workload: each timed call runs after a write of 512 MB
    (L2 flushed: the layer's 14 MB of experts would otherwise stay in L2), timed alone with
    CUDA events; a bench step is `reps` such calls."""
    import torch
    import synth
    import quantized_moe_router_b200 as qm
    reps = 50
    layers, bits = build_layers(w)
    lw = layers[0]
    nx = reps
    xs = torch.empty((nx, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    import synth.device as sd
    for s in range(nx):
        sd.hidden(w, s, 0, out=xs[s])
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    out = torch.empty((nx, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((nx, w.T, w.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((nx, w.T, w.k), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]

    def one_step(timed):
        for r in range(reps):
            flush.fill_(float(r))
            if timed:
                evs[r][0].record(st)
            qm.forward_decode(xs[r], lw.wr, lw.bias, lw.packed, w.I, w.E, w.k, ws, out=out[r], idx_out=idx[r],
                              w_out=wts[r])
            if timed:
                evs[r][1].record(st)

    W = max(args.warmup, 3)
    for _ in range(W):
        one_step(False)
    torch.cuda.synchronize()
    barrier(world)
    total = 0.0
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.steps):
            one_step(True)
            torch.cuda.synchronize()
            total += sum(a.elapsed_time(b) for a, b in evs)
    total = max_over_ranks(total, world)
    assert qm.device_status(ws) == qm.MOE_OK
    per_call_ms = total / (args.steps * reps)
    idn = idx.cpu().numpy()
    per = np.array([expert_bytes(w.H, w.I, b) for b in bits[0]], np.float64)
    expert_b = float(np.mean([per[np.unique(idn[r])].sum() for r in range(reps)]))
    layer_bytes = expert_b + w.E * w.H * 4 + 2 * w.T * w.H * 2
    hbm, _, _, peak_src = measured_peaks()
    achieved = layer_bytes / (per_call_ms * 1e-3) / 1e9
    res = {
        "metric": metric_name(w), "value": world * w.T / (per_call_ms * 1e-3), "unit": "tokens/s",
        "steps": args.steps, "warmup": W, "ms_per_step": total / args.steps, "tokens_per_step": reps * w.T,
        "config": dict(base_config(w, world),
                       l2=f"flushed: a {L2_FLUSH_BYTES >> 20} MB write before every timed call; each call timed "
                          f"alone with CUDA events, {reps} calls per bench step"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": None, "peak_source": peak_src,
                     "kernel": "decode megakernel (moe_expert_forward_decode)", "bytes_per_launch": layer_bytes,
                     "expert_bytes_per_launch": expert_b, "kernel_us_per_launch": per_call_ms * 1e3,
                     "expert_bytes_frac": expert_b / (per_call_ms * 1e-3) / 1e9 / hbm},
        "gpu_launches": args.steps * reps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_ties:
        import oracle
        res["routing"] = dict(tie_stats(oracle.get(), bf16_np(xs).reshape(nx * w.T, w.H), synth.router_weights(w, 0),
                                        synth.router_bias(w, 0), w.k, idn.reshape(-1, w.k),
                                        wts.cpu().numpy().reshape(-1, w.k)), calls=reps, band=TIE)
    if not args.no_e2e:
        xh = torch.empty((2, reps, w.T, w.H), dtype=torch.bfloat16).pin_memory()
        xh[0].copy_(xs.cpu())
        xh[1].copy_(torch.roll(xs, 1, 0).cpu())
        oh = torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
        e_total = 0.0
        ea, eb_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(args.steps):
            for r in range(reps):
                flush.fill_(float(r))
                ea.record(st)
                xd.copy_(xh[i % 2, r], non_blocking=True)
                qm.forward_decode(xd, lw.wr, lw.bias, lw.packed, w.I, w.E, w.k, ws, out=out[r])
                oh.copy_(out[r], non_blocking=True)
                eb_.record(st)
                eb_.synchronize()
                e_total += ea.elapsed_time(eb_)
        e_total = max_over_ranks(e_total, world)
        res["e2e"] = {"value": world * w.T * args.steps * reps / (e_total * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": reps * w.T * w.H * 2, "d2h_bytes_per_step": reps * w.T * w.H * 2,
                      "inputs": "2 pinned host batches alternating per step"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res.update(cpu_baselines(w))
    del layers, flush
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------ ours: prefill

def prefill_flops(w):
    """Expert-GEMM flops of one prefill layer: gate, up and down for every (token, expert) pair."""
    return 2.0 * w.T * w.k * 3 * w.I * w.H


def prefill_leg(args, w, world, rank):
    """One step = all w.T tokens through w.layers prefill layers (route + bucket + grouped GEMMs +
    combine per layer), fresh x per layer."""
    import torch
    import synth
    import synth.device as sd
    import quantized_moe_router_b200 as qm
    layers, _ = build_layers(w)
    xs = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    for l in range(w.layers):
        sd.hidden(w, 0, l, out=xs[l])
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_PREFILL)
    out = torch.empty((w.layers, w.T, w.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((w.layers, w.T, w.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((w.layers, w.T, w.k), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()

    def step(ev=None):
        for l, lw in enumerate(layers):
            if ev:
                ev[l][0].record(st)
            qm.prefill_route(xs[l], lw.wr, lw.bias, w.I, w.E, w.k, ws, idx_out=idx[l], w_out=wts[l])
            if ev:
                ev[l][1].record(st)
            qm.prefill_experts(xs[l], lw.packed, w.I, w.E, w.k, ws, out=out[l])
            if ev:
                ev[l][2].record(st)

    W = max(args.warmup, 3)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)
    nsteps = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(w.layers)] for _ in range(nsteps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(st)
        for i in range(nsteps):
            step(evs[i])
        e1.record(st)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    route_ms = float(np.mean([ev[0].elapsed_time(ev[1]) for evl in evs for ev in evl]))
    gemm_ms = float(np.mean([ev[1].elapsed_time(ev[2]) for evl in evs for ev in evl]))
    assert qm.device_status(ws) == qm.MOE_OK
    _, bf16, bf16_sus, peak_src = measured_peaks()
    achieved = prefill_flops(w) / (gemm_ms * 1e-3) / 1e12
    res = {
        "metric": metric_name(w), "value": world * w.T * nsteps / (ms * 1e-3), "unit": "tokens/s",
        "steps": nsteps, "warmup": W, "ms_per_step": ms / nsteps, "ms_per_layer": ms / nsteps / w.layers,
        "tokens_per_step": w.T, "route_ms_per_layer": route_ms, "experts_ms_per_layer": gemm_ms,
        "dtype": "fp16 tensor-core operands, fp32 accumulation (bf16 in and out)",
        "config": dict(base_config(w, world),
                       l2="no flush: each layer streams the weights of all its experts (453 MB > 126 MB L2)"),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                     "frac": achieved / bf16,
                     "frac_of_sustained": achieved / bf16_sus if bf16_sus else None,
                     "traffic": recorded_traffic("prefill_tc_grouped_prefill_t4096_h2048.txt", PREFILL_SOURCES)
                     if w.name == PREFILL_WORKLOAD else None,
                     "peak_source": peak_src + " (burst cuBLAS bf16; fp16 runs at the same tensor rate)",
                     "flops_per_launch": prefill_flops(w),
                     "kernel": "expert phase (moe_prefill_experts: grouped gate/up + down GEMMs, combine)",
                     "kernel_ms_per_launch": gemm_ms,
                     "whole_layer_frac": prefill_flops(w) / (ms / nsteps / w.layers * 1e-3) / 1e12 / bf16},
        "clocks": clk.summary(),
        "gpu_launches": nsteps * w.layers * PREFILL_LAUNCHES_PER_LAYER,
    }
    if rank == 0 and not args.no_ties:
        import oracle
        o = oracle.get()
        xb = bf16_np(xs)
        idn, wn = idx.cpu().numpy(), wts.cpu().numpy()
        parts = [tie_stats(o, xb[l], layers[l].wr.cpu().numpy(), synth.router_bias(w, l), w.k, idn[l], wn[l])
                 for l in range(w.layers)]
        res["routing"] = dict(merge_ties(parts), calls=w.layers, band=TIE)
    if not args.no_e2e:
        xh = torch.empty((2,) + tuple(xs.shape), dtype=torch.bfloat16).pin_memory()
        xh[0].copy_(xs.cpu())
        xh[1].copy_(torch.roll(xs, 1, 1).cpu())
        oh = torch.empty(tuple(out.shape), dtype=torch.bfloat16).pin_memory()
        for i in range(W):
            xs.copy_(xh[i % 2], non_blocking=True)
            step()
            oh.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ee0.record(st)
        for i in range(nsteps):
            xs.copy_(xh[i % 2], non_blocking=True)
            step()
            oh.copy_(out, non_blocking=True)
        ee1.record(st)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), world)
        res["e2e"] = {"value": world * w.T * nsteps / (e2e_ms * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": xs.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                      "inputs": "2 pinned host batches alternating per step"}
        del xh, oh
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res.update(cpu_baselines(w))
    del layers, xs, out
    torch.cuda.empty_cache()
    return res



# ------------------------------------------------------------------------------ next rows

# fp64 issue rate of the part: 148 SMs x 64 fp64 lanes x 1.965 GHz, one operation per lane and clock
FP64_OPS_PEAK = 148 * 64 * 1.965e9


def quantizer_leg():
    """moe_quantize_hqq on whole expert matrices (published defaults p = 0.7, beta = 10,
    kappa = 1.01, 20 steps): weights per second, and the fp64 operations of its definition per
    second against the fp64 issue rate. Per weight, an error pass is 10 operations (3 of them a
    division, rint and clamps counted as one each) and a zero pass 15 (2 divisions); a group
    that ran n steps did n error passes and at least n - 1 zero passes (counted: n - 1)."""
    import torch
    import oracle
    import synth
    import quantized_moe_router_b200 as qm
    res = {}
    gen = torch.Generator(device="cuda")
    for label, rows, cols, bits in (("gate_up_I512xH2048_64experts_int4", 64 * 512, 2048, 4),
                                    ("down_H2048xI512_64experts_int8", 64 * 2048, 512, 8),
                                    ("gate_up_I1024xH4096_16experts_int4", 16 * 1024, 4096, 4)):
        gen.manual_seed(rows + cols + bits)
        wt = (torch.randn((rows, cols), generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        qm.quantize_hqq(wt, bits, with_iters=True)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        with ClockSampler(torch.cuda.current_device()) as clk:
            e0.record()
            for _ in range(reps):
                codes, sc, zr, it = qm.quantize_hqq(wt, bits, with_iters=True)
            e1.record()
            torch.cuda.synchronize()
        t = e0.elapsed_time(e1) * 1e-3 / reps
        steps = it.to(torch.int64)
        ops = 64.0 * float((10 * steps + 15 * (steps - 1).clamp(min=0)).sum())
        ent = {"weights": rows * cols, "bits": bits, "ms": t * 1e3, "weights_per_s": rows * cols / t,
               "mean_steps": float(steps.float().mean()),
               "roofline": {"bound": "alu", "achieved": ops / t / 1e12, "peak": FP64_OPS_PEAK / 1e12,
                            "unit": "T fp64 op/s", "frac": ops / t / FP64_OPS_PEAK, "traffic": None,
                            "peak_source": "148 SMs x 64 fp64 lanes x 1.965 GHz (nominal issue rate)"},
               "clocks": clk.summary()}
        if label.startswith("gate_up_I512"):
            # stored zeros against the oracle on the first 512 rows (one expert's gate matrix)
            wb = wt[:512].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
            _, rs, rz, rit = oracle.get().hqq_quantize(wb, bits)
            z16 = zr[:512].cpu().numpy().view(np.uint16)
            zsame = synth.f16_bits_to_f64(z16) == synth.f16_bits_to_f64(rz)
            ent["oracle_check"] = {"groups": int(zsame.size), "zero_mismatch": int((~zsame).sum()),
                                   "scale_equal": bool(np.array_equal(sc[:512].cpu().numpy().view(np.uint16), rs)),
                                   "steps_equal": bool(np.array_equal(it[:512].cpu().numpy(), rit))}
        res[label] = ent
        del wt, codes, sc, zr, it
    torch.cuda.empty_cache()
    return res


def streamed_leg(slot_counts=(96, 256, 640), L=4, S=4):
    """Decode through an ExpertCache: the layers of the mixed 4/6/8-bit Zipf workload stay in
    pinned host memory, a device pool of `slots` experts serves the calls. Per call the routing
    names the experts (moe_route_topk), the missing ones are copied (moe_cache_commit) and the
    fused decode kernel reads them through the layer's cache header. Two schedules: serial
    (route, copy, compute per layer) and overlapped (the next layer's copies on a second stream
    while this layer computes; the benchmark's inputs are independent per layer, so the next
    layer's routing is known a layer ahead -- a model would need a predictor for it)."""
    import torch
    import synth
    import synth.device as sd
    import quantized_moe_router_b200 as qm
    w = synth.WORKLOADS["decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1"]
    host, wrs, biases, bits = [], [], [], []
    for l in range(L):
        b = synth.expert_bits(w, l)
        experts = [sd.expert_tensors(w, l, e, int(b[e])) for e in range(w.E)]
        host.append(qm.pack_layer(experts, w.H, w.I).cpu().pin_memory())
        del experts
        wrs.append(sd.router_weights(w, l))
        bb = synth.router_bias(w, l)
        biases.append(None if bb is None else torch.from_numpy(bb).cuda())
        bits.append(b)
    torch.cuda.empty_cache()
    xs = [[sd.hidden(w, s, l) for l in range(L)] for s in range(S + 1)]
    nbytes = [[expert_bytes(w.H, w.I, int(bits[l][e])) for e in range(w.E)] for l in range(L)]
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((w.T, w.k), dtype=torch.float32, device="cuda")
    # every call's routing, for the requests (the fused kernel routes again; the two must agree)
    routes = [[None] * L for _ in range(S + 1)]
    for s in range(S + 1):
        for l in range(L):
            qm.route_topk(xs[s][l], wrs[l], biases[l], w.k, idx_out=idx, w_out=wts)
            routes[s][l] = sorted(set(idx.cpu().flatten().tolist()))
    comp = torch.cuda.current_stream()
    cst = torch.cuda.Stream()
    res = {}
    for slots in slot_counts:
        ent = {}
        for sched in ("serial", "overlapped"):
            cache = qm.ExpertCache(host, slots, keep_recent=2)
            outside = 0

            def run(s, count):
                nonlocal outside
                loaded = 0
                pk = [None] * L
                ev = [None] * L

                def fetch(l, stream):
                    nonlocal loaded
                    le, _ = cache.request(l, routes[s][l])
                    loaded += sum(nbytes[l][e] for e in le)
                    pk[l] = cache.commit(stream)
                    ev[l] = torch.cuda.Event()
                    ev[l].record(stream)
                done = [None] * L
                if sched == "overlapped":
                    cst.wait_stream(comp)
                    fetch(0, cst)
                for l in range(L):
                    if sched == "serial":
                        fetch(l, comp)
                    comp.wait_event(ev[l])
                    qm.forward_decode(xs[s][l], wrs[l], biases[l], pk[l], w.I, w.E, w.k, ws, out=out,
                                      idx_out=idx, w_out=wts, stream=comp)
                    done[l] = torch.cuda.Event()
                    done[l].record(comp)
                    if sched == "overlapped" and l + 1 < L:
                        # keep_recent = 2 protects this layer's experts and the next one's; the
                        # copies wait until the call before this one has read its experts
                        if l >= 1:
                            cst.wait_event(done[l - 1])
                        fetch(l + 1, cst)
                    if count and not set(idx.cpu().flatten().tolist()) <= set(routes[s][l]):
                        outside += 1
                return loaded
            run(S, False)   # warm: the first pass fills the pool
            torch.cuda.synchronize()
            h0 = cache.stats()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(torch.cuda.current_device()) as clk:
                t0 = time.perf_counter()
                e0.record(comp)
                loaded = sum(run(s, False) for s in range(S))
                e1.record(comp)
                torch.cuda.synchronize()
                wall = time.perf_counter() - t0
            dev = e0.elapsed_time(e1) * 1e-3
            h1 = cache.stats()
            hits, miss = h1["hits"] - h0["hits"], h1["misses"] - h0["misses"]
            # the fused kernel's own routing against the requests, outside the timed region
            run(S, True)
            torch.cuda.synchronize()
            assert qm.device_status(ws) == qm.MOE_OK
            ent[sched] = {"tokens_per_s": w.T * S / dev, "ms_per_token_step": dev / S * 1e3,
                          "host_GBps": loaded / dev / 1e9, "hit_rate": hits / max(1, hits + miss),
                          "expert_misses": miss, "wall_s": wall, "calls_outside_request": outside,
                          "clocks": clk.summary()}
            cache.close()
        res[f"slots_{slots}"] = ent
    return {"workload": f"{w.name} (first {L} layers in pinned host memory, {w.T} tokens per call, {S} steps)",
            "experts_in_play": L * w.E, "schedules": res}


def next_rows_leg(args, world, rank):
    import dataclasses
    import synth
    pw = synth.WORKLOADS[PREFILL_WORKLOAD]
    mixed = dataclasses.replace(pw, name="prefill_t4096_l2_h2048_e256_k8_i512_mixed468", mixed_bits=True, layers=2)
    a2 = argparse.Namespace(**vars(args))
    a2.no_cpu_baseline = True
    a2.steps = 40   # ~50 ms timed: enough clock samples

    def guarded(fn, *fa):
        # a failing next row is reported in its entry and does not take the benchmark line down
        try:
            return fn(*fa)
        except Exception as ex:  # noqa: BLE001
            return {"error": f"{type(ex).__name__}: {ex}"[:300]}
    return {"quantizer": guarded(quantizer_leg),
            "streamed_decode": guarded(streamed_leg),
            "mixed_prefill": guarded(prefill_leg, a2, mixed, world, rank)}


def leg(args, w, world, rank):
    if w.mode == "prefill":
        return prefill_leg(args, w, world, rank)
    if w.layers == 1 and w.steps == 1:
        return single_leg(args, w, world, rank)
    return decode_leg(args, w, world, rank)


def run_ours(args, w):
    import synth
    rank, world, _ = dist_setup()
    head = leg(args, w, world, rank)
    others = {}
    if not args.only:
        for name in synth.WORKLOAD_ORDER:
            if name != w.name:
                others[name] = leg(args, synth.WORKLOADS[name], world, rank)
    dtype = "bf16" if w.mode == "decode" else "fp16"
    line = {"metric": head.pop("metric"), "value": head.pop("value"), "unit": head.pop("unit"), "n_gpus": world,
            "steps": head.pop("steps"), "warmup": head.pop("warmup"), "ms_per_step": head.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded SplitMix64 / Box-Muller inputs of the workload recipe)",
            "config": head.pop("config")}
    line.update(head)
    if others:
        line["configs"] = others
    if args.next or not args.only:
        line["next_rows"] = next_rows_leg(args, world, rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


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
