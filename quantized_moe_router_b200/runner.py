"""Launch sequencing for a stack of decode layers: one CUDA graph per step.

Plumbing only: the graph holds one moe_expert_forward_decode launch per layer (each a
programmatic-dependent launch, so layer l+1's CTAs are scheduled while layer l finishes) and
nothing else; all arithmetic is in the CUDA library.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import MODE_DECODE, MODE_PREFILL, forward_decode, forward_prefill, workspace


class LayerWeights:
    """Device tensors of one layer: router [E x H] fp32, optional bias [E], packed experts."""

    def __init__(self, wr: torch.Tensor, bias: Optional[torch.Tensor], packed: torch.Tensor):
        self.wr, self.bias, self.packed = wr, bias, packed


class DecodeStack:
    """L decode layers of the same shape sharing one workspace, replayed as one CUDA graph.

    x_in[l] / out[l] are fixed device buffers (T x H bf16) that the graph reads and writes.
    """

    def __init__(self, layers: Sequence[LayerWeights], T: int, H: int, I: int, E: int, k: int,
                 device="cuda", with_routing_outputs: bool = True):
        self.layers = list(layers)
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        L = len(self.layers)
        self.ws = workspace(T, H, I, E, k, MODE_DECODE, device)
        self.x_in = torch.zeros((L, T, H), dtype=torch.bfloat16, device=device)
        self.out = torch.zeros((L, T, H), dtype=torch.bfloat16, device=device)
        self.idx = torch.zeros((L, T, k), dtype=torch.int32, device=device) if with_routing_outputs else None
        self.wts = torch.zeros((L, T, k), dtype=torch.float32, device=device) if with_routing_outputs else None
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def launch(self, stream=None):
        for l, lw in enumerate(self.layers):
            forward_decode(self.x_in[l], lw.wr, lw.bias, lw.packed, self.I, self.E, self.k, self.ws,
                           out=self.out[l], idx_out=None if self.idx is None else self.idx[l],
                           w_out=None if self.wts is None else self.wts[l], stream=stream)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.launch()          # warm-up outside the graph (also sets kernel attributes)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch()
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()


class DecodeRun:
    """S decode steps through L layers of the same shape, replayed as one CUDA graph of S * L
    launches (step-major: every layer of step 0, then step 1, ...).

    x is the caller's device tensor [S, L, T, H] bf16 that the graph reads in place (copy new
    hidden states into it between replays); out [S, L, T, H], idx [S, L, T, k] and
    wts [S, L, T, k] hold every call's results after a replay. One workspace serves all calls,
    so the calls are ordered, as the layers of a model are.
    """

    def __init__(self, layers: Sequence[LayerWeights], x: torch.Tensor, I: int, E: int, k: int,
                 with_routing_outputs: bool = True):
        S, L, T, H = x.shape
        if L != len(layers):
            raise ValueError(f"x has {L} layers, {len(layers)} layer weights given")
        self.layers = list(layers)
        self.x = x
        self.S, self.L, self.T, self.H, self.I, self.E, self.k = S, L, T, H, I, E, k
        dev = x.device
        self.ws = workspace(T, H, I, E, k, MODE_DECODE, dev)
        self.out = torch.zeros((S, L, T, H), dtype=torch.bfloat16, device=dev)
        self.idx = torch.zeros((S, L, T, k), dtype=torch.int32, device=dev) if with_routing_outputs else None
        self.wts = torch.zeros((S, L, T, k), dtype=torch.float32, device=dev) if with_routing_outputs else None
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def launch(self, stream=None):
        for s in range(self.S):
            for l, lw in enumerate(self.layers):
                forward_decode(self.x[s, l], lw.wr, lw.bias, lw.packed, self.I, self.E, self.k, self.ws,
                               out=self.out[s, l], idx_out=None if self.idx is None else self.idx[s, l],
                               w_out=None if self.wts is None else self.wts[s, l], stream=stream)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.launch()          # warm-up outside the graph (also sets kernel attributes)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch()
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    @property
    def launches(self) -> int:
        return self.S * self.L


class PrefillStack:
    """L prefill layers of the same shape sharing one workspace, launched back to back."""

    def __init__(self, layers: Sequence[LayerWeights], T: int, H: int, I: int, E: int, k: int, device="cuda"):
        self.layers = list(layers)
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        L = len(self.layers)
        self.ws = workspace(T, H, I, E, k, MODE_PREFILL, device)
        self.x_in = torch.zeros((L, T, H), dtype=torch.bfloat16, device=device)
        self.out = torch.zeros((L, T, H), dtype=torch.bfloat16, device=device)

    def launch(self, stream=None, idx_out: Optional[torch.Tensor] = None, w_out: Optional[torch.Tensor] = None):
        """idx_out / w_out: optional [L, T, k] tensors that receive every layer's routing."""
        for l, lw in enumerate(self.layers):
            forward_prefill(self.x_in[l], lw.wr, lw.bias, lw.packed, self.I, self.E, self.k, self.ws,
                            out=self.out[l], idx_out=None if idx_out is None else idx_out[l],
                            w_out=None if w_out is None else w_out[l], stream=stream)


def forward_through_cache(cache, layer: int, x: torch.Tensor, w_router: torch.Tensor,
                          bias: Optional[torch.Tensor], I: int, E: int, k: int, ws: torch.Tensor,
                          mode: int = MODE_DECODE, retries: int = 2):
    """One layer call whose experts come through an ExpertCache, on the current stream.

    Prefill: routing and bucketing first (prefill_route), then exactly the experts the buckets
    name are made resident and the grouped GEMMs read them through the layer's cache header.
    Decode: the fused kernel routes again inside; the experts of a separate routing call are made
    resident, and the call's own idx_out is checked against them. An expert outside them (the two
    routings can differ only where two logits tie to fp32 rounding) is loaded and the call
    repeated. Returns (out, idx, w). Plumbing only: every step runs in the library."""
    from . import prefill_experts, prefill_route, route_topk
    T, H = x.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    wts = torch.empty((T, k), dtype=torch.float32, device=x.device)
    if mode == MODE_PREFILL:
        prefill_route(x, w_router, bias, I, E, k, ws, idx_out=idx, w_out=wts)
        packed = cache.prepare(layer, sorted(set(idx.cpu().flatten().tolist())))
        return prefill_experts(x, packed, I, E, k, ws), idx, wts
    route_topk(x, w_router, bias, k, idx_out=idx, w_out=wts)
    want = set(idx.cpu().flatten().tolist())
    for _ in range(retries + 1):
        packed = cache.prepare(layer, sorted(want))
        out = forward_decode(x, w_router, bias, packed, I, E, k, ws, idx_out=idx, w_out=wts)
        used = set(idx.cpu().flatten().tolist())
        if used <= want:
            return out, idx, wts
        want |= used
    raise RuntimeError("the decode call kept selecting experts outside the cache request")
