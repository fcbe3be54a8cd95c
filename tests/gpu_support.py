"""Helpers for the GPU tests: device copies of synthetic / hand-built layers."""
from __future__ import annotations

import numpy as np
import torch

import synth
import synth.device as sd
import quantized_moe_router_b200 as qm


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def upload_expert(ex: dict) -> dict:
    return {"bits": ex["bits"],
            "codes": [torch.from_numpy(np.ascontiguousarray(c)).cuda() for c in ex["codes"]],
            "scale": [torch.from_numpy(np.ascontiguousarray(s).view(np.int16)).cuda() for s in ex["scale"]],
            "zero": [torch.from_numpy(np.ascontiguousarray(z).view(np.int16)).cuda() for z in ex["zero"]]}


class SynthLayer:
    """One layer of a synthetic workload on the device (packed), plus host-side accessors."""

    def __init__(self, w: synth.Workload, layer: int):
        self.w, self.layer = w, layer
        self.bits = synth.expert_bits(w, layer)
        self.wr = sd.router_weights(w, layer)
        b = synth.router_bias(w, layer)
        self.bias_np = b
        self.bias = None if b is None else torch.from_numpy(b).cuda()
        experts = [sd.expert_tensors(w, layer, e, int(self.bits[e])) for e in range(w.E)]
        self.packed = qm.pack_layer(experts, w.H, w.I)
        torch.cuda.synchronize()
        del experts
        self._wr_np = None

    @property
    def wr_np(self):
        if self._wr_np is None:
            self._wr_np = synth.router_weights(self.w, self.layer)
        return self._wr_np

    def expert_fn(self, e: int) -> dict:
        return synth.expert_tensors(self.w, self.layer, e, int(self.bits[e]))


class HandLayer:
    """A layer from explicit numpy experts (canonical form) and router weights."""

    def __init__(self, experts_np, wr_np, bias_np, H, I):
        self.experts_np = experts_np
        self.wr_np = np.ascontiguousarray(wr_np, np.float32)
        self.bias_np = None if bias_np is None else np.ascontiguousarray(bias_np, np.float32)
        self.wr = torch.from_numpy(self.wr_np).cuda()
        self.bias = None if bias_np is None else torch.from_numpy(self.bias_np).cuda()
        self.packed = qm.pack_layer([upload_expert(e) for e in experts_np], H, I)
        torch.cuda.synchronize()

    def expert_fn(self, e: int) -> dict:
        return self.experts_np[e]
