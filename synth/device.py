"""Device-side generation of the synthetic inputs (same values as the numpy functions in
``synth``; the GPU tests check the two agree bit for bit). Input plumbing only."""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import torch

import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "csrc", "synth.cu")
LIB = os.path.join(_HERE, "libmoe_synth.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build() -> str:
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-Xcompiler", "-fPIC",
                    "-shared", "-o", LIB, SRC], check=True)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
            build()
        L = C.CDLL(LIB)
        L.synth_fill.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_int, C.c_int, C.c_void_p]
        L.synth_bytes.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_void_p]
        _lib = L
    return _lib


def _st():
    return torch.cuda.current_stream().cuda_stream


def _fill(out: torch.Tensor, key: int, kind: int, param: int = 0, start: int = 0) -> torch.Tensor:
    rc = lib().synth_fill(out.data_ptr(), key, start, out.numel(), kind, param, _st())
    if rc != 0:
        raise RuntimeError(f"synth_fill failed ({rc})")
    return out


def hidden(w: synth.Workload, step: int, layer: int, out=None, device="cuda") -> torch.Tensor:
    if out is None:
        out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=device)
    return _fill(out, synth.stream_key(w.seed, synth.K_X, step, layer), 0)


def router_weights(w: synth.Workload, layer: int, out=None, device="cuda") -> torch.Tensor:
    if out is None:
        out = torch.empty((w.E, w.H), dtype=torch.float32, device=device)
    return _fill(out, synth.stream_key(w.seed, synth.K_WR, layer), 1, w.H)


def expert_tensors(w: synth.Workload, layer: int, e: int, bits: int, device="cuda") -> dict:
    """Canonical tensors of one expert on the device (codes uint8, scale/zero fp16)."""
    out = {"bits": bits, "codes": [], "scale": [], "zero": []}
    for m in range(3):
        rows, cols = w.matrix_shape(m)
        codes = torch.empty((rows, cols * bits // 8), dtype=torch.uint8, device=device)
        rc = lib().synth_bytes(codes.data_ptr(), synth.stream_key(w.seed, synth.K_CODES, layer, e, m), 0,
                               codes.numel(), _st())
        if rc != 0:
            raise RuntimeError(f"synth_bytes failed ({rc})")
        s = torch.empty((rows, cols // synth.GROUP), dtype=torch.float16, device=device)
        z = torch.empty_like(s)
        _fill(s, synth.stream_key(w.seed, synth.K_SCALE, layer, e, m), 2, bits)
        _fill(z, synth.stream_key(w.seed, synth.K_ZERO, layer, e, m), 3, bits)
        out["codes"].append(codes)
        out["scale"].append(s)
        out["zero"].append(z)
    return out
