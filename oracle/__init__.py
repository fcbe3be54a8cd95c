"""fp64 CPU oracle of the quantized MoE expert block (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` import
this package. The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, compiled with
``-ffp-contract=off`` and no fast-math); this file only marshals numpy arrays into it.
It shares no code with the CUDA library.

Pins (what ties the oracle to something other than itself) are in
``tests/test_oracle_pins.py``; every public function here is pinned there.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "moe_oracle.c")
LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fopenmp"]


def build(src: str = SRC, out: str = LIB, extra: Sequence[str] = ()) -> str:
    """Compile the oracle (or a variant of its source, for the pin-sensitivity tests)."""
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


# Published defaults of the HQQ zero-point optimiser (l_p norm, initial beta, beta growth
# per iteration, iteration cap).
HQQ_P, HQQ_BETA, HQQ_KAPPA, HQQ_ITERS = 0.7, 10.0, 1.01, 20


class _Expert(C.Structure):
    _fields_ = [("codes", C.c_void_p * 3), ("scale", C.c_void_p * 3), ("zero", C.c_void_p * 3),
                ("bits", C.c_int32)]


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str = LIB):
        if path == LIB and (not os.path.exists(LIB)
                            or os.path.getmtime(LIB) < os.path.getmtime(SRC)):
            build()
        self.lib = C.CDLL(path)
        L = self.lib
        vp, i32 = C.c_void_p, C.c_int
        L.oracle_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.oracle_topk.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_expert_ffn.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
        L.oracle_combine.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
        L.oracle_moe_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_weight.argtypes = [vp, i32, i32, i32, i32, i32]
        L.oracle_weight.restype = C.c_double
        L.oracle_max_threads.restype = C.c_int
        L.oracle_set_threads.argtypes = [C.c_int]
        f64 = C.c_double
        L.oracle_f64_to_f16.argtypes = [f64]
        L.oracle_f64_to_f16.restype = C.c_uint16
        L.oracle_hqq_shrink.argtypes = [f64, f64, f64]
        L.oracle_hqq_shrink.restype = f64
        L.oracle_hqq_group.argtypes = [vp, i32, f64, f64, f64, i32, vp, vp, vp, vp, vp, vp]
        L.oracle_hqq_quantize.argtypes = [vp, i32, i32, i32, f64, f64, f64, i32, vp, vp, vp, vp]
        L.oracle_hqq_codes.argtypes = [vp, i32, i32, i32, vp, vp, vp]

    # -------------------------------------------------------------- marshalling helpers
    @staticmethod
    def _expert_struct(ex: Optional[dict], keep: list) -> _Expert:
        s = _Expert()
        if ex is None:
            s.bits = 0
            return s
        for m in range(3):
            c = np.ascontiguousarray(ex["codes"][m], dtype=np.uint8)
            sc = np.ascontiguousarray(ex["scale"][m], dtype=np.uint16)
            z = np.ascontiguousarray(ex["zero"][m], dtype=np.uint16)
            keep += [c, sc, z]
            s.codes[m], s.scale[m], s.zero[m] = _ptr(c), _ptr(sc), _ptr(z)
        s.bits = int(ex["bits"])
        return s

    def _expert_table(self, experts: Sequence[Optional[dict]], keep: list):
        arr = (_Expert * len(experts))()
        for e, ex in enumerate(experts):
            arr[e] = self._expert_struct(ex, keep)
        return arr

    def threads(self) -> int:
        return self.lib.oracle_max_threads()

    def set_threads(self, n: int) -> None:
        self.lib.oracle_set_threads(n)

    # -------------------------------------------------------------- API
    def router_logits(self, x_bf16: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray]):
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        wr = np.ascontiguousarray(wr, dtype=np.float32)
        T, H = x.shape
        E = wr.shape[0]
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        out = np.empty((T, E), np.float64)
        self.lib.oracle_router_logits(_ptr(x), _ptr(wr), None if b is None else _ptr(b),
                                      T, H, E, _ptr(out))
        return out

    def topk(self, logits: np.ndarray, k: int):
        l = np.ascontiguousarray(logits, dtype=np.float64)
        T, E = l.shape
        idx = np.empty((T, k), np.int32)
        w = np.empty((T, k), np.float64)
        self.lib.oracle_topk(_ptr(l), T, E, k, _ptr(idx), _ptr(w))
        return idx, w

    def expert_ffn(self, x_tok_bf16: np.ndarray, ex: dict, H: int, I: int):
        """One token through one expert: returns (g, u, h, y) in fp64."""
        keep: list = []
        s = self._expert_struct(ex, keep)
        x = np.ascontiguousarray(x_tok_bf16, dtype=np.uint16).reshape(H)
        g, u, h = (np.empty(I, np.float64) for _ in range(3))
        y = np.empty(H, np.float64)
        self.lib.oracle_expert_ffn(_ptr(x), C.addressof(s), H, I, _ptr(g), _ptr(u), _ptr(h),
                                   _ptr(y))
        return g, u, h, y

    def weight(self, ex: dict, m: int, rows: int, cols: int, r: int, c: int) -> float:
        keep: list = []
        s = self._expert_struct(ex, keep)
        return self.lib.oracle_weight(C.addressof(s), m, rows, cols, r, c)

    def combine(self, x_bf16: np.ndarray, experts: Sequence[Optional[dict]], H: int, I: int,
                idx: np.ndarray, w: np.ndarray):
        keep: list = []
        tab = self._expert_table(experts, keep)
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        w = np.ascontiguousarray(w, dtype=np.float64)
        T, k = idx.shape
        for e in np.unique(idx):
            if experts[int(e)] is None:
                raise ValueError(f"expert {int(e)} selected but not supplied")
        out = np.empty((T, H), np.float64)
        self.lib.oracle_combine(_ptr(x), C.addressof(tab), T, H, I, len(experts), k, _ptr(idx),
                                _ptr(w), _ptr(out))
        return out

    def forward(self, x_bf16, wr, bias, experts: Sequence[Optional[dict]], H: int, I: int,
                k: int):
        """Whole block: returns (out [T x H] fp64, idx [T x k], w [T x k], logits [T x E])."""
        logits = self.router_logits(x_bf16, wr, bias)
        idx, w = self.topk(logits, k)
        out = self.combine(x_bf16, experts, H, I, idx, w)
        return out, idx, w, logits

    # -------------------------------------------------------------- quantiser
    def f64_to_f16(self, v: float) -> int:
        """IEEE binary16 bits of v, round to nearest even."""
        return int(self.lib.oracle_f64_to_f16(float(v)))

    def hqq_shrink(self, x: float, beta: float, p: float) -> float:
        """The generalised soft threshold of the zero-point iteration."""
        return float(self.lib.oracle_hqq_shrink(float(x), float(beta), float(p)))

    def hqq_group(self, w: np.ndarray, bits: int, p: float = HQQ_P, beta: float = HQQ_BETA,
                  kappa: float = HQQ_KAPPA, iters: int = HQQ_ITERS):
        """One group of 64 fp64 weights: (s16 bits, z16 bits, codes [64], z trace, err trace)."""
        w = np.ascontiguousarray(w, dtype=np.float64).reshape(64)
        s16, z16 = C.c_uint16(), C.c_uint16()
        q = np.empty(64, np.uint8)
        zt = np.empty(max(iters, 1), np.float64)
        et = np.empty(max(iters, 1), np.float64)
        ran = C.c_int()
        self.lib.oracle_hqq_group(_ptr(w), bits, p, beta, kappa, iters, C.addressof(s16),
                                  C.addressof(z16), _ptr(q), _ptr(zt), _ptr(et),
                                  C.addressof(ran))
        return s16.value, z16.value, q, zt[:ran.value].copy(), et[:ran.value].copy()

    def hqq_quantize(self, w_bf16: np.ndarray, bits: int, p: float = HQQ_P,
                     beta: float = HQQ_BETA, kappa: float = HQQ_KAPPA, iters: int = HQQ_ITERS):
        """bf16 bits [rows x cols] -> (codes uint8 [rows x cols], s16 bits, z16 bits
        [rows x cols/64], iterations run per group [rows x cols/64])."""
        w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
        rows, cols = w.shape
        if cols % 64 or bits not in (4, 6, 8) or iters < 0:
            raise ValueError("cols must be a multiple of 64, bits 4/6/8, iters >= 0")
        q = np.empty((rows, cols), np.uint8)
        s16 = np.empty((rows, cols // 64), np.uint16)
        z16 = np.empty((rows, cols // 64), np.uint16)
        ran = np.empty((rows, cols // 64), np.int32)
        self.lib.oracle_hqq_quantize(_ptr(w), rows, cols, bits, p, beta, kappa, iters, _ptr(q),
                                     _ptr(s16), _ptr(z16), _ptr(ran))
        return q, s16, z16, ran

    def hqq_codes(self, w_bf16: np.ndarray, bits: int, s16: np.ndarray, z16: np.ndarray):
        """Nearest codes of bf16 weights on the grid of the given fp16 scale and zero bits."""
        w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
        rows, cols = w.shape
        s = np.ascontiguousarray(s16, dtype=np.uint16).reshape(rows, cols // 64)
        z = np.ascontiguousarray(z16, dtype=np.uint16).reshape(rows, cols // 64)
        q = np.empty((rows, cols), np.uint8)
        self.lib.oracle_hqq_codes(_ptr(w), rows, cols, bits, _ptr(s), _ptr(z), _ptr(q))
        return q


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
