"""Seeded synthetic inputs for the quantized MoE expert block.

This module is input plumbing shared by the fp64 oracle (under ``oracle/``) and the CUDA
library (``quantized_moe_router_b200``). It holds none of the expert block's arithmetic: no
routing, no dequantisation, no matmul. It only draws random numbers and rounds them to the
storage types the block consumes.

Generator (identical on the host, here, and on the device, ``synth/csrc/synth.cu``):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014) used counter-style: draw ``i`` of a stream with key ``K`` is the (i+1)-th
  output of SplitMix64 started from state ``K``, i.e. ``mix64(K + (i+1)*GAMMA)``.
* One key per tensor: ``key = mix64(seed*GAMMA + stream_id*GAMMA2)`` with ``stream_id`` made
  of (kind, a, b, c) fields, so every element of every tensor is a pure function of
  (seed, tensor, index) and any slice can be regenerated without generating the rest.
* Open uniform ``u = (2*(d >> 12) + 1) * 2**-53`` in (0, 1), exact in fp64.
* Normals by the Box-Muller transform (Box & Muller, 1958), cosine branch:
  ``z_i = sqrt(-2 ln u(d_2i)) * cos(2 pi u(d_2i+1))``. The logarithm is the atanh series
  ``ln m = 2 artanh((m-1)/(m+1))`` (Abramowitz & Stegun 4.1.27) after splitting off the
  binary exponent; the cosine is the Taylor series of cos / sin after an exact reduction of
  the turn fraction to [0, 1/8]. Both are written here with a fixed order of IEEE-754
  double operations (no fused multiply-add), and the CUDA side evaluates the same
  operations in the same order, so host and device produce the same bits.
* Storage rounding: double -> fp32 round-to-nearest-even (RNE); fp32 -> bf16 RNE;
  fp32 -> fp16 RNE. (fp16/bf16 values are therefore rounded twice, by definition.)

Workload recipes (the synthetic configurations, with the readings taken where the recipe
text is open):

* x ~ N(0, 1) rounded to bf16, a fresh draw per (step, layer).
* router weights W_r ~ N(0, 1/H) (second argument = variance), fp32, [E x H] row-major.
* codes uniform on 0..2^b-1: the canonical packed byte arrays are filled with uniform random
  bytes, which makes every b-bit field uniform.
* scale = |N(0, 0.02)| + 1e-3 (variance 0.02) rounded to fp16; for b != 4 it is multiplied
  by 15/(2^b - 1) before rounding so that dequantised magnitudes match across widths.
* zero ~ continuous uniform on [0, 2^b - 1], rounded to fp16.
* mixed widths: per layer a seeded shuffle of the experts gives the first round(0.1 E)
  experts 8 bits, the next round(0.3 E) 6 bits, the rest 4 bits.
* Zipf(1.1) popularity: a seeded permutation ranks the experts 1..E and the router bias
  is ``-1.1 * ln(rank)``, added to the logits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
GAMMA2 = 0xD1B54A32D192ED03

# stream kinds
K_X, K_WR, K_CODES, K_SCALE, K_ZERO, K_BITS, K_ZIPF = 1, 2, 3, 4, 5, 6, 7

# series constants, written as hex so the CUDA side embeds exactly the same doubles
LN2 = float.fromhex("0x1.62e42fefa39efp-1")
TWO_PI = float.fromhex("0x1.921fb54442d18p+2")
SQRT2 = float.fromhex("0x1.6a09e667f3bcdp+0")
SQRT_0_02 = float.fromhex("0x1.21a1851ff630ap-3")
# 1/(2n+1), n = 0..11
ATANH_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "0x1.5555555555555p-2", "0x1.999999999999ap-3",
    "0x1.2492492492492p-3", "0x1.c71c71c71c71cp-4", "0x1.745d1745d1746p-4",
    "0x1.3b13b13b13b14p-4", "0x1.1111111111111p-4", "0x1.e1e1e1e1e1e1ep-5",
    "0x1.af286bca1af28p-5", "0x1.8618618618618p-5", "0x1.642c8590b2164p-5")]
# (-1)^n/(2n)!, n = 0..10
COS_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.0000000000000p-1", "0x1.5555555555555p-5",
    "-0x1.6c16c16c16c17p-10", "0x1.a01a01a01a01ap-16", "-0x1.27e4fb7789f5cp-22",
    "0x1.1eed8eff8d898p-29", "-0x1.93974a8c07c9dp-37", "0x1.ae7f3e733b81fp-45",
    "-0x1.6827863b97d97p-53", "0x1.e542ba4020225p-62")]
# (-1)^n/(2n+1)!, n = 0..10
SIN_C = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.5555555555555p-3", "0x1.1111111111111p-7",
    "-0x1.a01a01a01a01ap-13", "0x1.71de3a556c734p-19", "-0x1.ae64567f544e4p-26",
    "0x1.6124613a86d09p-33", "-0x1.ae7f3e733b81fp-41", "0x1.952c77030ad4ap-49",
    "-0x1.2f49b46814157p-57", "0x1.71b8ef6dcf572p-66")]


# ----------------------------------------------------------------------------- SplitMix64

def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int."""
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_id(kind: int, a: int = 0, b: int = 0, c: int = 0) -> int:
    """64-bit stream id: kind (8 bits) | a (20 bits) | b (20 bits) | c (16 bits)."""
    assert 0 <= kind < 256 and 0 <= a < (1 << 20) and 0 <= b < (1 << 20) and 0 <= c < (1 << 16)
    return (kind << 56) | (a << 36) | (b << 16) | c


def stream_key(seed: int, kind: int, a: int = 0, b: int = 0, c: int = 0) -> int:
    return mix64_int((seed * GAMMA + stream_id(kind, a, b, c) * GAMMA2) & M64)


def draws(key: int, start: int, n: int) -> np.ndarray:
    """Draws start..start+n-1 of the stream with key ``key`` (uint64)."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + i * np.uint64(GAMMA))


def uniform_open(d: np.ndarray) -> np.ndarray:
    """(2*(d>>12)+1) * 2^-53: a dyadic uniform strictly inside (0, 1)."""
    return ((d >> np.uint64(12)).astype(np.float64) * 2.0 + 1.0) * (2.0 ** -53)


# ----------------------------------------------------------------------------- own ln / cos

def ln_series(u: np.ndarray) -> np.ndarray:
    """ln(u) for normal positive doubles: u = m 2^e, m in [sqrt(1/2), sqrt(2)),
    ln m = 2 artanh(t), t = (m-1)/(m+1), artanh by its odd power series (Horner in t^2)."""
    bits = u.view(np.uint64)
    e = ((bits >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64) - 1023
    m = ((bits & np.uint64(0x000FFFFFFFFFFFFF)) | np.uint64(0x3FF0000000000000)).view(np.float64)
    big = m > SQRT2
    m = np.where(big, m * 0.5, m)
    e = np.where(big, e + 1, e)
    t = (m - 1.0) / (m + 1.0)
    t2 = t * t
    p = np.full_like(t, ATANH_C[-1])
    for c in ATANH_C[-2::-1]:
        p = p * t2 + c
    ln_m = 2.0 * (t * p)
    return e.astype(np.float64) * LN2 + ln_m


def cos_turns(v: np.ndarray) -> np.ndarray:
    """cos(2 pi v) for v in (0, 1): exact reduction to w in [0, 1/4], then the Taylor series
    of cos (w <= 1/8) or of sin at the complementary angle (w > 1/8)."""
    v = np.where(v > 0.5, 1.0 - v, v)
    neg = v > 0.25
    v = np.where(neg, 0.5 - v, v)
    use_cos = v <= 0.125
    a = TWO_PI * np.where(use_cos, v, 0.25 - v)
    a2 = a * a
    pc = np.full_like(a, COS_C[-1])
    for c in COS_C[-2::-1]:
        pc = pc * a2 + c
    ps = np.full_like(a, SIN_C[-1])
    for c in SIN_C[-2::-1]:
        ps = ps * a2 + c
    ps = a * ps
    r = np.where(use_cos, pc, ps)
    return np.where(neg, -r, r)


def normals(key: int, start: int, n: int) -> np.ndarray:
    """Standard normals start..start+n-1 of stream ``key`` (fp64)."""
    d = draws(key, 2 * start, 2 * n)
    u1 = uniform_open(d[0::2])
    u2 = uniform_open(d[1::2])
    return np.sqrt(-2.0 * ln_series(u1)) * cos_turns(u2)


def uniforms(key: int, start: int, n: int) -> np.ndarray:
    return uniform_open(draws(key, start, n))


def random_bytes(key: int, start_byte: int, nbytes: int) -> np.ndarray:
    """Bytes start_byte.. of the stream: byte j is byte (j mod 8) (little-endian) of draw j//8."""
    if nbytes == 0:
        return np.zeros(0, np.uint8)
    w0 = start_byte // 8
    w1 = (start_byte + nbytes + 7) // 8
    d = draws(key, w0, w1 - w0)
    b = d.astype("<u8").view(np.uint8)
    off = start_byte - 8 * w0
    return b[off:off + nbytes].copy()


# ----------------------------------------------------------------------------- storage rounding

def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(np.asarray(v, dtype=np.float64).astype(np.float32))


def to_f16_bits(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------- canonical packing

GROUP = 64


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Canonical code layout: rows x (cols*bits/8) bytes. Group g of a row (codes 64g..64g+63)
    is a block of 8*bits bytes; code j of the group occupies bits [j*bits, (j+1)*bits) of that
    block read as one little-endian bit string (bit 0 = LSB of the first byte)."""
    q = np.asarray(q)
    rows, cols = q.shape
    assert cols % GROUP == 0 and bits in (4, 6, 8)
    assert q.min(initial=0) >= 0 and q.max(initial=0) < (1 << bits)
    qb = ((q.astype(np.uint16)[..., None] >> np.arange(bits, dtype=np.uint16)) & 1).astype(np.uint8)
    flat = qb.reshape(rows, cols * bits)  # LSB-first bit string per row (groups are contiguous)
    return np.packbits(flat, axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, bits: int, cols: int) -> np.ndarray:
    """Inverse of pack_codes (used by tests to build dense reference matrices)."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    flat = np.unpackbits(packed, axis=1, bitorder="little")[:, :cols * bits]
    qb = flat.reshape(rows, cols, bits).astype(np.uint16)
    return (qb << np.arange(bits, dtype=np.uint16)).sum(axis=2).astype(np.int64)


# ----------------------------------------------------------------------------- workloads

@dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the MoE expert block."""
    name: str
    mode: str          # "decode" or "prefill"
    T: int             # tokens per layer call
    H: int             # hidden size
    E: int             # experts
    k: int             # experts per token
    I: int             # expert intermediate size
    layers: int = 1
    steps: int = 1
    mixed_bits: bool = False   # 60/30/10 % of experts at 4/6/8 bits
    zipf: Optional[float] = None
    seed: int = 0
    bits: int = 4      # width when not mixed

    def matrix_shape(self, m: int):
        """(rows, cols) of matrix m: 0 gate [I x H], 1 up [I x H], 2 down [H x I]."""
        return (self.I, self.H) if m < 2 else (self.H, self.I)


WORKLOADS = {
    w.name: w for w in (
        Workload("moe_t1_h1024_e32_k4_i256_int4", "decode", 1, 1024, 32, 4, 256),
        Workload("decode_t1_l48_h2048_e256_k8_i512_int4", "decode", 1, 2048, 256, 8, 512,
                 layers=48, steps=256),
        Workload("decode_t1_l16_h4096_e512_k10_i1024_int4", "decode", 1, 4096, 512, 10, 1024,
                 layers=16, steps=128),
        Workload("decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1", "decode", 16, 2048, 256, 8,
                 768, layers=24, steps=128, mixed_bits=True, zipf=1.1),
        Workload("prefill_t4096_l8_h2048_e256_k8_i512_int4", "prefill", 4096, 2048, 256, 8, 512,
                 layers=8, steps=1),
    )
}
WORKLOAD_ORDER = list(WORKLOADS)


def expert_bits(w: Workload, layer: int) -> np.ndarray:
    """Per-expert code width for one layer (int32 [E])."""
    if not w.mixed_bits:
        return np.full(w.E, w.bits, np.int32)
    keys = draws(stream_key(w.seed, K_BITS, layer), 0, w.E)
    order = np.lexsort((np.arange(w.E), keys))   # by key, ties by index
    n8 = int(round(0.1 * w.E))
    n6 = int(round(0.3 * w.E))
    bits = np.full(w.E, 4, np.int32)
    bits[order[:n8]] = 8
    bits[order[n8:n8 + n6]] = 6
    return bits


def router_bias(w: Workload, layer: int) -> Optional[np.ndarray]:
    """Zipf popularity bias -s*ln(rank) (fp32 [E]) or None."""
    if w.zipf is None:
        return None
    keys = draws(stream_key(w.seed, K_ZIPF, layer), 0, w.E)
    order = np.lexsort((np.arange(w.E), keys))
    rank = np.empty(w.E, np.int64)
    rank[order] = np.arange(1, w.E + 1)
    return (-w.zipf * np.log(rank.astype(np.float64))).astype(np.float32)


def hidden(w: Workload, step: int, layer: int, T: Optional[int] = None) -> np.ndarray:
    """x for (step, layer): bf16 bits [T x H]."""
    T = w.T if T is None else T
    z = normals(stream_key(w.seed, K_X, step, layer), 0, T * w.H)
    return to_bf16_bits(z).reshape(T, w.H)


def router_weights(w: Workload, layer: int) -> np.ndarray:
    """W_r: fp32 [E x H] ~ N(0, 1/H)."""
    z = normals(stream_key(w.seed, K_WR, layer), 0, w.E * w.H)
    return (z / math.sqrt(w.H)).astype(np.float32).reshape(w.E, w.H)


def scale_mult(bits: int) -> float:
    return 15.0 / float((1 << bits) - 1)


def expert_tensors(w: Workload, layer: int, e: int, bits: Optional[int] = None) -> dict:
    """Canonical tensors of one expert: codes (uint8), scale and zero (fp16 bits) per matrix."""
    if bits is None:
        bits = int(expert_bits(w, layer)[e])
    out = {"bits": bits, "codes": [], "scale": [], "zero": []}
    for m in range(3):
        rows, cols = w.matrix_shape(m)
        nb = rows * cols * bits // 8
        ng = rows * cols // GROUP
        codes = random_bytes(stream_key(w.seed, K_CODES, layer, e, m), 0, nb)
        out["codes"].append(codes.reshape(rows, cols * bits // 8))
        z = normals(stream_key(w.seed, K_SCALE, layer, e, m), 0, ng)
        s = (np.abs(z) * SQRT_0_02 + 1e-3) * scale_mult(bits)
        out["scale"].append(to_f16_bits(s).reshape(rows, cols // GROUP))
        u = uniforms(stream_key(w.seed, K_ZERO, layer, e, m), 0, ng)
        out["zero"].append(to_f16_bits(u * float((1 << bits) - 1)).reshape(rows, cols // GROUP))
    return out


def tiny(name="tiny", T=3, H=128, E=8, k=2, I=64, **kw) -> Workload:
    """A small workload for tests (same recipe, custom shape)."""
    return Workload(name, kw.pop("mode", "decode"), T, H, E, k, I, **kw)
