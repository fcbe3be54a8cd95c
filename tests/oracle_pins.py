"""Pins of the fp64 oracle: checks against things other than the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when it fails. They compare the
oracle with
  * a numpy brute force that never unpacks bytes: it draws integer codes, dequantises them to
    dense fp64 matrices and runs textbook matmuls, SciPy's ``softmax``/``expit`` and a full
    stable sort (the method's plain definition evaluated by library routines);
  * hand-derived bytes of the canonical packing (tests/golden/canonical_pack_layout.txt);
  * closed forms and invariants that hold exactly in fp64 (zero experts, doubled scales,
    expert relabelling, one-hot inputs, k = E, k = 1).
Run as a script (``python tests/oracle_pins.py <lib.so>``) it evaluates every pin against the
given oracle build and prints a JSON map of pin -> "ok" / error text; the mutation tests use
that to show each plausible mistake in the oracle trips at least one pin.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np
from scipy.special import expit, softmax

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
import oracle as oracle_mod  # noqa: E402

G = synth.GROUP
GOLDEN = os.path.join(ROOT, "tests", "golden", "canonical_pack_layout.txt")


# ----------------------------------------------------------------------------- builders

def f16(bits):
    return synth.f16_bits_to_f64(bits)


def make_expert(rng, H, I, bits, q=None, s=None, z=None):
    """Random expert in canonical form plus its dense dequantised matrices (numpy fp64)."""
    ex = {"bits": bits, "codes": [], "scale": [], "zero": []}
    dense = []
    for m in range(3):
        rows, cols = (I, H) if m < 2 else (H, I)
        qm = rng.integers(0, 1 << bits, size=(rows, cols)) if q is None else q[m]
        sm = (synth.to_f16_bits(np.abs(rng.normal(0, 0.1, (rows, cols // G))) + 1e-3)
              if s is None else s[m])
        zm = (synth.to_f16_bits(rng.uniform(0, (1 << bits) - 1, (rows, cols // G)))
              if z is None else z[m])
        ex["codes"].append(synth.pack_codes(qm, bits))
        ex["scale"].append(np.asarray(sm, np.uint16))
        ex["zero"].append(np.asarray(zm, np.uint16))
        dense.append((qm - np.repeat(f16(zm), G, axis=1)) * np.repeat(f16(sm), G, axis=1))
    return ex, dense


def random_x(rng, T, H):
    return synth.to_bf16_bits(rng.normal(0, 1, (T, H)))


def xf(xbits):
    return synth.bf16_bits_to_f32(xbits).astype(np.float64)


def dense_ffn(W, x):
    g = W[0] @ x
    u = W[1] @ x
    h = g * expit(g) * u
    return g, u, h, W[2] @ h


def dense_forward(xbits, wr, bias, dense, k):
    x = xf(xbits)
    l = x @ wr.astype(np.float64).T
    if bias is not None:
        l = l + bias.astype(np.float64)
    idx = np.argsort(-l, axis=1, kind="stable")[:, :k]
    w = softmax(np.take_along_axis(l, idx, axis=1), axis=1)
    out = np.zeros((x.shape[0], dense[0][2].shape[0]))
    for t in range(x.shape[0]):
        for i in range(k):
            out[t] += w[t, i] * dense_ffn(dense[idx[t, i]], x[t])[3]
    return out, idx, w, l


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ----------------------------------------------------------------------------- pins

def pin_pack_golden(o):
    """The canonical packer reproduces the hand-derived group bytes."""
    rules = {
        "j%16": lambda j: j % 16, "j": lambda j: j, "63-j": lambda j: 63 - j,
        "(5*j+3)%256": lambda j: (5 * j + 3) % 256,
    }
    n = 0
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        f = line.split()
        bits, rule, want = int(f[1]), f[3], bytes.fromhex("".join(f[5:]))
        q = np.array([[rules[rule](j) for j in range(G)]])
        got = synth.pack_codes(q, bits)[0].tobytes()[:len(want)]
        assert got == want, (bits, rule, got.hex(), want.hex())
        n += 1
    assert n == 4


def pin_unpack_codes(o):
    """With s=1, z=0 the oracle's weight at (r, c) is the integer code drawn for (r, c)."""
    rng = np.random.default_rng(11)
    for bits in (4, 6, 8):
        H, I = 128, 64
        one = synth.to_f16_bits(np.ones((I, H // G)))
        zero = synth.to_f16_bits(np.zeros((I, H // G)))
        one_d = synth.to_f16_bits(np.ones((H, I // G)))
        zero_d = synth.to_f16_bits(np.zeros((H, I // G)))
        q = [rng.integers(0, 1 << bits, (I, H)), rng.integers(0, 1 << bits, (I, H)),
             rng.integers(0, 1 << bits, (H, I))]
        ex, _ = make_expert(rng, H, I, bits, q=q, s=[one, one, one_d], z=[zero, zero, zero_d])
        for m, (rows, cols) in enumerate([(I, H), (I, H), (H, I)]):
            for r, c in zip(rng.integers(0, rows, 200), rng.integers(0, cols, 200)):
                assert o.weight(ex, m, rows, cols, int(r), int(c)) == float(q[m][r, c]), (bits, m)


def pin_f16_values(o):
    """Scale/zero decoding equals numpy's IEEE binary16 conversion, subnormals included."""
    rng = np.random.default_rng(12)
    H, I = 64, 64
    bits = 4
    s_bits = np.array([0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x1234, 0x2E66, 0x0200]
                      * 8, np.uint16)[: I * (H // G)].reshape(I, H // G)
    q = [np.full((I, H), 5), np.full((I, H), 5), np.full((H, I), 5)]
    z = [synth.to_f16_bits(np.zeros((I, 1)))] * 2 + [synth.to_f16_bits(np.zeros((H, 1)))]
    s = [s_bits, s_bits, s_bits]
    ex, dense = make_expert(rng, H, I, bits, q=q, s=s, z=z)
    for r in range(I):
        assert o.weight(ex, 0, I, H, r, 3) == 5.0 * float(np.uint16(s_bits[r, 0]).view(np.float16))


def pin_dense_bruteforce(o):
    """Whole block equals the dense numpy brute force, for every code width and a bias."""
    rng = np.random.default_rng(13)
    for bits in (4, 6, 8, "mixed"):
        T, H, I, E, k = 5, 128, 64, 6, 2
        widths = [4, 6, 8, 4, 6, 8] if bits == "mixed" else [bits] * E
        exs = [make_expert(rng, H, I, b) for b in widths]
        x = random_x(rng, T, H)
        wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
        bias = rng.normal(0, 0.5, E).astype(np.float32)
        out, idx, w, l = o.forward(x, wr, bias, [e[0] for e in exs], H, I, k)
        rout, ridx, rw, rl = dense_forward(x, wr, bias, [e[1] for e in exs], k)
        assert np.array_equal(idx, ridx), (bits, idx, ridx)
        assert rel(l, rl) < 1e-13, bits
        assert rel(w, rw) < 1e-13, bits
        assert rel(out, rout) < 1e-12, (bits, rel(out, rout))


def pin_expert_stages(o):
    """g, u, h and y of one expert equal the dense matmuls and SciPy's logistic function."""
    rng = np.random.default_rng(14)
    for bits in (4, 6, 8):
        H, I = 192, 128
        ex, dense = make_expert(rng, H, I, bits)
        x = random_x(rng, 1, H)[0]
        g, u, h, y = o.expert_ffn(x, ex, H, I)
        rg, ru, rh, ry = dense_ffn(dense, xf(x))
        for a, b in ((g, rg), (u, ru), (h, rh), (y, ry)):
            assert rel(a, b) < 1e-12, bits


def pin_topk_full_sort(o):
    """Top-k equals the first k of a full stable sort by (logit desc, index asc), ties included."""
    rng = np.random.default_rng(15)
    for E, k in ((8, 3), (32, 4), (256, 8), (512, 10), (17, 17)):
        l = rng.normal(0, 1, (40, E))
        l[:, 1::3] = np.round(l[:, 1::3], 1)   # many exact ties
        l[:5, :] = 0.25                         # all equal
        idx, w = o.topk(l, k)
        ref = np.argsort(-l, axis=1, kind="stable")[:, :k]
        assert np.array_equal(idx, ref), (E, k)


def pin_weights_sum_one(o):
    rng = np.random.default_rng(16)
    l = rng.normal(0, 3, (64, 64))
    for k in (1, 2, 8, 64):
        _, w = o.topk(l, k)
        assert np.max(np.abs(w.sum(1) - 1.0)) < 1e-12
        assert np.all(w > 0)
        assert np.all(np.diff(w, axis=1) <= 0)   # weights follow the logit order


def pin_k_equals_E(o):
    """k = E gives the plain softmax over all experts (SciPy), in descending order."""
    rng = np.random.default_rng(17)
    l = rng.normal(0, 2, (10, 12))
    idx, w = o.topk(l, 12)
    sm = softmax(l, axis=1)
    assert rel(w, np.take_along_axis(sm, idx, axis=1)) < 1e-13
    assert rel(np.sort(w, 1), np.sort(sm, 1)) < 1e-13


def pin_zero_expert(o):
    """An expert with all-zero codes and zero point 0 contributes exactly 0."""
    rng = np.random.default_rng(18)
    T, H, I, E, k = 4, 128, 64, 3, 2
    zq = [np.zeros((I, H), int), np.zeros((I, H), int), np.zeros((H, I), int)]
    zz = [synth.to_f16_bits(np.zeros((I, H // G)))] * 2 + [synth.to_f16_bits(np.zeros((H, I // G)))]
    e0, d0 = make_expert(rng, H, I, 4, q=zq, z=zz)
    e1, d1 = make_expert(rng, H, I, 4)
    x = random_x(rng, T, H)
    g, u, h, y = o.expert_ffn(x[0], e0, H, I)
    assert np.all(y == 0.0) and np.all(g == 0.0)
    idx = np.array([[0, 1]] * T, np.int32)
    w = np.array([[0.3, 0.7]] * T)
    out = o.combine(x, [e0, e1, None], H, I, idx, w)
    only = o.combine(x, [e0, e1, None], H, I, idx[:, 1:], w[:, 1:])
    assert np.array_equal(out, only)


def pin_q_equals_z(o):
    """Codes all equal to c with zero point c dequantise to 0 (for every width)."""
    rng = np.random.default_rng(19)
    H, I = 128, 64
    for bits in (4, 6, 8):
        c = (1 << bits) - 3
        q = [np.full((I, H), c), np.full((I, H), c), np.full((H, I), c)]
        z = [synth.to_f16_bits(np.full((I, H // G), c))] * 2 + \
            [synth.to_f16_bits(np.full((H, I // G), c))]
        ex, _ = make_expert(rng, H, I, bits, q=q, z=z)
        _, _, _, y = o.expert_ffn(random_x(rng, 1, H)[0], ex, H, I)
        assert np.all(y == 0.0)


def pin_k1_dense_ffn(o):
    """k = 1: the weight is exactly 1 and the block is one dense FFN of the arg-max expert."""
    rng = np.random.default_rng(20)
    T, H, I, E = 3, 128, 128, 5
    exs = [make_expert(rng, H, I, 6) for _ in range(E)]
    x = random_x(rng, T, H)
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    out, idx, w, l = o.forward(x, wr, None, [e[0] for e in exs], H, I, 1)
    assert np.all(w == 1.0)
    for t in range(T):
        e = int(np.argmax(xf(x[t]) @ wr.astype(np.float64).T))
        assert idx[t, 0] == e
        assert rel(out[t], dense_ffn(exs[e][1], xf(x[t]))[3]) < 1e-12


def pin_double_down_scale(o):
    """Doubling every down-projection scale doubles the output exactly."""
    rng = np.random.default_rng(21)
    T, H, I, E, k = 3, 128, 64, 4, 2
    exs = [make_expert(rng, H, I, 4)[0] for _ in range(E)]
    x = random_x(rng, T, H)
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    out, idx, w, _ = o.forward(x, wr, None, exs, H, I, k)
    dbl = []
    for ex in exs:
        d = {"bits": ex["bits"], "codes": ex["codes"], "zero": ex["zero"],
             "scale": ex["scale"][:2] + [synth.to_f16_bits(2.0 * f16(ex["scale"][2]))]}
        dbl.append(d)
    out2, idx2, _, _ = o.forward(x, wr, None, dbl, H, I, k)
    assert np.array_equal(idx, idx2) and np.array_equal(out2, 2.0 * out)


def pin_relabel_experts(o):
    """Permuting the experts together with the router rows leaves the output unchanged."""
    rng = np.random.default_rng(22)
    T, H, I, E, k = 4, 128, 64, 7, 3
    exs = [make_expert(rng, H, I, [4, 6, 8][e % 3])[0] for e in range(E)]
    x = random_x(rng, T, H)
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    bias = rng.normal(0, 0.3, E).astype(np.float32)
    out, idx, w, _ = o.forward(x, wr, bias, exs, H, I, k)
    p = rng.permutation(E)
    out2, idx2, w2, _ = o.forward(x, wr[p], bias[p], [exs[i] for i in p], H, I, k)
    assert np.array_equal(p[idx2], idx) and np.array_equal(w2, w) and np.array_equal(out2, out)


def pin_onehot_x(o):
    """x = e_j makes g and u exactly column j of the dequantised gate and up matrices."""
    rng = np.random.default_rng(23)
    H, I = 128, 64
    for bits in (4, 6, 8):
        ex, dense = make_expert(rng, H, I, bits)
        for j in (0, 63, 64, 127):
            x = synth.to_bf16_bits(np.eye(H)[j])
            g, u, _, _ = o.expert_ffn(x, ex, H, I)
            assert np.array_equal(g, dense[0][:, j]) and np.array_equal(u, dense[1][:, j])


# ----------------------------------------------------------------------------- quantiser pins

def grid_distances(w, s, z, Q):
    """|w_j - (q - z) * s| for every weight j and every code q in 0..Q (brute force)."""
    cand = (np.arange(Q + 1, dtype=np.float64) - z) * s
    return np.abs(np.asarray(w, np.float64)[:, None] - cand[None, :])


def check_nearest(w, q, s, z, Q, what=""):
    """Every code is a nearest point of the grid (q - z) * s, q in 0..Q."""
    d = grid_distances(w, s, z, Q)
    chosen = d[np.arange(len(w)), np.asarray(q, np.int64)]
    assert np.all(chosen <= d.min(1) + 1e-12 * s), what


def f16_of(v):
    """numpy's binary16 rounding of a double (round to nearest even), as bits."""
    with np.errstate(over="ignore"):
        return int(np.array([v], np.float64).astype(np.float16).view(np.uint16)[0])


def pin_f16_conversion(o):
    """The oracle's double -> binary16 rounding equals numpy's, ties, subnormals and overflow
    included."""
    rng = np.random.default_rng(30)
    vals = list(rng.normal(0, 1, 400) * 10.0 ** rng.integers(-9, 6, 400))
    h = np.arange(0, 0x7BFF, 37, dtype=np.uint16)
    hv = h.view(np.float16).astype(np.float64)
    nv = (h + 1).view(np.float16).astype(np.float64)
    mid = (hv + nv) / 2                                     # exact in fp64: ties
    vals += list(hv) + list(mid) + list(np.nextafter(mid, 0)) + list(np.nextafter(mid, 1e9))
    vals += [0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.001,
             2.0 ** -26, 3 * 2.0 ** -25, 2.0 ** -14 - 2.0 ** -25, 1e-300]
    for v in vals:
        for sg in (1.0, -1.0):
            assert o.f64_to_f16(sg * v) == f16_of(sg * v), (sg * v, hex(o.f64_to_f16(sg * v)))


def pin_hqq_minmax_rounding(o):
    """iters = 0 is min-max rounding: s = fp16((max - min) / Q) and z = fp16(-min / s) as numpy
    rounds them, and every code is a nearest grid point (brute force over all 2^b codes)."""
    rng = np.random.default_rng(31)
    for bits in (4, 6, 8):
        Q = (1 << bits) - 1
        wb = synth.to_bf16_bits(rng.normal(0, 0.05, (6, 256)) + rng.normal(0, 0.03, (6, 1)))
        q, s16, z16, ran = o.hqq_quantize(wb, bits, iters=0)
        assert np.all(ran == 0)
        w = xf(wb)
        for r in range(6):
            for g in range(4):
                wg = w[r, G * g:G * (g + 1)]
                lo, hi = wg.min(), wg.max()
                assert s16[r, g] == f16_of((hi - lo) / Q), bits
                s = f16(s16[r, g])
                assert z16[r, g] == f16_of(-lo / s), bits
                check_nearest(wg, q[r, G * g:G * (g + 1)], s, f16(z16[r, g]), Q, bits)


def pin_hqq_codes_nearest(o):
    """After the zero-point iteration, and for arbitrary given scales and zeros, every code is a
    nearest point of the stored fp16 grid."""
    rng = np.random.default_rng(32)
    for bits, p, beta in ((4, 0.7, 10.0), (6, 0.7, 1e4), (8, 1.0, 1e3), (4, 0.5, 1e5)):
        Q = (1 << bits) - 1
        wb = synth.to_bf16_bits(rng.standard_t(3, (5, 192)) * 0.03)
        q, s16, z16, _ = o.hqq_quantize(wb, bits, p=p, beta=beta)
        w = xf(wb)
        for r in range(5):
            for g in range(3):
                sl = slice(G * g, G * (g + 1))
                check_nearest(w[r, sl], q[r, sl], f16(s16[r, g]), f16(z16[r, g]), Q, bits)
        s_any = synth.to_f16_bits(np.abs(rng.normal(0, 0.01, (5, 3))) + 1e-4)
        z_any = synth.to_f16_bits(rng.uniform(-5, Q + 5, (5, 3)))
        q2 = o.hqq_codes(wb, bits, s_any, z_any)
        for r in range(5):
            for g in range(3):
                sl = slice(G * g, G * (g + 1))
                check_nearest(w[r, sl], q2[r, sl], f16(s_any[r, g]), f16(z_any[r, g]), Q, bits)


def pin_hqq_exact_grid(o):
    """Weights that already lie on a b-bit grid spanning codes 0..Q come back exactly (scale,
    zero and codes), with and without the zero-point iteration."""
    rng = np.random.default_rng(33)
    for bits in (4, 6, 8):
        Q = (1 << bits) - 1
        rows = 8
        q = rng.integers(0, Q + 1, (rows, 2 * G))
        q[:, 0], q[:, G - 1], q[:, G], q[:, 2 * G - 1] = 0, Q, Q, 0
        s = 2.0 ** rng.integers(-9, -3, (rows, 2)).astype(np.float64)
        z = rng.integers(0, Q + 1, (rows, 2)).astype(np.float64)
        w = (q - np.repeat(z, G, 1)) * np.repeat(s, G, 1)
        wb = synth.to_bf16_bits(w)
        assert np.array_equal(xf(wb), w)
        for iters in (0, 20):
            qq, s16, z16, _ = o.hqq_quantize(wb, bits, iters=iters)
            assert np.array_equal(qq, q) and np.array_equal(f16(s16), s), (bits, iters)
            assert np.array_equal(f16(z16), z), (bits, iters)


TRACE_CASES = ((4, 0.7, 10.0, 1.01, 1.0), (4, 0.7, 1e4, 1.01, 0.05), (6, 1.0, 1e3, 1.05, 0.5),
               (8, 0.5, 1e5, 1.2, 0.02), (4, 1.0, 30.0, 1.01, 2.0))


HQQ_FALL = 1.0 - 2.0 ** -40


def pin_hqq_trace(o):
    """Each iteration's error is the brute-force L1 distance of the group to its nearest grid
    points at that iteration's zero; each step that continues has an error below 1 - 2^-40
    times the one before; only the last step run may fail that (the stop); the stored zero is
    the fp16 value of the zero with the least error."""
    rng = np.random.default_rng(34)
    for bits, p, beta, kappa, scale in TRACE_CASES:
        Q = (1 << bits) - 1
        for _ in range(12):
            wg = xf(synth.to_bf16_bits(rng.standard_t(3, G) * scale))
            s16, z16, q, zt, et = o.hqq_group(wg, bits, p=p, beta=beta, kappa=kappa, iters=20)
            s = f16(s16)
            assert 1 <= len(et) <= 20
            for i in range(len(et)):
                err = grid_distances(wg, s, zt[i], Q).min(1).sum()
                assert abs(et[i] - err) <= 1e-12 * max(err, s), (bits, i)
            assert np.all(et[1:-1] < et[:-2] * HQQ_FALL)
            if len(et) < 20:
                assert len(et) >= 2 and not et[-1] < et[-2] * HQQ_FALL
            last_fell = len(et) == 1 or et[-1] < et[-2] * HQQ_FALL
            best = len(et) - 1 if last_fell else len(et) - 2
            assert z16 == f16_of(zt[best]), (bits, best)


def pin_hqq_zero_update(o):
    """Each new zero is the least-squares solution (numpy lstsq) of q - z = (w - e) / s, with q
    the nearest codes at the previous zero, e the shrunk residual and beta_i = beta * kappa^i."""
    rng = np.random.default_rng(35)
    for bits, p, beta, kappa, scale in TRACE_CASES:
        Q = (1 << bits) - 1
        for _ in range(8):
            wg = xf(synth.to_bf16_bits(rng.standard_t(3, G) * scale))
            s16, _, _, zt, _ = o.hqq_group(wg, bits, p=p, beta=beta, kappa=kappa, iters=20)
            s = f16(s16)
            for i in range(len(zt) - 1):
                qn = grid_distances(wg, s, zt[i], Q).argmin(1)
                res = wg - (qn - zt[i]) * s
                e = np.array([o.hqq_shrink(x, beta * kappa ** i, p) for x in res])
                rhs = qn - (wg - e) / s
                z_ls = np.linalg.lstsq(np.ones((G, 1)), rhs, rcond=None)[0][0]
                assert abs(zt[i + 1] - z_ls) <= 1e-10 * max(1.0, abs(z_ls)), (bits, i)


def pin_hqq_shrink(o):
    """p = 1: the shrink is the proximal map of |y| / beta (brute-force minimisation). p < 1: an
    odd map toward 0 that is exactly 0 up to |x| = beta^(-1/(2-p)) and nonzero beyond, grows
    with beta, and tends to the p = 1 map as p -> 1."""
    from scipy.optimize import minimize_scalar
    rng = np.random.default_rng(36)
    for beta in (0.5, 3.0, 40.0):
        for x in rng.normal(0, 2.0 / beta, 25):
            f = lambda y, x=x: 0.5 * (y - x) ** 2 + abs(y) / beta  # noqa: E731
            r = minimize_scalar(f, bounds=(-abs(x) - 1, abs(x) + 1), method="bounded",
                                options={"xatol": 1e-13})
            assert abs(o.hqq_shrink(x, beta, 1.0) - r.x) < 1e-7, (beta, x)
    for p in (0.5, 0.7, 0.9):
        for beta in (10.0, 1e3):
            thr = beta ** (-1.0 / (2.0 - p))
            for m in (0.1, 0.5, 0.99, 0.9999, 1.0001, 1.01, 2.0, 10.0):
                for x in (m * thr, -m * thr):
                    e = o.hqq_shrink(x, beta, p)
                    assert o.hqq_shrink(-x, beta, p) == -e
                    if m < 1:
                        assert e == 0.0, (p, beta, m)
                    else:
                        assert e != 0 and np.sign(e) == np.sign(x) and abs(e) < abs(x), (p, m)
                        assert abs(o.hqq_shrink(x, 2 * beta, p)) > abs(e)
            x = 3 * thr
            assert abs(o.hqq_shrink(x, beta, 1 - 1e-9) - o.hqq_shrink(x, beta, 1.0)) < 1e-6 * x
    assert o.hqq_shrink(0.0, 10.0, 0.7) == 0.0


def pin_hqq_constant_groups(o):
    """An all-zero group is stored exactly; a constant group c is reproduced to fp16 precision."""
    for bits in (4, 6, 8):
        Q = (1 << bits) - 1
        for c in (0.0, 0.75, -0.0390625, 3.0e-3, -7.5):
            wb = synth.to_bf16_bits(np.full((1, G), c))
            cv = float(xf(wb)[0, 0])
            q, s16, z16, _ = o.hqq_quantize(wb, bits)
            rec = (q[0].astype(np.float64) - f16(z16[0, 0])) * f16(s16[0, 0])
            if cv == 0.0:
                assert np.all(rec == 0.0), bits
            else:
                assert np.all(np.abs(rec - cv) <= abs(cv) * 2.0 ** -10), (bits, c)
            assert np.all(q <= Q)


def pin_hqq_power_of_two_scaling(o):
    """p = 1: scaling the weights by 2^k and beta by 2^-k scales the stored scale by 2^k and
    leaves zeros, codes and iteration counts unchanged (exact in binary arithmetic)."""
    rng = np.random.default_rng(37)
    wb = synth.to_bf16_bits(rng.standard_t(3, (4, 128)) * 0.02)
    w = xf(wb)
    for bits, beta in ((4, 300.0), (6, 3000.0), (8, 30.0)):
        q0, s0, z0, r0 = o.hqq_quantize(wb, bits, p=1.0, beta=beta, kappa=1.03)
        for k in (-3, 2, 5):
            wk = synth.to_bf16_bits(w * 2.0 ** k)
            q1, s1, z1, r1 = o.hqq_quantize(wk, bits, p=1.0, beta=beta * 2.0 ** -k, kappa=1.03)
            assert np.array_equal(q1, q0) and np.array_equal(z1, z0) and np.array_equal(r1, r0)
            assert np.array_equal(f16(s1), f16(s0) * 2.0 ** k), (bits, k)


def pin_hqq_matrix_layout(o):
    """The matrix call quantises group g of row r from columns 64g..64g+63 of that row."""
    rng = np.random.default_rng(38)
    wb = synth.to_bf16_bits(rng.normal(0, 0.04, (3, 320)))
    q, s16, z16, ran = o.hqq_quantize(wb, 6, beta=1e4)
    w = xf(wb)
    for r in range(3):
        for g in range(5):
            sg, zg, qg, zt, _ = o.hqq_group(w[r, G * g:G * (g + 1)], 6, beta=1e4)
            assert (sg, zg, len(zt)) == (s16[r, g], z16[r, g], ran[r, g])
            assert np.array_equal(qg, q[r, G * g:G * (g + 1)])


def pin_hqq_beats_minmax(o):
    """Summed over many groups, the stored result has less L1 reconstruction error than plain
    min-max rounding (the iteration starts there and only keeps improvements)."""
    rng = np.random.default_rng(39)
    for bits in (4, 6, 8):
        wb = synth.to_bf16_bits(rng.standard_t(4, (16, 512)) * 0.02)
        w = xf(wb)
        errs = []
        for iters in (0, 20):
            q, s16, z16, _ = o.hqq_quantize(wb, bits, iters=iters)
            rec = (q - np.repeat(f16(z16), G, 1)) * np.repeat(f16(s16), G, 1)
            errs.append(np.abs(rec - w).sum())
        assert errs[1] < errs[0], (bits, errs)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]


def run_all(o) -> dict:
    res = {}
    for p in PINS:
        try:
            p(o)
            res[p.__name__] = "ok"
        except Exception as e:  # noqa: BLE001 - report every failure kind
            res[p.__name__] = f"{type(e).__name__}: {str(e)[:200]}"
    return res


if __name__ == "__main__":
    lib = sys.argv[1]
    print(json.dumps(run_all(oracle_mod.Oracle(lib))))
