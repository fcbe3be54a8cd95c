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
