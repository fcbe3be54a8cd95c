"""HQQ-style quantiser (moe_quantize_hqq) against the fp64 oracle.

The kernel evaluates the quantiser's definition with the same IEEE fp64 operations in the same
order as the oracle (one thread per group, both sums over the group in index order), so the
min-max scale, the number of steps run and the codes are compared exactly. One function differs:
the power |x|^(p-1) of the shrink, where CUDA's and the C library's results may differ in the
last place. Where the shrink is active this can move a zero by a unit in the last place of
fp64, which changes the stored fp16 zero only when that zero lies on an fp16 rounding midpoint.
Zeros are averages of binary fractions and do land there. Such groups must stay rare (at most 1
in 200, at least 4 allowed), their two stored zeros must be neighbouring fp16 values, and the
GPU's codes must be nearest points of its own stored grid, checked by a numpy brute force over
all 2^b codes. Every other code must equal the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from gpu_support import HandLayer, bf16_f64, to_dev_bf16
from parity import check_block
from tests_support import pins_module

pytestmark = pytest.mark.gpu
pins = pins_module()
G = synth.GROUP


def weights(rng, rows, cols, kind):
    if kind == "t3":        # heavy-tailed, the magnitude of LLM weights
        v = rng.standard_t(3, (rows, cols)) * 0.02
    elif kind == "normal":
        v = rng.normal(0, 1, (rows, cols))
    elif kind == "wide":    # large values: the shrink acts at the published beta
        v = rng.standard_t(3, (rows, cols)) * 0.5
    else:
        raise ValueError(kind)
    return synth.to_bf16_bits(v)


def gpu_quantize(w_bits, bits, **prm):
    rows, cols = w_bits.shape
    codes, s, z, it = qm.quantize_hqq(to_dev_bf16(w_bits), bits, with_iters=True, **prm)
    torch.cuda.synchronize()
    q = synth.unpack_codes(codes.cpu().numpy(), bits, cols)
    s16 = s.cpu().numpy().view(np.uint16)
    z16 = z.cpu().numpy().view(np.uint16)
    return q, s16, z16, it.cpu().numpy()


def f16_neighbours(a_bits, b_bits):
    a = np.uint16(a_bits).view(np.float16)
    b = np.uint16(b_bits).view(np.float16)
    lo, hi = min(a, b), max(a, b)
    return bool(np.nextafter(lo, np.float16(np.inf)) == hi)


def check_quantizer(w_bits, bits, exact=False, **prm):
    rows, cols = w_bits.shape
    Q = (1 << bits) - 1
    o = oracle.get()
    oprm = {{"lp_norm": "p"}.get(k, k): v for k, v in prm.items()}
    rq, rs, rz, rit = o.hqq_quantize(w_bits, bits, **oprm)
    q, s16, z16, it = gpu_quantize(w_bits, bits, **prm)
    assert q.max() <= Q and q.min() >= 0
    assert np.array_equal(s16, rs), "min-max scales differ"
    assert np.array_equal(it, rit), "steps run differ"
    zsame = synth.f16_bits_to_f64(z16) == synth.f16_bits_to_f64(rz)
    same_cols = np.repeat(zsame, G, 1)
    assert np.array_equal(q[same_cols], rq[same_cols].astype(np.int64)), "codes differ where zeros agree"
    nbad = int((~zsame).sum())
    print(f"stored zeros differing from the oracle: {nbad} of {zsame.size} groups")
    if exact:
        assert nbad == 0, nbad
    # a CPU model of this kind of difference moved about 1 zero in 2000 groups (fp16 midpoints);
    # on a B200 none of the ~120,000 groups of these tests differed. The cap catches anything
    # above that model's rate; each differing group is checked below
    assert nbad <= max(2, zsame.size // 2000), f"{nbad} of {zsame.size} stored zeros differ"
    if nbad:
        w = synth.bf16_bits_to_f32(w_bits).astype(np.float64)
        for r, g in zip(*np.nonzero(~zsame)):
            assert f16_neighbours(z16[r, g], rz[r, g]), (r, g, z16[r, g], rz[r, g])
            sl = slice(G * g, G * (g + 1))
            pins.check_nearest(w[r, sl], q[r, sl], synth.f16_bits_to_f64(s16[r, g]),
                               synth.f16_bits_to_f64(z16[r, g]), Q, (r, g))
    return nbad


@pytest.mark.parametrize("rows,cols,bits,kind,prm", [
    (1, 64, 4, "t3", {}),
    (3, 640, 6, "normal", {}),
    (37, 128, 8, "wide", {"lp_norm": 1.0, "beta": 1e3, "kappa": 1.05}),
    (64, 2048, 4, "t3", {"lp_norm": 0.5, "beta": 1e5, "kappa": 1.2}),
    (8, 192, 6, "wide", {"beta": 1e4, "iters": 1000}),
    (129, 320, 8, "t3", {}),
    (5, 64, 4, "wide", {"iters": 1}),
])
def test_quantizer_matches_oracle(rows, cols, bits, kind, prm):
    rng = np.random.default_rng(rows * 1000 + cols + bits)
    check_quantizer(weights(rng, rows, cols, kind), bits, **prm)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_quantizer_minmax_is_exact(bits):
    """iters = 0 (min-max rounding) has no sums: every output is bit-exact."""
    rng = np.random.default_rng(bits)
    check_quantizer(weights(rng, 48, 512, "t3"), bits, exact=True, iters=0)


def test_quantizer_degenerate_groups():
    """All-zero, constant (positive, negative, tiny) and on-grid groups, next to random ones."""
    rng = np.random.default_rng(5)
    for bits in (4, 6, 8):
        Q = (1 << bits) - 1
        w = rng.standard_t(3, (8, 4 * G)) * 0.02
        w[0, :G] = 0.0
        w[1, G:2 * G] = 0.75
        w[2, 2 * G:3 * G] = -0.0390625
        w[3, :G] = 2.0 ** -20
        q = rng.integers(0, Q + 1, G)
        q[0], q[-1] = 0, Q
        w[4, 3 * G:] = (q - 5.0) * 2.0 ** -7
        w[5, :G] = -0.0
        wb = synth.to_bf16_bits(w)
        check_quantizer(wb, bits)
        qg, s16, z16, it = gpu_quantize(wb, bits)
        rq, rs, rz, rit = oracle.get().hqq_quantize(wb, bits)
        for r, g in ((0, 0), (1, 1), (2, 2), (3, 0), (4, 3), (5, 0)):
            sl = slice(G * g, G * (g + 1))
            assert np.array_equal(qg[r, sl], rq[r, sl]), (bits, r, g)
            assert s16[r, g] == rs[r, g] and it[r, g] == rit[r, g], (bits, r, g)
            assert synth.f16_bits_to_f64(z16[r, g]) == synth.f16_bits_to_f64(rz[r, g]), (bits, r, g)
        assert np.array_equal(qg[4, 3 * G:], q) and synth.f16_bits_to_f64(s16[4, 3]) == 2.0 ** -7
        assert np.all(qg[0, :G] == 0) and synth.f16_bits_to_f64(z16[0, 0]) == 0.0


@pytest.mark.parametrize("rows,cols,bits", [(512, 2048, 4), (2048, 512, 8), (1024, 4096, 4)])
def test_quantizer_full_expert_matrices(rows, cols, bits):
    """Whole gate/up and down matrices of the 2048/512 and 4096/1024 expert shapes."""
    rng = np.random.default_rng(rows + cols)
    check_quantizer(weights(rng, rows, cols, "t3"), bits)


def test_quantizer_with_caller_stream_and_no_iteration_output():
    rng = np.random.default_rng(9)
    w = weights(rng, 16, 256, "t3")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        wd = to_dev_bf16(w)
        codes, s, z = qm.quantize_hqq(wd, 6, stream=st)
    st.synchronize()
    rq, rs, rz, _ = oracle.get().hqq_quantize(w, 6)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs)
    assert codes.shape == (16, 256 * 6 // 8)


def test_quantized_experts_through_the_block():
    """bf16 experts quantised on the GPU, packed and run through the decode and prefill paths,
    against the oracle's block on the oracle's own quantisation of the same weights."""
    rng = np.random.default_rng(21)
    E, H, I, k, T = 6, 256, 128, 2, 5
    o = oracle.get()
    dev_experts, ref_experts = [], []
    for e in range(E):
        bits = (4, 6, 8)[e % 3]
        ex_dev = {"bits": bits, "codes": [], "scale": [], "zero": []}
        ex_ref = {"bits": bits, "codes": [], "scale": [], "zero": []}
        for rows, cols in ((I, H), (I, H), (H, I)):
            w = weights(rng, rows, cols, "t3")
            c, s, z = qm.quantize_hqq(to_dev_bf16(w), bits)
            ex_dev["codes"].append(c)
            ex_dev["scale"].append(s.view(torch.int16))
            ex_dev["zero"].append(z.view(torch.int16))
            rq, rs, rz, _ = o.hqq_quantize(w, bits)
            ex_ref["codes"].append(synth.pack_codes(rq, bits))
            ex_ref["scale"].append(rs)
            ex_ref["zero"].append(rz)
        dev_experts.append(ex_dev)
        ref_experts.append(ex_ref)
    packed = qm.pack_layer(dev_experts, H, I)
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    layer = HandLayer(ref_experts, wr, None, H, I)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    for mode in (qm.MODE_DECODE, qm.MODE_PREFILL):
        ws = qm.workspace(T, H, I, E, k, mode)
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        wo = torch.zeros((T, k), dtype=torch.float32, device="cuda")
        fwd = qm.forward_decode if mode == qm.MODE_DECODE else qm.forward_prefill
        out = fwd(to_dev_bf16(x), layer.wr, None, packed, I, E, k, ws, idx_out=idx, w_out=wo)
        assert qm.device_status(ws) == qm.MOE_OK
        check_block(o, x, wr, None, layer.expert_fn, E, H, I, k, bf16_f64(out), idx.cpu().numpy(),
                    wo.cpu().numpy())
