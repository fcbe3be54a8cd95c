"""Prefill path (moe_expert_forward_prefill) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from gpu_support import HandLayer, SynthLayer, bf16_f64, to_dev_bf16
from parity import check_block, route_check
from tests_support import pins_module

pytestmark = pytest.mark.gpu
pins = pins_module()


def prefill_call(layer, x_bits, I, E, k):
    T, H = x_bits.shape
    ws = qm.workspace(T, H, I, E, k, qm.MODE_PREFILL)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    out = qm.forward_prefill(to_dev_bf16(x_bits), layer.wr, layer.bias, layer.packed, I, E, k, ws,
                             idx_out=idx, w_out=w)
    assert qm.device_status(ws) == qm.MOE_OK
    return bf16_f64(out), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,H,I,k,widths", [
    (1, 8, 128, 64, 2, [4]), (7, 6, 192, 128, 2, [6]), (64, 5, 64, 64, 3, [8]), (300, 9, 256, 192, 4, [4, 6, 8]),
    (129, 33, 128, 64, 8, [4, 8]), (40, 16, 320, 128, 16, [6, 4]),
    (700, 4, 192, 128, 2, [4, 8]), (1200, 3, 128, 64, 1, [6]),
    (64, 1024, 128, 64, 32, [4, 8])])   # the largest E and k
def test_prefill_hand_layers(T, E, H, I, k, widths):
    rng = np.random.default_rng(T * 10 + E)
    exs = [pins.make_expert(rng, H, I, widths[e % len(widths)])[0] for e in range(E)]
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    b = rng.normal(0, 0.3, E).astype(np.float32)
    layer = HandLayer(exs, wr, b, H, I)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    out, idx, w = prefill_call(layer, x, I, E, k)
    check_block(oracle.get(), x, wr, b, layer.expert_fn, E, H, I, k, out, idx, w)


def test_prefill_full_size_all_routes_and_bucket_ends():
    """4096 tokens, 256 experts, top-8: the routing of every token against the oracle's logits,
    and the output rows of the first, 65th (the second 64-row token box) and last token of every
    expert's bucket, plus a random sample."""
    w = synth.WORKLOADS["prefill_t4096_l8_h2048_e256_k8_i512_int4"]
    layer = SynthLayer(w, 3)
    x = synth.hidden(w, 0, 3)
    out, idx, ww = prefill_call(layer, x, w.I, w.E, w.k)
    o = oracle.get()
    use_idx, _, stats = route_check(o.router_logits(x, layer.wr_np, None), w.k, idx, ww)
    print("routing of all tokens:", stats)
    picks = [0, 1, w.T - 1]
    for e in range(w.E):
        toks = np.nonzero((use_idx == e).any(axis=1))[0]   # the bucket: ascending token order
        if len(toks):
            picks += [toks[0], toks[-1]] + ([toks[64]] if len(toks) > 64 else [])
    rng = np.random.default_rng(0)
    picks += list(rng.choice(w.T, 64, replace=False))
    tokens = np.unique(np.asarray(picks))
    assert len(tokens) >= 256
    print(check_block(o, x, layer.wr_np, None, layer.expert_fn, w.E, w.H, w.I, w.k, out, idx, ww,
                      tokens=tokens), "rows", len(tokens))


def test_prefill_large_scales_zeros_and_activations():
    """Groups whose scale (|s| >= 32) or s*z (|s*z| >= 32768) is too large for the fp16 s*q path
    take the fp32 path; tokens with large activations are scaled down before the fp16 GEMM."""
    rng = np.random.default_rng(5)
    E, H, I, k, T = 6, 256, 128, 2, 150
    exs = []
    for e in range(E):
        bits = (4, 6, 8)[e % 3]
        s, z = [], []
        for m in range(3):
            rows, cols = (I, H) if m < 2 else (H, I)
            sm = np.abs(rng.normal(0, 0.1, (rows, cols // 64))) + 1e-3
            zm = rng.uniform(0, (1 << bits) - 1, (rows, cols // 64))
            big = rng.random((rows, cols // 64))
            sm[big < 0.1] = rng.uniform(32, 60, int((big < 0.1).sum()))                 # |s| >= 32
            zs = (big >= 0.1) & (big < 0.2)
            sm[zs] = 12.0
            zm[zs] = 3000.0                                                               # |s*z| >= 32768
            s.append(synth.to_f16_bits(sm))
            z.append(synth.to_f16_bits(zm))
        exs.append(pins.make_expert(rng, H, I, bits, s=s, z=z)[0])
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    layer = HandLayer(exs, wr, None, H, I)
    xv = rng.normal(0, 1, (T, H))
    xv[::7] *= 3000.0
    x = synth.to_bf16_bits(xv)
    out, idx, w = prefill_call(layer, x, I, E, k)
    print(check_block(oracle.get(), x, wr, None, layer.expert_fn, E, H, I, k, out, idx, w))


def test_prefill_agrees_with_decode_on_small_batch():
    w = synth.WORKLOADS["decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1"]
    layer = SynthLayer(w, 2)
    x = synth.hidden(w, 1, 2)
    o = oracle.get()
    out_p, idx_p, w_p = prefill_call(layer, x, w.I, w.E, w.k)
    check_block(o, x, layer.wr_np, layer.bias_np, layer.expert_fn, w.E, w.H, w.I, w.k, out_p, idx_p, w_p)


def test_prefill_route_then_experts_matches_oracle():
    """The two halves of the prefill entry point, called separately on one workspace."""
    rng = np.random.default_rng(77)
    E, H, I, k, T = 12, 192, 128, 3, 257
    exs = [pins.make_expert(rng, H, I, 4)[0] for e in range(E)]
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    layer = HandLayer(exs, wr, None, H, I)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    xd = to_dev_bf16(x)
    ws = qm.workspace(T, H, I, E, k, qm.MODE_PREFILL)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    qm.prefill_route(xd, layer.wr, None, I, E, k, ws, idx_out=idx, w_out=w)
    out = qm.prefill_experts(xd, layer.packed, I, E, k, ws)
    assert qm.device_status(ws) == qm.MOE_OK
    check_block(oracle.get(), x, wr, None, layer.expert_fn, E, H, I, k, bf16_f64(out), idx.cpu().numpy(),
                w.cpu().numpy())
    out2, idx2, _ = prefill_call(layer, x, I, E, k)
    assert np.array_equal(idx2, idx.cpu().numpy())
