"""Decode megakernel (moe_expert_forward_decode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import synth.device as sd
import quantized_moe_router_b200 as qm
from quantized_moe_router_b200.runner import DecodeStack, LayerWeights
from gpu_support import HandLayer, SynthLayer, bf16_f64, to_dev_bf16
from parity import check_block
from tests_support import pins_module

pytestmark = pytest.mark.gpu
pins = pins_module()


def hand_layer(rng, E, H, I, widths, bias=True):
    exs = [pins.make_expert(rng, H, I, widths[e % len(widths)])[0] for e in range(E)]
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    b = rng.normal(0, 0.3, E).astype(np.float32) if bias else None
    return HandLayer(exs, wr, b, H, I)


def decode_call(layer, x_bits, I, E, k, ws=None):
    T, H = x_bits.shape
    if ws is None:
        ws = qm.workspace(T, H, I, E, k, qm.MODE_DECODE)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    out = qm.forward_decode(to_dev_bf16(x_bits), layer.wr, layer.bias, layer.packed, I, E, k, ws,
                            idx_out=idx, w_out=w)
    assert qm.device_status(ws) == qm.MOE_OK
    return bf16_f64(out), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,H,I,k,widths", [
    (1, 8, 128, 64, 2, [4]), (3, 6, 192, 128, 2, [6]), (8, 5, 64, 64, 3, [8]), (13, 9, 256, 192, 4, [4, 6, 8]),
    (32, 16, 128, 64, 8, [4, 8]), (1, 4, 64, 64, 1, [4]), (5, 12, 320, 64, 12, [6, 4]), (2, 40, 128, 256, 7, [4])])
def test_decode_hand_layers(T, E, H, I, k, widths):
    rng = np.random.default_rng(T * 100 + E)
    layer = hand_layer(rng, E, H, I, widths)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    out, idx, w = decode_call(layer, x, I, E, k)
    check_block(oracle.get(), x, layer.wr_np, layer.bias_np, layer.expert_fn, E, H, I, k, out, idx, w)


@pytest.mark.parametrize("T,E,H,I,k,widths", [
    (1, 24, 256, 512, 8, [4, 6, 8]),      # one token, per-expert widths: work cut by bytes
    (1, 16, 8192, 128, 8, [4, 6, 8]),     # the largest H: 128 row super-tiles, 5 gate/up chunks per unit
    (1, 1024, 256, 64, 32, [4]),          # the largest E and k: wide top-k, 32 slots of 4 units
    (16, 48, 2048, 192, 8, [6, 8, 4]),    # several tokens with shared experts, mixed widths
    (1, 6, 4096, 64, 6, [8])])            # few units (24) over all CTAs, all 8-bit
def test_decode_unit_cuts_and_limits(T, E, H, I, k, widths):
    rng = np.random.default_rng(T * 7 + E + H)
    layer = hand_layer(rng, E, H, I, widths)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    out, idx, w = decode_call(layer, x, I, E, k)
    check_block(oracle.get(), x, layer.wr_np, layer.bias_np, layer.expert_fn, E, H, I, k, out, idx, w)


def test_decode_workspace_reuse_and_zero_expert():
    rng = np.random.default_rng(5)
    E, H, I, T, k = 6, 128, 64, 4, 2
    exs = [pins.make_expert(rng, H, I, 4)[0] for _ in range(E)]
    zq = [np.zeros((I, H), int), np.zeros((I, H), int), np.zeros((H, I), int)]
    zz = [synth.to_f16_bits(np.zeros((I, H // 64)))] * 2 + [synth.to_f16_bits(np.zeros((H, I // 64)))]
    exs[0] = pins.make_expert(rng, H, I, 4, q=zq, z=zz)[0]
    wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
    wr[0] = wr[1] * 3.0   # expert 0 (all-zero codes, zero point 0) is often selected
    layer = HandLayer(exs, wr, None, H, I)
    ws = qm.workspace(T, H, I, E, k, qm.MODE_DECODE)
    for trial in range(3):
        x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
        out, idx, w = decode_call(layer, x, I, E, k, ws)
        check_block(oracle.get(), x, wr, None, layer.expert_fn, E, H, I, k, out, idx, w)


def synth_decode_check(name, layer_ids, steps, tokens=None):
    w = synth.WORKLOADS[name]
    o = oracle.get()
    res = []
    for l in layer_ids:
        layer = SynthLayer(w, l)
        ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
        for s in steps:
            x = synth.hidden(w, s, l)
            out, idx, ww = decode_call(layer, x, w.I, w.E, w.k, ws)
            res.append(check_block(o, x, layer.wr_np, layer.bias_np, layer.expert_fn, w.E, w.H, w.I, w.k,
                                   out, idx, ww, tokens=tokens))
        del layer
        torch.cuda.empty_cache()
    return res


def test_decode_single_layer_config():
    print(synth_decode_check("moe_t1_h1024_e32_k4_i256_int4", [0], [0]))


def test_decode_48layer_config_sampled_layers():
    print(synth_decode_check("decode_t1_l48_h2048_e256_k8_i512_int4", [0, 47], [0, 1, 255]))


def test_decode_large_sparse_config_one_layer():
    print(synth_decode_check("decode_t1_l16_h4096_e512_k10_i1024_int4", [15], [0, 127]))


def test_decode_mixed_precision_batch16():
    print(synth_decode_check("decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1", [0], [0, 5]))


def test_decode_graph_stack_matches_oracle():
    """The launch configuration the benchmark times: a CUDA graph of several layers with
    programmatic dependent launch, one workspace shared by all layers."""
    w = synth.WORKLOADS["decode_t1_l48_h2048_e256_k8_i512_int4"]
    L = 4
    layers = [SynthLayer(w, l) for l in range(L)]
    stack = DecodeStack([LayerWeights(sl.wr, sl.bias, sl.packed) for sl in layers], w.T, w.H, w.I, w.E, w.k)
    o = oracle.get()
    for step in (0, 9):
        for l in range(L):
            sd.hidden(w, step, l, out=stack.x_in[l])
        stack.replay()
        torch.cuda.synchronize()
        assert qm.device_status(stack.ws) == qm.MOE_OK
        for l in range(L):
            check_block(o, synth.hidden(w, step, l), layers[l].wr_np, None, layers[l].expert_fn, w.E, w.H, w.I,
                        w.k, bf16_f64(stack.out[l]), stack.idx[l].cpu().numpy(), stack.wts[l].cpu().numpy())


def test_decode_workspace_shared_across_shapes():
    """One workspace, sized for the largest call, serves decode calls of different T, E and k in
    any order (its fixed regions keep the call tags, accumulators and counters consistent)."""
    rng = np.random.default_rng(11)
    H, I = 128, 64
    la = hand_layer(rng, 8, H, I, [4])
    lb = hand_layer(rng, 20, H, I, [6, 4])
    ws = qm.workspace(32, H, I, 20, 5, qm.MODE_DECODE)
    for layer, E, k, T in ((la, 8, 2, 3), (lb, 20, 4, 11), (la, 8, 2, 1), (lb, 20, 5, 32), (la, 8, 1, 7)):
        x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
        out, idx, w = decode_call(layer, x, I, E, k, ws)
        check_block(oracle.get(), x, layer.wr_np, layer.bias_np, layer.expert_fn, E, H, I, k, out, idx, w)


@pytest.mark.parametrize("E,k,dups", [
    (16, 16, [(2, 5), (0, 15)]),      # one expert per lane: ties between lanes (the exact fallback)
    (40, 32, [(3, 35), (10, 20)]),    # a tie inside a lane (3, 35) and one between lanes (10, 20)
    (64, 8, [(3, 35), (10, 20), (0, 63)]),    # the merging selection (k <= 8): ties across lanes and lists
    (256, 4, [(7, 200), (100, 101)])])
def test_decode_exact_ties_take_lower_index(E, k, dups):
    rng = np.random.default_rng(E * 31 + k)
    T, H, I = 5, 128, 64
    layer0 = hand_layer(rng, E, H, I, [4], bias=False)
    wr = layer0.wr_np.copy()
    for lo, hi in dups:
        wr[hi] = wr[lo]            # identical logits in every precision
    layer = HandLayer(layer0.experts_np, wr, None, H, I)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    out, idx, w = decode_call(layer, x, I, E, k)
    for t in range(T):
        pos = {int(e): i for i, e in enumerate(idx[t])}
        for lo, hi in dups:
            if lo in pos and hi in pos:
                assert pos[lo] < pos[hi], (t, lo, hi, idx[t])   # equal logits: lower index first
    check_block(oracle.get(), x, layer.wr_np, layer.bias_np, layer.expert_fn, E, H, I, k, out, idx, w)
