"""moe_expert_forward_decode_noalloc: the decode entry point for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc at all -- an operator plugin that its host
runtime hands only input and output buffers, or a process whose device memory belongs to
another allocator -- so they cannot provide the workspace that moe_expert_forward_decode needs.
This entry point uses a fixed scratch array inside the library instead. The tests call it
through the C ABI on calls of different shapes in a row (the array keeps the previous call's
contents, so later calls check that the kernel clears what must start at zero, also when the
shape changes), compare each call with the fp64 oracle and with the workspace entry point, read
its device status through moe_noalloc_get_device_status after an expired wait, and check that
unsupported shapes are refused on the host.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from gpu_support import SynthLayer, bf16_f64, to_dev_bf16
from parity import TOL, check_block, output_error

pytestmark = pytest.mark.gpu

MIXED = "decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1"
SINGLE = "decode_t1_l48_h2048_e256_k8_i512_int4"


def noalloc_call(layer, w, x_bits):
    """One moe_expert_forward_decode_noalloc call through the C ABI: (out, idx, weights)."""
    L = qm.lib()
    x = to_dev_bf16(x_bits)
    out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((w.T, w.k), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((w.T, w.k), dtype=torch.float32, device="cuda")
    rc = L.moe_expert_forward_decode_noalloc(x.data_ptr(), layer.wr.data_ptr(),
                                             None if layer.bias is None else layer.bias.data_ptr(),
                                             layer.packed.data_ptr(), w.T, w.H, w.I, w.E, w.k, out.data_ptr(),
                                             idx.data_ptr(), wts.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == qm.MOE_OK, qm.status_name(rc)
    assert L.moe_noalloc_get_device_status(torch.cuda.current_stream().cuda_stream) == qm.MOE_OK
    return x, out, idx, wts


def test_noalloc_shape_changes_match_oracle_and_workspace_call():
    o = oracle.get()
    layers = {name: SynthLayer(synth.WORKLOADS[name], 3) for name in (MIXED, SINGLE)}
    # 16 mixed-width tokens, then one token (a smaller output region over the previous call's
    # leftovers), then 16 tokens again, then one token again
    for name, step in ((MIXED, 0), (SINGLE, 1), (MIXED, 2), (SINGLE, 3)):
        w, layer = synth.WORKLOADS[name], layers[name]
        x_bits = synth.hidden(w, step, 3)
        x, out, idx, wts = noalloc_call(layer, w, x_bits)
        got = bf16_f64(out)
        assert np.isfinite(got).all()
        check_block(o, x_bits, layer.wr_np, layer.bias_np, layer.expert_fn, w.E, w.H, w.I, w.k, got,
                    idx.cpu().numpy(), wts.cpu().numpy())
        ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
        ref_idx = torch.zeros_like(idx)
        ref_w = torch.zeros_like(wts)
        ref = qm.forward_decode(x, layer.wr, layer.bias, layer.packed, w.I, w.E, w.k, ws, idx_out=ref_idx, w_out=ref_w)
        assert qm.device_status(ws) == qm.MOE_OK
        assert torch.equal(idx, ref_idx)
        assert torch.allclose(wts, ref_w, rtol=0, atol=1e-6)
        assert output_error(got, bf16_f64(ref)) <= TOL


def test_noalloc_status_after_an_expired_wait():
    name = "moe_t1_h1024_e32_k4_i256_int4"
    w = synth.WORKLOADS[name]
    layer = SynthLayer(w, 0)
    L = qm.lib()
    stream = torch.cuda.current_stream().cuda_stream
    x = to_dev_bf16(synth.hidden(w, 0, 0))
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    try:
        qm.set_wait_limit_ns(0)
        rc = L.moe_expert_forward_decode_noalloc(x.data_ptr(), layer.wr.data_ptr(), None, layer.packed.data_ptr(),
                                                 w.T, w.H, w.I, w.E, w.k, out.data_ptr(), None, None, stream)
        assert rc == qm.MOE_OK
        assert L.moe_noalloc_get_device_status(stream) == qm.MOE_ERR_TIMEOUT
    finally:
        qm.set_wait_limit_ns(2_000_000_000)
    assert L.moe_noalloc_get_device_status(stream) == qm.MOE_OK   # cleared
    x_bits = synth.hidden(w, 1, 0)
    _, out, idx, wts = noalloc_call(layer, w, x_bits)
    check_block(oracle.get(), x_bits, layer.wr_np, None, layer.expert_fn, w.E, w.H, w.I, w.k, bf16_f64(out),
                idx.cpu().numpy(), wts.cpu().numpy())


def test_noalloc_refuses_unsupported_shapes_on_the_host():
    # 33 tokens (decode takes at most 32) and H = 16384 (at most 8192), with real buffers of those
    # sizes: the call must return MOE_ERR_UNSUPPORTED without launching anything
    L = qm.lib()
    stream = torch.cuda.current_stream().cuda_stream
    E, k, I = 8, 2, 64
    for T, H in ((33, 128), (1, 16384)):
        x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
        wr = torch.zeros((E, H), dtype=torch.float32, device="cuda")
        packed = torch.zeros(qm.packed_layer_bytes(E, H, I, [4] * E), dtype=torch.uint8, device="cuda")
        out = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
        rc = L.moe_expert_forward_decode_noalloc(x.data_ptr(), wr.data_ptr(), None, packed.data_ptr(), T, H, I, E, k,
                                                 out.data_ptr(), None, None, stream)
        assert rc == qm.MOE_ERR_UNSUPPORTED
    assert L.moe_noalloc_get_device_status(stream) == qm.MOE_OK
