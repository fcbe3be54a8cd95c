"""Bounded device-side waits: with a zero wait limit the decode kernel's grid barriers expire,
the kernel returns with MOE_ERR_TIMEOUT in the workspace status word, the GPU context stays
usable and the next call (normal limit) is correct again."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from gpu_support import SynthLayer, bf16_f64, to_dev_bf16
from parity import check_block

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_recoverable():
    w = synth.WORKLOADS["moe_t1_h1024_e32_k4_i256_int4"]
    layer = SynthLayer(w, 0)
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    x = synth.hidden(w, 0, 0)
    try:
        qm.set_wait_limit_ns(0)
        qm.forward_decode(to_dev_bf16(x), layer.wr, None, layer.packed, w.I, w.E, w.k, ws)
        assert qm.device_status(ws) == qm.MOE_ERR_TIMEOUT
    finally:
        qm.set_wait_limit_ns(2_000_000_000)
    assert qm.device_status(ws) == qm.MOE_OK   # cleared
    idx = torch.zeros((1, w.k), dtype=torch.int32, device="cuda")
    wt = torch.zeros((1, w.k), dtype=torch.float32, device="cuda")
    out = qm.forward_decode(to_dev_bf16(x), layer.wr, None, layer.packed, w.I, w.E, w.k, ws, idx_out=idx, w_out=wt)
    assert qm.device_status(ws) == qm.MOE_OK
    check_block(oracle.get(), x, layer.wr_np, None, layer.expert_fn, w.E, w.H, w.I, w.k, bf16_f64(out),
                idx.cpu().numpy(), wt.cpu().numpy())


def test_invalid_arguments_on_device_tensors():
    w = synth.WORKLOADS["moe_t1_h1024_e32_k4_i256_int4"]
    layer = SynthLayer(w, 0)
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    x = to_dev_bf16(synth.hidden(w, 0, 0))
    with pytest.raises(qm.MoeError) as ei:
        qm.forward_decode(x, layer.wr, None, layer.packed, w.I, w.E, w.k, ws[:100])
    assert ei.value.status == qm.MOE_ERR_INVALID_ARG
    with pytest.raises(qm.MoeError) as ei:
        qm.forward_decode(x, layer.wr, None, layer.packed[16:], w.I, w.E, w.k, ws)
    assert ei.value.status == qm.MOE_ERR_INVALID_ARG
    with pytest.raises(qm.MoeError) as ei:
        qm.forward_decode(torch.zeros((33, w.H), dtype=torch.bfloat16, device="cuda"), layer.wr, None,
                          layer.packed, w.I, w.E, w.k, qm.workspace(33, w.H, w.I, w.E, w.k, qm.MODE_DECODE))
    assert ei.value.status == qm.MOE_ERR_UNSUPPORTED
