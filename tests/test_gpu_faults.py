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


def test_binding_refuses_wrong_tensors_before_launch():
    """Wrong dtypes, shapes and strided views are refused by the binding on the host."""
    w = synth.WORKLOADS["moe_t1_h1024_e32_k4_i256_int4"]
    layer = SynthLayer(w, 0)
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    x = to_dev_bf16(synth.hidden(w, 0, 0))
    args = (layer.wr, None, layer.packed, w.I, w.E, w.k, ws)
    with pytest.raises(ValueError, match="dtype"):
        qm.forward_decode(x.float(), *args)
    with pytest.raises(ValueError, match="dtype"):
        qm.forward_decode(x, layer.wr.double(), None, layer.packed, w.I, w.E, w.k, ws)
    with pytest.raises(ValueError, match="shape"):
        qm.forward_decode(x, layer.wr[:, :512].contiguous(), None, layer.packed, w.I, w.E, w.k, ws)
    with pytest.raises(ValueError, match="rows"):
        qm.forward_decode(x, layer.wr[:16].contiguous(), None, layer.packed, w.I, w.E, w.k, ws)
    with pytest.raises(ValueError, match="shape"):
        qm.forward_decode(x, *args, idx_out=torch.zeros((1, w.k + 1), dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="dtype"):
        qm.forward_decode(x, *args, w_out=torch.zeros((1, w.k), dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError, match="contiguous"):
        wide = torch.zeros((2, 2 * w.H), dtype=torch.bfloat16, device="cuda")
        qm.forward_decode(wide[:1, ::2], *args)
    with pytest.raises(ValueError, match="shape"):
        qm.forward_decode(x, *args, out=torch.zeros((1, w.H + 64), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError, match="dtype"):
        qm.quantize_hqq(torch.zeros((4, 128), dtype=torch.float16, device="cuda"), 4)
    assert qm.device_status(ws) == qm.MOE_OK
