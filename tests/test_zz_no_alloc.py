"""moe_expert_forward_decode_noalloc: the decode entry point for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc at all -- an operator plugin that its host
runtime hands only input and output buffers, or a process whose device memory belongs to
another allocator -- so they cannot provide the workspace that moe_expert_forward_decode needs.
This entry point uses a fixed scratch array inside the library instead. The test calls it
through the C ABI twice in a row (the array keeps the previous call's contents, so the second
call checks that the kernel clears what must start at zero) and compares each output and
routing with the workspace entry point's, within the tolerance the parity tests use. It also
checks that a shape whose scratch does not fit is refused before anything runs.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
import quantized_moe_router_b200 as qm
from gpu_support import SynthLayer, bf16_f64, to_dev_bf16
from parity import TOL, output_error

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    w = synth.WORKLOADS["decode_t1_l48_h2048_e256_k8_i512_int4"]
    layer = SynthLayer(w, 5)
    L = qm.lib()
    ws = qm.workspace(w.T, w.H, w.I, w.E, w.k, qm.MODE_DECODE)
    stream = torch.cuda.current_stream().cuda_stream
    for step in (3, 4):
        x = to_dev_bf16(synth.hidden(w, step, 5))
        ref = qm.forward_decode(x, layer.wr, None, layer.packed, w.I, w.E, w.k, ws)
        out = torch.full((w.T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        idx = torch.full((w.T, w.k), -1, dtype=torch.int32, device="cuda")
        wts = torch.zeros((w.T, w.k), dtype=torch.float32, device="cuda")
        rc = L.moe_expert_forward_decode_noalloc(x.data_ptr(), layer.wr.data_ptr(), None, layer.packed.data_ptr(),
                                                 w.T, w.H, w.I, w.E, w.k, out.data_ptr(), idx.data_ptr(),
                                                 wts.data_ptr(), stream)
        assert rc == qm.MOE_OK, qm.status_name(rc)
        torch.cuda.synchronize()
        assert qm.device_status(ws) == qm.MOE_OK
        ref_idx = torch.zeros_like(idx)
        ref_w = torch.zeros_like(wts)
        qm.forward_decode(x, layer.wr, None, layer.packed, w.I, w.E, w.k, ws, idx_out=ref_idx, w_out=ref_w)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.allclose(wts, ref_w, rtol=0, atol=1e-6)
        err = output_error(bf16_f64(out), bf16_f64(ref))
        assert np.isfinite(bf16_f64(out)).all() and err <= TOL, err


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # T=32 tokens x k=8 with I=4096 needs 8 MiB of decode scratch: more than the fixed 4 MiB
    L = qm.lib()
    T, H, I, E, k = 32, 2048, 4096, 64, 8
    assert L.moe_workspace_bytes(T, H, I, E, k, qm.MODE_DECODE) > (4 << 20)
    dev = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dev.data_ptr()
    rc = L.moe_expert_forward_decode_noalloc(p, p, None, p, T, H, I, E, k, p, None, None,
                                             torch.cuda.current_stream().cuda_stream)
    assert rc == qm.MOE_ERR_UNSUPPORTED
