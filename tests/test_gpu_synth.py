"""The device copy of the input generator reproduces the numpy generator bit for bit."""
import numpy as np
import pytest
import torch

import synth
import synth.device as sd
from gpu_support import bf16_bits

pytestmark = pytest.mark.gpu


def test_hidden_and_router_bitwise():
    for name in ("decode_t1_l48_h2048_e256_k8_i512_int4", "prefill_t4096_l8_h2048_e256_k8_i512_int4"):
        w = synth.WORKLOADS[name]
        for step, layer in ((0, 0), (3, 7)):
            assert np.array_equal(bf16_bits(sd.hidden(w, step, layer)), synth.hidden(w, step, layer))
    w = synth.WORKLOADS["decode_t1_l16_h4096_e512_k10_i1024_int4"]
    assert np.array_equal(sd.router_weights(w, 2).cpu().numpy(), synth.router_weights(w, 2))


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_expert_tensors_bitwise(bits):
    w = synth.WORKLOADS["decode_t16_l24_h2048_e256_k8_i768_mixed468_zipf1.1"]
    dev = sd.expert_tensors(w, 3, 17, bits)
    host = synth.expert_tensors(w, 3, 17, bits)
    for m in range(3):
        assert np.array_equal(dev["codes"][m].cpu().numpy(), host["codes"][m])
        assert np.array_equal(dev["scale"][m].cpu().view(torch.int16).numpy().view(np.uint16), host["scale"][m])
        assert np.array_equal(dev["zero"][m].cpu().view(torch.int16).numpy().view(np.uint16), host["zero"][m])
