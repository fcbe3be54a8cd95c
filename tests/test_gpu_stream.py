"""Experts streamed from host memory through an ExpertCache (moe_cache_*), against the resident
layer and the fp64 oracle, with fewer device slots than the experts the calls touch."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from quantized_moe_router_b200.runner import forward_through_cache
from gpu_support import HandLayer, bf16_f64, to_dev_bf16
from parity import check_block, output_error
from tests_support import pins_module

pytestmark = pytest.mark.gpu
pins = pins_module()


def layers(rng, L, E, H, I, widths):
    out = []
    for _ in range(L):
        exs = [pins.make_expert(rng, H, I, widths[e % len(widths)])[0] for e in range(E)]
        wr = (rng.normal(0, 1, (E, H)) / np.sqrt(H)).astype(np.float32)
        out.append(HandLayer(exs, wr, None, H, I))
    return out


@pytest.mark.parametrize("mode", [qm.MODE_DECODE, qm.MODE_PREFILL])
def test_layers_through_the_cache(mode):
    rng = np.random.default_rng(31 + mode)
    Lc, E, H, I, k, T = 3, 16, 256, 128, 2, 3
    lay = layers(rng, Lc, E, H, I, [4, 6, 8])
    host = [hl.packed.cpu().pin_memory() for hl in lay]
    cache = qm.ExpertCache(host, slots=6)
    ws = qm.workspace(T, H, I, E, k, mode)
    ws_ref = qm.workspace(T, H, I, E, k, mode)
    o = oracle.get()
    fwd = qm.forward_decode if mode == qm.MODE_DECODE else qm.forward_prefill
    for step in range(3):
        for l, hl in enumerate(lay):
            xb = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
            x = to_dev_bf16(xb)
            out, idx, w = forward_through_cache(cache, l, x, hl.wr, None, I, E, k, ws, mode=mode)
            assert qm.device_status(ws) == qm.MOE_OK
            idx_r = torch.empty_like(idx)
            w_r = torch.empty_like(w)
            ref = fwd(x, hl.wr, None, hl.packed, I, E, k, ws_ref, idx_out=idx_r, w_out=w_r)
            assert qm.device_status(ws_ref) == qm.MOE_OK
            assert torch.equal(idx, idx_r)
            assert torch.allclose(w, w_r, rtol=0, atol=1e-6)
            # the same kernel on the same bytes; its partial sums arrive in varying order, which
            # can move an output by one bf16 unit (2^-7 relative at most)
            assert output_error(bf16_f64(out), bf16_f64(ref)) <= 2.0 ** -7
            check_block(o, xb, hl.wr_np, None, hl.expert_fn, E, H, I, k, bf16_f64(out), idx.cpu().numpy(),
                        w.cpu().numpy())
    st = cache.stats()
    assert st["misses"] > 6 and st["evictions"] > 0, st   # the calls need more experts than slots
    cache.close()
