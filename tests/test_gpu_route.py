"""moe_route_topk against the oracle's fp64 logits and top-k."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_router_b200 as qm
from gpu_support import to_dev_bf16
from parity import route_check

pytestmark = pytest.mark.gpu


def run(T, H, E, k, seed, bias=False, dup_rows=False, scale=1.0):
    rng = np.random.default_rng(seed)
    x = synth.to_bf16_bits(rng.normal(0, 1, (T, H)))
    wr = (rng.normal(0, scale, (E, H)) / np.sqrt(H)).astype(np.float32)
    if dup_rows:
        wr[5] = wr[2]          # exact ties: identical logits in every precision
        wr[E - 1] = wr[0]
    b = rng.normal(0, 0.5, E).astype(np.float32) if bias else None
    idx, w = qm.route_topk(to_dev_bf16(x), torch.from_numpy(wr).cuda(),
                           None if b is None else torch.from_numpy(b).cuda(), k)
    torch.cuda.synchronize()
    logits = oracle.get().router_logits(x, wr, b)
    return logits, idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,H,E,k,bias", [
    (1, 128, 8, 2, False), (37, 256, 64, 5, True), (1, 1024, 32, 4, False), (5, 2048, 256, 8, False),
    (3, 4096, 512, 10, False), (16, 2048, 256, 8, True), (9, 64, 1024, 32, True), (7, 128, 32, 32, False),
    (1000, 2048, 256, 8, False), (13, 8192, 128, 1, True)])
def test_route_matches_oracle(T, H, E, k, bias):
    logits, idx, w = run(T, H, E, k, seed=T * 7 + E, bias=bias)
    route_check(logits, k, idx, w)


def test_route_full_prefill_size():
    w = synth.WORKLOADS["prefill_t4096_l8_h2048_e256_k8_i512_int4"]
    x = synth.hidden(w, 0, 0)
    wr = synth.router_weights(w, 0)
    idx, ww = qm.route_topk(to_dev_bf16(x), torch.from_numpy(wr).cuda(), None, w.k)
    logits = oracle.get().router_logits(x, wr, None)
    _, _, stats = route_check(logits, w.k, idx.cpu().numpy(), ww.cpu().numpy())
    print("near ties", stats)


def test_k_above_limit_rejected():
    with pytest.raises(qm.MoeError) as ei:
        run(7, 128, 33, 33, seed=1)
    assert ei.value.status == qm.MOE_ERR_INVALID_ARG


def test_exact_ties_take_lower_index():
    logits, idx, w = run(64, 256, 16, 16, seed=3, dup_rows=True)
    for t in range(64):
        pos = {int(e): i for i, e in enumerate(idx[t])}
        assert pos[2] < pos[5] and pos[0] < pos[15]   # equal logits: lower index first
        assert np.array_equal(np.sort(idx[t]), np.arange(16))
    route_check(logits, 16, idx, w)
