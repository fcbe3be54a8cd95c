"""Control flow of runner.forward_through_cache on the CPU, with the library calls replaced by
fakes: which experts each call asks the cache for, and the repeat of a decode call whose own
routing used an expert outside the request."""
import pytest
import torch

import quantized_moe_router_b200 as qm
from quantized_moe_router_b200 import runner


class FakeCache:
    def __init__(self):
        self.prepared = []

    def prepare(self, layer, experts, stream=None):
        self.prepared.append((layer, list(experts)))
        return ("packed", layer, tuple(experts))


def install(monkeypatch, routed, decode_uses):
    """routed: the routing call's idx; decode_uses: the idx each successive decode call reports."""
    log = {"decode": [], "experts": []}

    def route_topk(x, wr, bias, k, idx_out=None, w_out=None, stream=None):
        idx_out.copy_(torch.tensor(routed, dtype=torch.int32))
        w_out.fill_(1.0 / k)
        return idx_out, w_out

    def forward_decode(x, wr, bias, packed, I, E, k, ws, out=None, idx_out=None, w_out=None, stream=None):
        n = len(log["decode"])
        log["decode"].append(packed)
        idx_out.copy_(torch.tensor(decode_uses[min(n, len(decode_uses) - 1)], dtype=torch.int32))
        return torch.zeros(x.shape)

    def prefill_route(x, wr, bias, I, E, k, ws, idx_out=None, w_out=None, stream=None):
        idx_out.copy_(torch.tensor(routed, dtype=torch.int32))

    def prefill_experts(x, packed, I, E, k, ws, out=None, stream=None):
        log["experts"].append(packed)
        return torch.ones(x.shape)

    monkeypatch.setattr(qm, "route_topk", route_topk)
    monkeypatch.setattr(qm, "prefill_route", prefill_route)
    monkeypatch.setattr(qm, "prefill_experts", prefill_experts)
    monkeypatch.setattr(runner, "forward_decode", forward_decode)
    return log


def call(cache, mode=qm.MODE_DECODE, T=2, k=2):
    x = torch.zeros((T, 8))
    return runner.forward_through_cache(cache, 3, x, None, None, 64, 16, k, None, mode=mode)


def test_decode_inside_the_request_runs_once(monkeypatch):
    log = install(monkeypatch, [[4, 1], [1, 9]], [[[4, 1], [9, 1]]])
    cache = FakeCache()
    out, idx, w = call(cache)
    assert cache.prepared == [(3, [1, 4, 9])]
    assert log["decode"] == [("packed", 3, (1, 4, 9))]
    assert idx.tolist() == [[4, 1], [9, 1]]


def test_decode_outside_the_request_is_repeated_with_the_union(monkeypatch):
    log = install(monkeypatch, [[4, 1], [1, 9]], [[[4, 1], [1, 7]], [[4, 1], [1, 7]]])
    cache = FakeCache()
    call(cache)
    assert cache.prepared == [(3, [1, 4, 9]), (3, [1, 4, 7, 9])]
    assert len(log["decode"]) == 2


def test_decode_that_keeps_leaving_the_request_fails(monkeypatch):
    install(monkeypatch, [[0, 1], [0, 1]], [[[0, 2], [0, 1]], [[0, 3], [0, 1]], [[0, 4], [0, 1]], [[0, 5], [0, 1]]])
    with pytest.raises(RuntimeError, match="outside the cache request"):
        call(FakeCache())


def test_prefill_prepares_exactly_the_routed_experts(monkeypatch):
    log = install(monkeypatch, [[5, 2], [2, 11], [0, 5]], [])
    cache = FakeCache()
    out, idx, w = call(cache, mode=qm.MODE_PREFILL, T=3)
    assert cache.prepared == [(3, [0, 2, 5, 11])]
    assert log["experts"] == [("packed", 3, (0, 2, 5, 11))]
    assert torch.equal(out, torch.ones((3, 8)))
