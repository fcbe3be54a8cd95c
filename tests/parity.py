"""GPU-vs-oracle comparison of one expert-block call, with near-tie accounting.

Rules (applied per token):
  * top-k sets must be identical wherever the oracle's gap between the k-th and (k+1)-th
    logit exceeds TIE (1e-4);
  * where the gap is <= TIE the GPU may pick another set S', provided every logit of S' is
    >= l_(k) - TIE; the tie is counted and the oracle is re-run with S' (weights = softmax
    of the oracle's logits over S');
  * with equal sets, a different order is allowed only between logits within TIE (counted);
  * routing weights must match the oracle's within WTOL (absolute);
  * the call's output must satisfy max|gpu - ref| / max|ref| <= TOL (5e-3).
"""
from __future__ import annotations

import numpy as np

TOL = 5e-3
TIE = 1e-4
WTOL = 2e-5


def route_check(logits: np.ndarray, k: int, gpu_idx: np.ndarray, gpu_w=None):
    """Returns (idx, w, stats) to run the oracle with, after checking the GPU's routing."""
    T, E = logits.shape
    stats = {"tokens": T, "near_ties": 0, "order_swaps": 0}
    use_idx = np.empty((T, k), np.int64)
    use_w = np.empty((T, k), np.float64)
    for t in range(T):
        l = logits[t]
        order = np.argsort(-l, kind="stable")
        ref = order[:k]
        g = np.asarray(gpu_idx[t], np.int64)
        assert len(set(g.tolist())) == k and g.min() >= 0 and g.max() < E, (t, g)
        lk = l[ref[-1]]
        lk1 = l[order[k]] if k < E else -np.inf
        if set(g.tolist()) != set(ref.tolist()):
            assert lk - lk1 <= TIE, f"token {t}: top-k differs with gap {lk - lk1:.3e}: gpu {g} ref {ref}"
            assert np.all(l[g] >= lk - TIE), f"token {t}: gpu picked a non-tied expert"
            stats["near_ties"] += 1
        elif not np.array_equal(g, ref):
            # same set, other order: only among near-equal logits
            assert np.all(np.abs(l[g] - l[ref]) <= TIE), f"token {t}: order differs: {g} vs {ref}"
            stats["order_swaps"] += 1
        lg = l[g]
        ww = np.exp(lg - lg.max())
        ww /= ww.sum()
        use_idx[t] = g
        use_w[t] = ww
        if gpu_w is not None:
            err = np.max(np.abs(np.asarray(gpu_w[t], np.float64) - ww))
            assert err <= WTOL, f"token {t}: routing weights differ by {err:.3e}"
    return use_idx, use_w, stats


def output_error(gpu_out: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(gpu_out.astype(np.float64) - ref)) / max(np.max(np.abs(ref)), 1e-300))


def check_block(o, x_bits, wr, bias, expert_fn, E, H, I, k, gpu_out, gpu_idx, gpu_w, tokens=None):
    """Full check of one call. tokens: subset of token rows to compare (None = all)."""
    if tokens is not None:
        x_bits = x_bits[tokens]
        gpu_out = gpu_out[tokens]
        gpu_idx = gpu_idx[tokens]
        gpu_w = None if gpu_w is None else gpu_w[tokens]
    logits = o.router_logits(x_bits, wr, bias)
    idx, w, stats = route_check(logits, k, gpu_idx, gpu_w)
    experts = [None] * E
    for e in np.unique(idx):
        experts[int(e)] = expert_fn(int(e))
    ref = o.combine(x_bits, experts, H, I, idx, w)
    err = output_error(gpu_out, ref)
    stats["err"] = err
    assert err <= TOL, f"output error {err:.3e} > {TOL}"
    return stats
