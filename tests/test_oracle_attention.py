"""Pins of the oracle's decode-side attention over the stored factors: for every unit of small
compressed caches (JoLT and FlashJoLT, budgets that pick residual bit-widths 0 to 8), the
scores and outputs computed from U, P', the codes and the fp16 scales equal plain softmax
attention over the decompressed cache, X_hat q and p^T X_hat formed densely."""
import math

import numpy as np
import pytest

import oracle as O
from kv_cache_compression_group_b200 import synth


def _dense(Kh, Vh, q):
    s = q @ Kh.T / math.sqrt(q.shape[-1])
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return p, p @ Vh


@pytest.mark.parametrize("method,ratio", [("exact", 2.0), ("exact", 4.0), ("randomized", 3.0), ("randomized", 8.0)])
def test_factored_attention_equals_dense(method, ratio):
    w = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=64)
    K, V = synth.make_cache(w, 3, workers=1)
    K, V = K.float().numpy().astype(np.float64), V.float().numpy().astype(np.float64)
    opts = O.Options(token_ranks=(4, 8, 16), feature_ranks=(4, 8, w.D), bits=(0, 1, 2, 3, 4, 8), method=method)
    budget = O.budget_for_ratio(w.n_layers, w.n_heads, w.T, w.D, ratio)
    res = O.compress(K, V, w.layers_per_group, opts, budget, seed=11)
    assert res.status == "ok"
    Kh, Vh = O.decompress(res)
    rng = np.random.default_rng(5)
    by_unit = {(r.group, r.kv): r for r in res.units}
    seen_bits = set()
    for g in range(w.n_layers // w.layers_per_group):
        rk, rv = by_unit[(g, 0)], by_unit[(g, 1)]
        seen_bits |= {rk.b, rv.b}
        for l in range(w.layers_per_group):
            for h in range(w.n_heads):
                q = rng.standard_normal((3, w.D))
                p, out = O.slice_attention_factored(rk, rv, l, h, q)
                L = g * w.layers_per_group + l
                pd, od = _dense(Kh[L, h], Vh[L, h], q)
                np.testing.assert_allclose(p, pd, rtol=1e-10, atol=1e-13)
                np.testing.assert_allclose(out, od, rtol=1e-10, atol=1e-12)
                # scores alone (before the softmax), against X_hat q
                np.testing.assert_allclose(O.slice_scores_factored(rk, l, h, q), q @ Kh[L, h].T, rtol=1e-10,
                                           atol=1e-10)
    assert seen_bits   # the records exist; which bit-widths appear depends on the budget


def test_every_bit_width_is_exercised():
    """The budgets above must reach both the residual-free and the residual cases."""
    w = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=64)
    K, V = synth.make_cache(w, 3, workers=1)
    K, V = K.float().numpy().astype(np.float64), V.float().numpy().astype(np.float64)
    bits = set()
    for method, ratio in [("exact", 2.0), ("exact", 4.0), ("randomized", 3.0), ("randomized", 8.0)]:
        opts = O.Options(token_ranks=(4, 8, 16), feature_ranks=(4, 8, w.D), bits=(0, 1, 2, 3, 4, 8), method=method)
        res = O.compress(K, V, w.layers_per_group, opts, O.budget_for_ratio(w.n_layers, w.n_heads, w.T, w.D, ratio),
                         seed=11)
        bits |= {r.b for r in res.units}
    assert 0 in bits and len(bits - {0}) >= 2, bits
