"""The context baselines on the same synthetic caches, against the float64 oracle:
  * per-block b-bit quantisation of the cache itself (no factors, no rotation): per-unit
    errors within 1e-12 relative, scales and codes equal (both sides form codes in fp64);
  * cross-layer SVD: the compressor restricted to full feature rank and no residual (feature
    ranks {D}, bits {0}), end to end against the oracle's compress with the same sets;
and the relation the pages report (JoLT's error below both baselines), here on synthetic
caches at the 2x budget."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,bits", [("tiny", 4), ("mistral4", 4), ("mistral4", 2), ("mistral4", 8)])
def test_quant_baseline_against_oracle(name, bits):
    w = synth.WORKLOADS["tiny"] if name == "tiny" else synth.small_workload("mistral7b", n_layers=4)
    K, V = synth.make_cache(w, 0)
    sq, codes, scales = J.quant_baseline(K.cuda(), V.cuda(), bits, w.layers_per_group, keep_codes=True)
    sq = sq.cpu().numpy()
    codes = codes.cpu().numpy()
    scales = scales.cpu().numpy().astype(np.float64).reshape(-1, 2)
    nb_unit = w.layers_per_group * w.n_heads * w.T * w.D // 16
    ndiff = ntot = 0
    for u, (g, kv, X) in enumerate(O.units_of(synth.to_f64(K), synth.to_f64(V), w.layers_per_group)):
        c, lo, step, rhat, ok = O.quantize(X, bits)
        want = float(np.sum((X - rhat) ** 2)) if ok.all() else np.inf
        assert abs(sq[u, 0] - np.sum(X * X)) <= 1e-6 * np.sum(X * X)
        assert abs(sq[u, 1] - want) <= 1e-12 * want, (u, sq[u, 1], want)
        sc = scales[u * nb_unit:(u + 1) * nb_unit]
        assert np.array_equal(sc[:, 0], lo.reshape(-1)) and np.array_equal(sc[:, 1], step.reshape(-1))
        got = O.unpack_codes(codes[u * nb_unit * 2 * bits:(u + 1) * nb_unit * 2 * bits].reshape(nb_unit, 2 * bits),
                             bits)
        ndiff += int(np.count_nonzero(got.reshape(-1, 16) != c.reshape(-1, 16)))
        ntot += c.size
    print(f"\n[quant baseline {name} b={bits}] {ndiff} of {ntot} codes differ from the oracle's")
    assert ndiff == 0


@pytest.mark.parametrize("method", ["exact", "randomized"])
def test_cross_layer_svd_against_oracle(method):
    w = synth.small_workload("mistral7b", n_layers=4)
    K, V = synth.make_cache(w, 0)
    Kn, Vn = synth.to_f64(K), synth.to_f64(V)
    rt = J.default_options(w.T, w.D).token_ranks
    jo, oo = J.Options(rt, (w.D,), (0,), method), O.Options(rt, (w.D,), (0,), method)
    budget = w.bf16_bytes() // 2
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, jo)
    blob = comp.compress(K.cuda(), V.cuda(), budget, 0)
    _, total, recs = J.read_header(blob)
    res = O.compress(Kn, Vn, w.layers_per_group, oo, budget, 0)
    assert total <= budget
    assert [(r["r_T"], r["r_D"], r["bits"]) for r in recs] == [(u.r_T, u.r_D, u.b) for u in res.units]
    Kh, Vh = comp.decompress(blob, torch.float32)
    ek, ev = J.relative_errors(K.cuda(), V.cuda(), Kh, Vh, w.layers_per_group)
    Ko, Vo = O.decompress(res)
    assert abs(ek - O.relative_error(Kn, Ko)) <= 1e-4 and abs(ev - O.relative_error(Vn, Vo)) <= 1e-4


def test_jolt_below_both_baselines_at_2x():
    w = synth.WORKLOADS["mistral7b"]
    K, V = synth.make_cache(w, 0)
    Kd, Vd = K.cuda(), V.cuda()
    budget = w.bf16_bytes() // 2
    errs = {}
    for label, opts in (("jolt", J.default_options(w.T, w.D, "randomized")),
                        ("cross_layer_svd", J.Options(J.default_options(w.T, w.D).token_ranks, (w.D,), (0,),
                                                      "randomized"))):
        comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
        Kh, Vh = comp.decompress(comp.compress(Kd, Vd, budget, 0), torch.float32)
        errs[label] = J.relative_errors(Kd, Vd, Kh, Vh, w.layers_per_group)
    sq, _, _ = J.quant_baseline(Kd, Vd, 4, w.layers_per_group)
    sq = sq.cpu().numpy()
    errs["quant4"] = tuple(float(np.sqrt(sq[kv::2, 1].sum() / sq[kv::2, 0].sum())) for kv in (0, 1))
    print(f"\n[2x, mistral7b synthetic] relative errors (K, V): {errs} "
          f"(4-bit stores {(2 * 4 + 4) / 32:.3f} of bf16, i.e. {32 / 12:.2f}x)")
    for kv in (0, 1):
        assert errs["jolt"][kv] <= errs["cross_layer_svd"][kv] * (1 + 1e-6)
        assert errs["jolt"][kv] < errs["quant4"][kv]
