"""Decode-side attention over the stored factors (through the C ABI) against the float64
oracle's slice_attention_factored on the same stored bytes, for JoLT and FlashJoLT at
budgets whose choices span the residual widths 0 to 8, with grouped query heads and a token
count that leaves a partial last tile.  Tolerance: 2e-5 of the largest output magnitude
(fp32 sums of at most r_T + D terms per score and T terms per output, against fp64)."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth
from blob_helpers import as_record, blob_unit

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("method", ["exact", "randomized"])
@pytest.mark.parametrize("ratio", [1.2, 2.5, 6.0])
def test_attend_against_oracle(method, ratio):
    w = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=1040)
    K, V = synth.make_cache(w, 0)
    Kd, Vd = K.cuda(), V.cuda()
    opts = J.Options((32, 64, 128, 240), (32, 64, 96, 128), (0, 1, 2, 3, 4, 8), method)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    blob = comp.compress(Kd, Vd, int(w.bf16_bytes() / ratio), 0)
    _, total, recs = J.read_header(blob)
    bnp = blob[:total].cpu().numpy()
    nq = 2 * w.n_heads
    att = J.Attention(comp, blob, nq)
    rng = np.random.default_rng(int(ratio * 10))
    g = 0
    recK = as_record(blob_unit(bnp, recs[0], w), w, recs[0], g, 0, 0)
    recV = as_record(blob_unit(bnp, recs[1], w), w, recs[1], g, 1, 0)
    print(f"\n[{method} {ratio}x] K (r_T, r_D, b) = {(recK.r_T, recK.r_D, recK.b)}, "
          f"V = {(recV.r_T, recV.r_D, recV.b)}")
    for layer in range(w.n_layers):
        q = rng.standard_normal((nq, w.D)) * 0.3
        got = att.attend(layer, torch.from_numpy(q.astype(np.float32)).cuda()).double().cpu().numpy()
        qf = q.astype(np.float32).astype(np.float64)
        for j in range(nq):
            h = j // (nq // w.n_heads)
            _, want = O.slice_attention_factored(recK, recV, layer, h, qf[j:j + 1])
            err = np.abs(got[j] - want[0]).max()
            assert err <= 2e-5 * np.abs(want).max(), (layer, j, err, np.abs(want).max())


def test_attend_argument_errors():
    w = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=256)
    K, V = synth.make_cache(w, 0)
    opts = J.default_options(w.T, w.D, "randomized")
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    blob = comp.compress(K.cuda(), V.cuda(), w.bf16_bytes() // 2, 0)
    att = J.Attention(comp, blob, 4)
    q = torch.zeros((4, w.D), device="cuda")
    with pytest.raises(J.JoltError) as e:
        att.attend(7, q)
    assert e.value.name == "INVALID_ARG"
    bad = J.Attention.__new__(J.Attention)
    bad.__dict__.update(att.__dict__)
    bad.nq = 3
    with pytest.raises(J.JoltError) as e:
        bad.attend(0, torch.zeros((3, w.D), device="cuda"))
    assert e.value.name == "INVALID_ARG"
