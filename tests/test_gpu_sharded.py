"""Unit sharding on one GPU: two ranks' shares of one cache computed one after the other (the
all-gather replaced by concatenating their distortion rows), then one allocation and each
rank's encoding.  With the global index of its first unit passed to the library, a shard's
factors, tables and stored bytes are those of the same units in a one-rank compress of the
whole cache at the same payload budget, bit for bit."""
import pytest
import torch

from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import sharded as SH
from kv_cache_compression_group_b200 import synth

pytestmark = pytest.mark.gpu


def _payload(blob_np, rec, T, D, S):
    """The bytes of one stored unit: U, W, core, codes, scales."""
    parts = [blob_np[rec["off_U"]:rec["off_U"] + 2 * T * rec["r_T"]],
             blob_np[rec["off_W"]:rec["off_W"] + 2 * D * rec["r_D"]],
             blob_np[rec["off_C"]:rec["off_C"] + 2 * S * rec["r_T"] * rec["r_D"]]]
    if rec["bits"]:
        nblk = S * T * D // 16
        parts.append(blob_np[rec["off_codes"]:rec["off_codes"] + nblk * 2 * rec["bits"]])
        parts.append(blob_np[rec["off_scales"]:rec["off_scales"] + nblk * 4])
    return b"".join(p.tobytes() for p in parts)


@pytest.mark.parametrize("method", ["randomized", "exact"])
def test_shards_equal_one_rank_compress(method):
    w = synth.small_workload("mistral7b", n_layers=12, n_heads=2, T=256)
    K, V = (t.cuda() for t in synth.make_cache(w, 0))
    opts = J.default_options(w.T, w.D, method)
    world, NU, S = 2, 2 * w.n_groups, w.layers_per_group * w.n_heads
    shards = [SH.ShardedCompressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts, world, r)
              for r in range(world)]
    locs = [(K[sc.sp.layers.start:sc.sp.layers.stop].contiguous(), V[sc.sp.layers.start:sc.sp.layers.stop].contiguous())
            for sc in shards]
    states = [sc.local_tables(Kl, Vl, 0) for sc, (Kl, Vl) in zip(shards, locs)]
    full = torch.cat([s["table"] for s in states])
    budget = w.bf16_bytes() // 2
    avail = SH.payload_budget(budget, NU, world)
    nbytes = torch.tensor(shards[0].bytes_row, dtype=torch.int64, device="cuda").unsqueeze(0).expand(NU, -1)
    choice, lam, st = J.allocate(full, nbytes.contiguous(), avail)
    assert st.item() == 0
    blobs = [sc.encode(Kl, Vl, s, full, choice) for sc, (Kl, Vl), s in zip(shards, locs, states)]

    # one rank over the whole cache, same payload budget (one global header instead of two)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    U, W = comp.factor(K, V, 0)
    _, tab = comp.table(K, V, U.to(torch.bfloat16), W.to(torch.bfloat16), 0)
    assert torch.equal(tab, full)                                   # same rows, bit for bit
    ref = comp.compress(K, V, avail + 64 + 64 * NU, 0)
    _, ref_total, ref_recs = J.read_header(ref)
    assert [r["choice"] for r in ref_recs] == choice.cpu().tolist()
    ref_np = ref[:ref_total].cpu().numpy()
    Kr, Vr = comp.decompress(ref, torch.float32)
    total = 0
    for sc, blob in zip(shards, blobs):
        _, tot, recs = J.read_header(blob)
        total += tot
        bnp = blob[:tot].cpu().numpy()
        for i, rec in enumerate(recs):
            u = sc.sp.u0 + i
            assert (rec["r_T"], rec["r_D"], rec["bits"]) == (ref_recs[u]["r_T"], ref_recs[u]["r_D"], ref_recs[u]["bits"])
            assert _payload(bnp, rec, w.T, w.D, S) == _payload(ref_np, ref_recs[u], w.T, w.D, S), u
        Ks, Vs = sc.comp.decompress(blob, torch.float32)
        lay = slice(sc.sp.layers.start, sc.sp.layers.stop)
        assert torch.equal(Ks, Kr[lay]) and torch.equal(Vs, Vr[lay])
    assert total <= budget and total == ref_total + 64
