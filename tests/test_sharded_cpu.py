"""Unit sharding of one cache over ranks, on CPU: contiguous layer groups per rank, one
all-gather of the distortion tables (two gloo ranks), then the same allocation on every rank.
The tables are the float64 oracle's (the library needs a GPU); the sharding logic under test
is the product's (kv_cache_compression_group_b200/sharded.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from kv_cache_compression_group_b200 import sharded as SH


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("G,world", [(8, 2), (8, 3), (10, 4), (5, 5), (1, 1)])
def test_group_ranges_partition_the_groups(G, world):
    seen = []
    sizes = []
    for r in range(world):
        g0, g1 = SH.group_range(G, world, r)
        seen.extend(range(g0, g1))
        sizes.append(g1 - g0)
    assert seen == list(range(G))                      # contiguous, in rank order, each once
    assert max(sizes) - min(sizes) <= 1
    sp = SH.plan(G * 4, 4, world, world - 1)
    assert sum(sp.counts()) == 2 * G and sp.u0 + sp.n_local_units == 2 * G


def test_payload_budget_pays_every_blob_header():
    assert SH.payload_budget(10_000, 8, 2) == 10_000 - 2 * 64 - 8 * 64
    with pytest.raises(ValueError):
        SH.plan(8, 4, 3, 0)                            # 2 groups cannot feed 3 ranks


def _oracle_tables(K, V, lg, groups, opts, seed):
    import oracle as O
    rows = []
    for g in groups:
        for kv, X in ((0, K), (1, V)):
            Xu = np.asarray(X[g * lg:(g + 1) * lg], dtype=np.float64)
            f = O.unit_factors(Xu, g, kv, opts, seed)
            rows.append(O.distortion_table(Xu, f.U_s, f.W_s, f.C_s, f.sigma, opts).reshape(-1))
    return np.stack(rows)


def _oracle_alloc(D, B, avail):
    import oracle as O
    al = O.allocate(D.numpy(), B.numpy(), int(avail))
    return torch.as_tensor(al.choice), al.lam, 0 if al.status == "ok" else 4


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import oracle as O
    from kv_cache_compression_group_b200 import ranks, synth
    ranks.init(world, backend="gloo", timeout_s=60)
    try:
        w = synth.small_workload("mistral7b", n_layers=12, n_heads=1, T=64)
        K, V = (synth.to_f64(t) for t in synth.make_cache(w, 0, workers=1))
        opts = O.Options((8, 16, 32), (32, 64, 128), (0, 2, 4), "randomized", oversample=8, power_iters=1)
        sp = SH.plan(w.n_layers, w.layers_per_group, world, rank)
        local = torch.from_numpy(_oracle_tables(K, V, w.layers_per_group, range(sp.g0, sp.g1), opts, 0))
        bytes_row = O.bytes_table(w.T, w.D, w.layers_per_group * w.n_heads, opts).reshape(-1)
        budget = w.bf16_bytes() // 3
        full, choice, lam, status = SH.allocate_shared(local, bytes_row, budget, sp, _oracle_alloc)
        q.put(dict(rank=rank, full=full.numpy(), choice=np.asarray(choice), lam=lam, status=status,
                   g=(sp.g0, sp.g1), budget=budget, bytes=bytes_row))
    finally:
        ranks.shutdown(world)


def test_two_gloo_ranks_share_one_allocation():
    """Each rank computes the tables of its own layer groups; after the all-gather every rank
    holds the whole cache's table and picks the same choices and lambda, bit for bit equal to
    the one-rank allocation over the same table at the same payload budget, and all blobs
    together stay within the global budget."""
    import oracle as O
    from kv_cache_compression_group_b200 import synth
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=300) for _ in range(world)), key=lambda d: d["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0]["g"] == (0, 2) and out[1]["g"] == (2, 3)        # 3 groups over 2 ranks
    w = synth.small_workload("mistral7b", n_layers=12, n_heads=1, T=64)
    K, V = (synth.to_f64(t) for t in synth.make_cache(w, 0, workers=1))
    opts = O.Options((8, 16, 32), (32, 64, 128), (0, 2, 4), "randomized", oversample=8, power_iters=1)
    whole = _oracle_tables(K, V, w.layers_per_group, range(3), opts, 0)
    for d in out:
        assert d["status"] == 0
        assert np.array_equal(d["full"], whole)                       # gathered rows in unit order
    assert np.array_equal(out[0]["choice"], out[1]["choice"])
    assert np.float64(out[0]["lam"]).tobytes() == np.float64(out[1]["lam"]).tobytes()
    B = np.stack([out[0]["bytes"]] * 6)
    avail = SH.payload_budget(out[0]["budget"], 6, world)
    al = O.allocate(whole, B, avail)
    assert list(al.choice) == list(out[0]["choice"])
    assert np.float64(al.lam).tobytes() == np.float64(out[0]["lam"]).tobytes()
    total = world * 64 + 6 * 64 + sum(int(B[u, c]) for u, c in enumerate(out[0]["choice"]))
    assert total <= out[0]["budget"]
