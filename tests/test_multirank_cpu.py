"""The multi-process path on CPU: two gloo ranks run the rank plumbing the benchmark uses
(environment, seeds, barrier, max over ranks, whole-job throughput) and the host-side
preparation of their caches and budgets."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from kv_cache_compression_group_b200 import ranks, synth
    from kv_cache_compression_group_b200 import jolt as J
    r, w, local = ranks.dist_env()
    ranks.init(w, backend="gloo", timeout_s=30)
    try:
        # each rank its own cache: different seeds, reproducible
        wl = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=128)
        K, V = synth.make_cache(wl, ranks.rank_seed(r), workers=1)
        K2, _ = synth.make_cache(wl, ranks.rank_seed(r), workers=1)
        # the same budgets and candidate sets on every rank
        opts = J.default_options(wl.T, wl.D, "randomized")
        budgets = [int(wl.bf16_bytes() / x) for x in (2.0, 3.0)]
        ranks.barrier(w)
        t_ms = 10.0 + 5.0 * r               # a fake device time per rank
        t_max = ranks.max_over_ranks(t_ms, w)
        value = ranks.aggregate_gbs(w, 2 * wl.input_bytes(), t_max)
        q.put(dict(rank=r, world=w, local=local, k0=float(K.float().sum()), same=bool(torch.equal(K, K2)),
                   t_max=t_max, value=value, budgets=budgets, ranks=list(opts.token_ranks)))
    finally:
        ranks.shutdown(w)


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda d: d["rank"])
    assert [d["rank"] for d in out] == [0, 1] and all(d["world"] == 2 for d in out)
    assert [d["local"] for d in out] == [0, 1]
    assert all(d["same"] for d in out)                      # a rank's cache is reproducible
    assert out[0]["k0"] != out[1]["k0"]                       # ranks compress different caches
    assert out[0]["t_max"] == out[1]["t_max"] == 15.0         # max over ranks, seen by every rank
    assert out[0]["value"] == out[1]["value"]
    from kv_cache_compression_group_b200 import synth
    wl = synth.small_workload("mistral7b", n_layers=4, n_heads=2, T=128)
    assert out[0]["value"] == pytest.approx(2 * 2 * wl.input_bytes() / 15e-3 / 1e9)
    assert out[0]["budgets"] == out[1]["budgets"] and out[0]["ranks"] == out[1]["ranks"]


def test_single_rank_defaults(monkeypatch):
    from kv_cache_compression_group_b200 import ranks
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert ranks.dist_env() == (0, 1, 0)
    ranks.init(1)
    ranks.barrier(1)
    assert ranks.max_over_ranks(3.5, 1) == 3.5
    assert ranks.aggregate_gbs(1, 1e9, 1000.0) == pytest.approx(1.0)
