"""One process per GPU: the rank plumbing of the benchmark and of multi-GPU callers.

Every rank compresses its own cache (its own seed): the units of different caches are
independent and the compressor's only coupling (one byte budget) is inside one cache, so the
work shards with no data-path collective (weak scaling).  The one collective is the
max-over-ranks of the timed region, taken on the device clock of every rank.
"""
from __future__ import annotations

import os
from datetime import timedelta


def dist_env():
    """(rank, world, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, backend: str = "nccl", device=None, timeout_s: float = 120.0):
    """Join the process group (no-op for a single process).  A short timeout makes ranks
    that wait for a missing peer end with an error instead of hanging."""
    if world <= 1:
        return
    import torch.distributed as dist
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` over all ranks (every rank gets it)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of the cache a rank compresses (one independent request per rank)."""
    return rank


def aggregate_gbs(world: int, bytes_per_rank: float, t_ms_max: float) -> float:
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return world * bytes_per_rank / (t_ms_max / 1e3) / 1e9


def shutdown(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
