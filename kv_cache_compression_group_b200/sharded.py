"""One cache's layer groups sharded over ranks (one process per GPU).

The compressor's units (layer group g, K or V) are independent through the factors, the
distortion table and the encoding; the single coupling is the one byte budget that the
Lagrangian dual spreads over all of them ("A JoLT for the KV cache: Near-Lossless KV Cache
Compression via Joint Rank-bit Allocation", abstract: one dual sets the ranks and bit-widths
of every group under a single global byte limit; AI Radio episode, "The Core Mechanism":
bytes move between groups and between K and V).  So a cache too large or too slow for one
GPU shards by layer groups:

  * rank r holds a contiguous range of layer groups (K and V of a group on the same rank) and
    computes their factors and distortion table with the library, passing the global index
    of its first unit so the rotation signs and sketches are those of the whole cache;
  * one all-gather of the distortion tables (n_units x n_choices fp64, a few KB); the byte
    cost of a choice is the same for every unit;
  * every rank runs the same deterministic allocation over all units (identical inputs give
    identical choices and lambda on every rank) and encodes its own units into its own blob.

The byte budget covers every rank's blob: each blob has its own 64-byte global header and 64
bytes per unit, so the payload available to the dual is budget - 64 * world - 64 * n_units.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

GLOBAL_HEADER_BYTES = 64
UNIT_HEADER_BYTES = 64


def group_range(n_groups: int, world: int, rank: int):
    """Contiguous layer groups [g0, g1) of `rank`: the first n_groups % world ranks take one
    group more than the others."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    base, rem = divmod(n_groups, world)
    g0 = rank * base + min(rank, rem)
    return g0, g0 + base + (1 if rank < rem else 0)


def payload_budget(budget: int, n_units: int, world: int) -> int:
    """Bytes of the global budget left to the dual once every rank's blob headers are paid."""
    return int(budget) - GLOBAL_HEADER_BYTES * world - UNIT_HEADER_BYTES * n_units


def gather_tables(local, counts, world, all_gather=None):
    """All units' distortion tables in unit order from every rank's local rows.

    local: [n_local, n_choices] tensor of this rank; counts: units per rank.  The collective
    moves equal-sized buffers (padded to the largest count); rows are concatenated in rank
    order, which is unit order because the ranks hold contiguous layer groups."""
    import torch
    if world == 1:
        return local
    width = local.shape[1]
    mx = max(counts)
    pad = torch.zeros((mx, width), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    if all_gather is None:
        import torch.distributed as dist
        dist.all_gather(parts, pad)
    else:
        all_gather(parts, pad)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)


@dataclass
class ShardPlan:
    n_groups: int
    world: int
    rank: int
    g0: int
    g1: int
    layers_per_group: int

    @property
    def n_units(self) -> int:
        return 2 * self.n_groups

    @property
    def u0(self) -> int:
        return 2 * self.g0

    @property
    def n_local_units(self) -> int:
        return 2 * (self.g1 - self.g0)

    @property
    def layers(self):
        return range(self.g0 * self.layers_per_group, self.g1 * self.layers_per_group)

    def counts(self):
        return [2 * (b - a) for a, b in (group_range(self.n_groups, self.world, r) for r in range(self.world))]


def plan(n_layers: int, layers_per_group: int, world: int, rank: int) -> ShardPlan:
    G = n_layers // layers_per_group
    if G < world:
        raise ValueError(f"{G} layer groups cannot be spread over {world} ranks")
    g0, g1 = group_range(G, world, rank)
    return ShardPlan(G, world, rank, g0, g1, layers_per_group)


def allocate_shared(local_table, bytes_row, budget: int, sp: ShardPlan, allocate_fn, all_gather=None):
    """The one collective step: gather every rank's distortion rows, then the same allocation
    on every rank.  allocate_fn(table [units, choices], bytes [units, choices], payload budget)
    returns (choices, lambda, status) with status 0 when feasible.  Returns (table, choices,
    lambda, status) -- identical on every rank."""
    import torch
    full = gather_tables(local_table, sp.counts(), sp.world, all_gather)
    nbytes = torch.as_tensor(list(bytes_row), dtype=torch.int64, device=full.device)
    nbytes = nbytes.unsqueeze(0).expand(sp.n_units, -1).contiguous()
    avail = payload_budget(budget, sp.n_units, sp.world)
    if avail < 0:
        return full, None, float("inf"), 4
    choice, lam, status = allocate_fn(full, nbytes, avail)
    return full, choice, lam, status


class ShardedCompressor:
    """This rank's share of a compress over `world` ranks, through the library's stage entry
    points (jolt_factor, jolt_table, jolt_allocate, jolt_encode) on this rank's layers."""

    def __init__(self, n_layers, n_heads, n_tokens, head_dim, layers_per_group, dtype, opts, world, rank,
                 device="cuda", all_gather=None):
        from . import jolt as J
        self.J = J
        self.sp = plan(n_layers, layers_per_group, world, rank)
        self.opts = replace(opts, unit_offset=self.sp.u0)
        n_local_layers = len(self.sp.layers)
        self.comp = J.Compressor(n_local_layers, n_heads, n_tokens, head_dim, layers_per_group, dtype, self.opts,
                                 device)
        self.bytes_row = J.choice_bytes(self.comp.shape, self.opts)
        self.all_gather = all_gather

    def local_tables(self, K_local, V_local, seed: int = 0):
        """Factors, stored core and distortion rows of this rank's units (no collective)."""
        import torch
        U, W = self.comp.factor(K_local, V_local, seed)
        Us, Ws = U.to(torch.bfloat16), W.to(torch.bfloat16)
        core, table = self.comp.table(K_local, V_local, Us, Ws, seed)
        return dict(Us=Us, Ws=Ws, core=core, table=table, seed=seed)

    def encode(self, K_local, V_local, state, full_table, choice):
        """This rank's blob for the allocation of all units (choice: every unit's choice)."""
        mine = slice(self.sp.u0, self.sp.u0 + self.sp.n_local_units)
        return self.comp.encode(K_local, V_local, state["Us"], state["Ws"], state["core"], choice[mine],
                                full_table[mine], state["seed"])

    def compress(self, K_local, V_local, budget: int, seed: int = 0):
        """Compress this rank's layers (K_local, V_local: [layers of this rank, H, T, D]) under the
        global budget.  Returns (blob, choices of all units, lambda); every rank returns the
        same choices and lambda.  Collective: every rank calls it with the same budget."""
        J = self.J

        def alloc(D, B, avail):
            ch, lam, st = J.allocate(D, B, avail)
            return ch, float(lam.item()), int(st.item())

        state = self.local_tables(K_local, V_local, seed)
        full, choice, lam, status = allocate_shared(state["table"], self.bytes_row, budget, self.sp, alloc,
                                                    self.all_gather)
        if status != 0:
            raise J.JoltError(5, "budget below the headers and every unit's fewest-bytes choice")
        return self.encode(K_local, V_local, state, full, choice), choice, lam
