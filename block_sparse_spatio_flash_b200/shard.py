"""Head-sharded attention over several GPUs (one process per GPU, torch.distributed).

Heads never exchange data during the forward pass (each head attends over its own K/V under its
own route's mask; "Sparse Attention Patterns" in "Google Speeds Up Video Diffusion on TPUs with
Optimized Sparse Attention"), so one call's heads can be split across ranks. Each rank then runs
the attention of its heads with no collective. The only exchange is optional: when one device needs
the whole output, `gather_heads` assembles O over the process group (an all-gather; NCCL over
NVLink on GPUs).

Balance: a head costs the visited half-tiles of its route's tile map (`pair_half_tiles` of the
tile-map summary), so spatial and temporal heads weigh what they compute. Heads go to ranks
longest-processing-time first: costliest head first, each to the least-loaded rank. The largest load
is then at most the mean load plus the largest single head cost.

Plumbing only: the attention itself is the library call of `svg.py`; this module moves head indices
and tensors.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import torch


@dataclass(frozen=True)
class HeadPlan:
    """owner[h] = rank of head h; local[r] = heads of rank r, ascending; load[r] = their summed cost."""
    heads: int
    world: int
    owner: tuple
    local: tuple
    load: tuple

    @property
    def max_local(self) -> int:
        return max((len(x) for x in self.local), default=0)


def plan_heads(costs: Sequence[int], world: int) -> HeadPlan:
    """Longest-processing-time-first assignment of heads (cost costs[h] >= 0) to `world` ranks.

    Deterministic: ties go to the lower head index first and to the lower rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = [int(c) for c in costs]
    if any(c < 0 for c in costs):
        raise ValueError("head costs must be non-negative")
    heads = len(costs)
    load = [0] * world
    assign = [[] for _ in range(world)]
    for h in sorted(range(heads), key=lambda h: (-costs[h], h)):
        r = min(range(world), key=lambda r: (load[r], len(assign[r]), r))
        assign[r].append(h)
        load[r] += costs[h]
    owner = [0] * heads
    for r, hs in enumerate(assign):
        for h in hs:
            owner[h] = r
    return HeadPlan(heads, world, tuple(owner), tuple(tuple(sorted(hs)) for hs in assign), tuple(load))


def head_costs(routes: Sequence[int], summaries) -> list:
    """Cost of each head: visited half-tiles of its route class. summaries[c] is the
    `svg_tilemap_summary` of class c's tile map (None for a class no head uses)."""
    out = []
    for r in routes:
        s = summaries[int(r)]
        if s is None:
            raise ValueError(f"no tile-map summary for route class {int(r)}")
        out.append(int(s.pair_half_tiles))
    return out


def local_routes(plan: HeadPlan, rank: int, routes: Sequence[int]) -> list:
    """Routes of rank `rank`'s heads, in its local head order."""
    return [int(routes[h]) for h in plan.local[rank]]


def local_heads(x: torch.Tensor, plan: HeadPlan, rank: int) -> torch.Tensor:
    """Rank `rank`'s heads of a [heads, ...] tensor that holds all heads, as a contiguous copy."""
    idx = torch.tensor(plan.local[rank], dtype=torch.long, device=x.device)
    return x.index_select(0, idx)


def attention_fwd_local(q, k, v, o, plan: HeadPlan, rank: int, routes: Sequence[int], ws_spatial, ws_temporal,
                        geom, mask, tile, **kw):
    """svg_attention_fwd on this rank's heads: q/k/v/o hold exactly plan.local[rank] heads (in that
    order); `routes` are the routes of ALL heads. A rank without heads does nothing."""
    from . import svg
    lr = local_routes(plan, rank, routes)
    if not lr:
        return o
    if q.shape[0] != len(lr):
        raise ValueError(f"rank {rank} holds {q.shape[0]} heads, the plan gives it {len(lr)}")
    return svg.svg_attention_fwd(q, k, v, o, lr, ws_spatial, ws_temporal, geom, mask, tile, **kw)


def assemble(blocks: Sequence[torch.Tensor], plan: HeadPlan, out: torch.Tensor) -> torch.Tensor:
    """out[h] = blocks[owner(h)][position of h in its rank's list]; blocks[r] has at least
    len(plan.local[r]) heads (padding beyond that is ignored)."""
    if len(blocks) != plan.world:
        raise ValueError("one block per rank")
    for r, hs in enumerate(plan.local):
        if not hs:
            continue
        idx = torch.tensor(hs, dtype=torch.long, device=out.device)
        out.index_copy_(0, idx, blocks[r][: len(hs)])
    return out


def gather_heads(o_local: torch.Tensor, plan: HeadPlan, out: Optional[torch.Tensor] = None, group=None):
    """All ranks: every rank's heads into one [heads, ...] tensor on every rank.

    Collective over `group` (every rank calls it, in the same order as its other collectives).
    Ranks hold different head counts, so each sends a block padded to the largest count."""
    import torch.distributed as dist
    shape = tuple(o_local.shape[1:])
    if out is None:
        out = torch.empty((plan.heads,) + shape, dtype=o_local.dtype, device=o_local.device)
    if plan.world == 1:
        return assemble([o_local], plan, out)
    n = plan.max_local
    send = o_local
    if o_local.shape[0] != n:
        send = torch.zeros((n,) + shape, dtype=o_local.dtype, device=o_local.device)
        send[: o_local.shape[0]].copy_(o_local)
    recv = [torch.empty_like(send) for _ in range(plan.world)]
    dist.all_gather(recv, send.contiguous(), group=group)
    return assemble(recv, plan, out)
