"""Seeded synthetic workloads shared by the CUDA path's tests, the bench and the oracle's callers.

This module holds only workload *descriptions* (shapes, head routes, mask constants,
tile shapes, seeds) and the random-number recipe that turns them into Q/K/V bytes. It
contains none of the attention arithmetic, imports neither the CUDA binding nor the
oracle, and can be imported on a machine with no GPU.

Workload recipe (all configs): Q, K, V are drawn independently as fp32 N(0, 1) with a
CPU ``torch.Generator`` seeded 0 (Q), 1 (K), 2 (V) plus ``seed_offset``, shaped
``[heads, tokens, d]`` in the ORIGINAL frame-major token order (token i = t*S + s with
S = grid_h*grid_w and s = y*grid_w + x), then rounded to bf16. Both sides read the same
bf16 bytes. The pages only ever benchmark synthetic BF16 inputs
("Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs", summary and
"Sources & evidence"), so no dataset stands behind these shapes.
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

import torch

ROUTE_SPATIAL = 0
ROUTE_TEMPORAL = 1

MASK_EXACT = 0
MASK_ROUNDED = 1

LAYOUT_SINK_PREFIX = 0
LAYOUT_FULL_SPACE_MAJOR = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    frames: int
    grid_h: int
    grid_w: int
    routes: Tuple[int, ...]          # one route per head
    d: int
    frame_window: int                # spatial heads: |t_q - t_k| <= frame_window
    spatial_band: int                # temporal heads: |s_q - s_k| <= spatial_band
    sink_frames: int = 1             # keys in frames [0, sink_frames) are always kept
    layout: int = LAYOUT_SINK_PREFIX  # token order of temporal heads
    variant: int = MASK_EXACT
    bq: int = 128
    bk: int = 128
    sample_rows: int = 0             # 0: every query row is checked against the oracle

    @property
    def tokens(self) -> int:
        return self.frames * self.grid_h * self.grid_w

    @property
    def frame_size(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def heads(self) -> int:
        return len(self.routes)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Mask constants the pages leave open are fixed here:
#  * spatial window k = 3 frames at the pages' shape, k = 1 on the tiny grid;
#  * temporal band b = 715 at 75,600 tokens and b = 2,863 at 302,400 tokens (the integer
#    bands whose kept share is closest to the ~38.87% the pages quote), b = 16 on the tiny grid;
#  * a one-frame key-side sink (frame 0), as the pages state both masks keep the first frame.
TINY = Workload("tiny_512", frames=4, grid_h=8, grid_w=16, routes=(ROUTE_SPATIAL, ROUTE_TEMPORAL),
                d=64, frame_window=1, spatial_band=16, bq=64, bk=64)
SPATIAL_75K = Workload("spatial_75600", frames=21, grid_h=45, grid_w=80, routes=(ROUTE_SPATIAL,) * 10,
                       d=128, frame_window=3, spatial_band=715, sample_rows=2048)
TEMPORAL_75K = Workload("temporal_75600", frames=21, grid_h=45, grid_w=80, routes=(ROUTE_TEMPORAL,) * 10,
                        d=128, frame_window=3, spatial_band=715, sample_rows=2048)
MIXED_75K = Workload("mixed_75600", frames=21, grid_h=45, grid_w=80,
                     routes=(ROUTE_SPATIAL,) * 5 + (ROUTE_TEMPORAL,) * 5,
                     d=128, frame_window=3, spatial_band=715, sample_rows=2048)
P1440 = Workload("p1440_302400", frames=21, grid_h=90, grid_w=160,
                 routes=(ROUTE_SPATIAL,) * 5 + (ROUTE_TEMPORAL,) * 5,
                 d=128, frame_window=3, spatial_band=2863, sample_rows=2048)

WORKLOADS = {w.name: w for w in (TINY, SPATIAL_75K, TEMPORAL_75K, MIXED_75K, P1440)}

# Tile-shape sweep of the mixed workload.
TILE_SWEEP: List[Tuple[int, int]] = [(bq, bk) for bq in (128, 256, 512) for bk in (64, 128)]


def make_qkv(w: Workload, seed_offset: int = 0, dtype=torch.bfloat16):
    """Return CPU tensors (q, k, v), each [heads, tokens, d] in original token order."""
    out = []
    for which in range(3):
        g = torch.Generator(device="cpu")
        g.manual_seed(which + seed_offset)
        x = torch.randn((w.heads, w.tokens, w.d), generator=g, dtype=torch.float32)
        out.append(x.to(dtype))
    return tuple(out)


def sample_rows(w: Workload, head: int, seed: int = 1234) -> torch.Tensor:
    """Seeded query rows (original token indices, sorted) checked for one head.

    Always includes the first and last rows of the sequence and the rows of the
    final, ragged query tile, so the tail is covered at every size."""
    n = w.tokens
    if w.sample_rows <= 0 or w.sample_rows >= n:
        return torch.arange(n, dtype=torch.int64)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 7919 * head)
    r = torch.randperm(n, generator=g)[: w.sample_rows]
    fixed = torch.tensor([0, 1, n // 2, n - 2, n - 1], dtype=torch.int64)
    tail = torch.arange(max(0, n - 96), n, dtype=torch.int64)
    return torch.unique(torch.cat([r, fixed, tail]))


def make_routed_qkv(w: Workload, kinds, strength: float = 1.5, seed_offset: int = 0, dtype=torch.bfloat16):
    """Q/K/V with planted head structure, original order, for routing checks.

    kinds[h] = ROUTE_SPATIAL: every frame has its own random direction, added (times `strength`)
    to the queries and keys of that frame, so a query's largest scores are within its frame.
    kinds[h] = ROUTE_TEMPORAL: every patch position has its own direction instead, so a query's
    largest scores are at its patch across frames. V is plain N(0, 1)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(100 + seed_offset)
    T, S, N, d = w.frames, w.frame_size, w.tokens, w.d
    q = torch.randn((w.heads, N, d), generator=g)
    k = torch.randn((w.heads, N, d), generator=g)
    v = torch.randn((w.heads, N, d), generator=g)
    tok = torch.arange(N)
    for h, kind in enumerate(kinds):
        if kind == ROUTE_SPATIAL:
            dirs = torch.randn((T, d), generator=g)
            idx = tok // S
        else:
            dirs = torch.randn((S, d), generator=g)
            idx = tok % S
        q[h] += strength * dirs[idx]
        k[h] += strength * dirs[idx]
    return q.to(dtype), k.to(dtype), v.to(dtype)
