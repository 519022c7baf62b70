"""Head sharding across ranks: the partition, the all-gather of O (gloo ranks on CPU, world sizes
2 and 3), the pairing of each rank's heads with their own routes (against the oracle), and on one
GPU the sharded compute of a two-rank plan, run rank by rank (against the single call and the
oracle) and as two processes whose device outputs are gathered (against the oracle)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_spatio_flash_b200 import shard
from block_sparse_spatio_flash_b200 import synthetic as syn


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# ------------------------------------------------------------------ the partition (host logic)
@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 12])
@pytest.mark.parametrize("costs", [[5] * 10, [9, 1, 9, 1, 9, 1, 9, 1, 9, 1], [3, 8, 2, 7, 7, 1, 0, 4], [1]])
def test_plan_covers_every_head_once_and_balances(costs, world):
    p = shard.plan_heads(costs, world)
    assert p.heads == len(costs) and p.world == world
    seen = sorted(h for hs in p.local for h in hs)
    assert seen == list(range(len(costs)))
    for r, hs in enumerate(p.local):
        assert list(hs) == sorted(hs)
        assert all(p.owner[h] == r for h in hs)
        assert p.load[r] == sum(costs[h] for h in hs)
    # longest-processing-time-first bound: max load <= mean load + largest single cost
    assert max(p.load) <= sum(costs) / world + max(costs) + 1e-9
    assert shard.plan_heads(costs, world) == p  # deterministic


def test_plan_equal_costs_split_evenly_and_brute_force_optimum_small():
    p = shard.plan_heads([4] * 10, 4)
    assert sorted(len(hs) for hs in p.local) == [2, 2, 3, 3]
    # on small cases LPT is optimal or within its 4/3 bound of the brute-force optimum
    import itertools
    costs = [7, 5, 4, 4, 3, 3, 2]
    best = min(max(sum(c for c, a in zip(costs, asg) if a == r) for r in range(3))
               for asg in itertools.product(range(3), repeat=len(costs)))
    assert max(shard.plan_heads(costs, 3).load) <= best * 4 / 3


def test_plan_errors_and_costs_from_summaries():
    with pytest.raises(ValueError):
        shard.plan_heads([1, 2], 0)
    with pytest.raises(ValueError):
        shard.plan_heads([1, -2], 2)

    class Summ:
        def __init__(self, n):
            self.pair_half_tiles = n
    assert shard.head_costs([0, 1, 1, 0], [Summ(10), Summ(7)]) == [10, 7, 7, 10]
    with pytest.raises(ValueError):
        shard.head_costs([1], [Summ(1), None])
    p = shard.plan_heads([10, 7, 7, 10], 2)
    assert shard.local_routes(p, 0, [0, 1, 1, 0]) == [[0, 1, 1, 0][h] for h in p.local[0]]


def test_local_heads_and_assemble_single_process():
    x = torch.arange(6 * 3 * 2, dtype=torch.float32).view(6, 3, 2)
    p = shard.plan_heads([1, 5, 2, 4, 3, 3], 3)
    blocks = [shard.local_heads(x, p, r) for r in range(3)]
    for r in range(3):
        for i, h in enumerate(p.local[r]):
            assert torch.equal(blocks[r][i], x[h])
    out = shard.assemble(blocks, p, torch.empty_like(x))
    assert torch.equal(out, x)
    assert torch.equal(shard.gather_heads(x.clone(), shard.plan_heads([1] * 6, 1)), x)


# ------------------------------------------------------------------ all-gather over gloo ranks
def _gather_worker(rank, world, port, costs, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(1234)
        full = torch.randn(len(costs), 5, 4, generator=g).to(torch.bfloat16)  # same on every rank
        p = shard.plan_heads(costs, world)
        mine = shard.local_heads(full, p, rank)
        got = shard.gather_heads(mine, p)
        out[rank] = bool(torch.equal(got, full))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,costs", [(2, [5, 5, 5, 5, 5, 5, 5, 5, 5, 5]), (2, [9, 1, 1, 1, 1]),
                                         (3, [3, 8, 2, 7, 7, 1, 0, 4]), (3, [1, 1])])
def test_gather_heads_gloo(world, costs):
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_gather_worker, args=(world, port, costs, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {r: True for r in range(world)}


# ------------------------------------------------------------------ each head keeps its own route
def _oracle_worker(rank, world, port, out):
    import numpy as np
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = syn.TINY.replace(routes=(0, 1, 1, 0, 1))
        q, k, v = syn.make_qkv(w)
        rows = np.arange(0, w.tokens, 37, dtype=np.int64)
        costs = [3 if r == 0 else 2 for r in w.routes]
        p = shard.plan_heads(costs, world)
        lr = shard.local_routes(p, rank, w.routes)
        ql, kl, vl = (shard.local_heads(x, p, rank) for x in (q, k, v))
        res = torch.zeros(max(p.max_local, 1), len(rows), w.d, dtype=torch.float64)
        for i, route in enumerate(lr):
            o, _ = oracle.attention_rows(ql[i], kl[i], vl[i], rows, route=route, layout=w.layout, T=w.frames,
                                         S=w.frame_size, frame_window=w.frame_window, band=w.spatial_band,
                                         F0=w.sink_frames)
            res[i] = torch.from_numpy(o)
        got = shard.gather_heads(res[: len(lr)], p)
        ok = True
        for h in range(w.heads):
            o, _ = oracle.attention_rows(q[h], k[h], v[h], rows, route=w.routes[h], layout=w.layout, T=w.frames,
                                         S=w.frame_size, frame_window=w.frame_window, band=w.spatial_band,
                                         F0=w.sink_frames)
            ok = ok and torch.equal(got[h], torch.from_numpy(o))
        out[rank] = ok
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharded_heads_keep_their_routes_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_oracle_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: True, 1: True}


# ------------------------------------------------------------------ GPU: a two-rank plan, rank by rank
@pytest.mark.gpu
def test_sharded_compute_matches_single_call_gpu():
    from block_sparse_spatio_flash_b200 import svg as S
    from tests import gpu_path as gp
    dev = torch.device("cuda")
    w = syn.Workload("medium_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 1, 0, 1), d=128, frame_window=1,
                     spatial_band=20)
    g, m, t = gp.geom_mask_tile(w)
    routes = list(w.routes)
    q, k, v = (x.to(dev) for x in syn.make_qkv(w, seed_offset=17))
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for a, b in ((q, qp), (k, kp), (v, vp)):
        S.svg_permute(a, b, routes, g, m)
    maps = gp.build_maps(w, g, m, t, routes)
    summ = [S.svg_tilemap_summary(x) if x is not None else None for x in maps]
    sc = S.alloc_scratch(dev)
    o_full = torch.empty_like(qp)
    S.svg_attention_fwd(qp, kp, vp, o_full, routes, maps[0], maps[1], g, m, t, scratch=sc)
    p = shard.plan_heads(shard.head_costs(routes, summ), 2)
    assert all(p.local)
    blocks = []
    for r in range(2):
        ql, kl, vl = (shard.local_heads(x, p, r) for x in (qp, kp, vp))
        ol = torch.empty_like(ql)
        shard.attention_fwd_local(ql, kl, vl, ol, p, r, routes, maps[0], maps[1], g, m, t, scratch=sc)
        blocks.append(ol)
    torch.cuda.synchronize()
    assert S.svg_read_status(sc) == 0
    got = shard.assemble(blocks, p, torch.empty_like(o_full))
    assert torch.equal(got, o_full)  # same kernel, same rows: bitwise
    # and the sharded result against the oracle, every row of every head (original order)
    o_orig = torch.empty_like(got)
    S.svg_permute(got, o_orig, routes, g, m, inverse=True)
    torch.cuda.synchronize()
    q0, k0, v0 = syn.make_qkv(w, seed_offset=17)
    gp.compare_rows(w, q0, k0, v0, o_orig.cpu(), None)


# ------------------------------------------------------------------ GPU: two ranks, device outputs gathered
GPU_SHARD_W = syn.Workload("shard_gpu_1200", frames=5, grid_h=12, grid_w=20, routes=(1, 0, 1, 1, 0), d=128,
                           frame_window=1, spatial_band=20)


def _gpu_rank_worker(rank, world, port, out):
    """One rank of a two-process group on the one GPU here: its heads' attention on the device, O back
    to the original order on the device, then the all-gather of O (gloo, host copies of the device
    blocks). The ranks' kernels never wait on each other."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_spatio_flash_b200 import svg as S
        from tests import gpu_path as gp
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        w = GPU_SHARD_W
        routes = list(w.routes)
        g, m, t = gp.geom_mask_tile(w)
        maps = gp.build_maps(w, g, m, t, routes)
        summ = [S.svg_tilemap_summary(x) if x is not None else None for x in maps]
        p = shard.plan_heads(shard.head_costs(routes, summ), world)
        lr = shard.local_routes(p, rank, routes)
        q, k, v = syn.make_qkv(w, seed_offset=29)
        ql, kl, vl = (shard.local_heads(x, p, rank).to(dev) for x in (q, k, v))
        qp, kp, vp = (torch.empty_like(x) for x in (ql, kl, vl))
        for a, b in ((ql, qp), (kl, kp), (vl, vp)):
            S.svg_permute(a, b, lr, g, m)
        o = torch.empty_like(qp)
        sc = S.alloc_scratch(dev)
        shard.attention_fwd_local(qp, kp, vp, o, p, rank, routes, maps[0], maps[1], g, m, t, scratch=sc)
        o_orig = torch.empty_like(o)
        S.svg_permute(o, o_orig, lr, g, m, inverse=True)
        torch.cuda.synchronize()
        status = S.svg_read_status(sc)
        full = shard.gather_heads(o_orig.cpu(), p)
        ok = status == 0 and tuple(full.shape) == (w.heads, w.tokens, w.d)
        if ok and rank == 0:
            gp.compare_rows(w, q, k, v, full, None)
        out[rank] = bool(ok)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_ranks_gather_device_outputs_gpu():
    from block_sparse_spatio_flash_b200 import build
    build.build()
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_gpu_rank_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: True, 1: True}
