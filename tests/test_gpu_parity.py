"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tile maps, retained counts and permutations are compared bit for bit; attention outputs
within relative L2 <= 1e-2 and max-abs <= 2e-2 per head (LSE within 5e-3), on every row for
small problems and on seeded sampled rows (plus the ragged tail) for the pages' sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_flash_b200 import synthetic as syn
from tests import gpu_path as gp
from tests.test_oracle_pins import closed_form_spatial, closed_form_temporal

pytestmark = pytest.mark.gpu

MEDIUM = syn.Workload("medium_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 0, 1), d=128,
                      frame_window=1, spatial_band=20, bq=128, bk=128)


@pytest.fixture(scope="module")
def S():
    from block_sparse_spatio_flash_b200 import build
    build.build()
    return gp.svg()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def expected_group_entries(cls, N, bq, bk, G):
    """Execution lists derived from the class map for groups of G 128-row blocks (G = 2: the pairs
    of the kernel's 256-row items). Block flag: 0 skip, 1 full, 2 masked, 3 full but ragged key
    tile; block i of a group sits at bit 32 - 2G + 2i; per group, the entries in which block i is
    active."""
    nq, nk = cls.shape
    rows = 128 * G
    ngroups = -(-N // rows)
    ragged = np.zeros(nk, dtype=bool)
    if N % bk:
        ragged[-1] = True
    ents, cnts = [], []
    for p in range(ngroups):
        flags = []
        for i in range(G):
            r0 = rows * p + 128 * i
            if r0 >= N:
                flags.append(np.zeros(nk, dtype=np.uint32))
                continue
            r1 = min(N, r0 + 128)
            cs = cls[r0 // bq: (r1 - 1) // bq + 1]
            anyk = (cs != 0).any(axis=0)
            allf = (cs == 1).all(axis=0)
            flags.append(np.where(~anyk, 0, np.where(allf, np.where(ragged, 3, 1), 2)).astype(np.uint32))
        phase = [np.zeros(nk, dtype=bool), np.zeros(nk, dtype=bool)]
        for i in range(G):
            phase[i % 2] |= flags[i] != 0
        act = phase[0] | phase[1]
        e = np.nonzero(act)[0].astype(np.uint32)
        for i in range(G):
            e = e | (flags[i][act] << np.uint32(32 - 2 * G + 2 * i))
        ents.append(e)
        cnts.append((int(phase[0].sum()), int(phase[1].sum())))
    return ents, cnts


def check_group_lists(A, summ, cls, N, bq, bk, G):
    key = "pair"
    ents, cnts = expected_group_entries(cls, N, bq, bk, G)
    ptr = u32(A[key + "_ptr"]).astype(np.int64)
    ent = u32(A[key + "_ent"])
    cnt = u32(A[key + "_cnt"]).reshape(-1, 2)
    for p in range(len(ents)):
        assert np.array_equal(ent[ptr[p]: ptr[p + 1]], ents[p]), (key, p)
        assert tuple(cnt[p]) == cnts[p], (key, p)
    work = cnt.sum(axis=1).astype(np.int64)
    order = u32(A[key + "_order"]).astype(np.int64)
    assert np.array_equal(order, np.lexsort((np.arange(len(work)), -work)))
    if G == 2:  # runs of equal work along the order, for the work-ordered scheduler
        ws = work[order]
        grp = u32(A["pair_grp"]).astype(np.int64).reshape(-1, 2)
        for p_ in range(len(ws)):
            same = np.nonzero(ws == ws[p_])[0]
            assert grp[p_, 0] == same[0] and grp[p_, 1] == same[-1] + 1, (p_, grp[p_], same[[0, -1]])
    tot_e = summ.pair_entries
    tot_w = summ.pair_half_tiles
    assert tot_e == sum(len(e) for e in ents) and tot_w == int(work.sum())


def check_tilemap(S, w, route, variant, bq, bk, qts=None):
    g, m, t = gp.geom_mask_tile(w, variant, bq, bk)
    ws = S.alloc_workspace(g, t)
    S.svg_build_tilemap(g, m, t, route, ws)
    summ = S.svg_tilemap_summary(ws)
    A = S.tilemap_arrays(ws, g, t)
    N = w.tokens
    cls = A["cls"].cpu().numpy()
    cnt = u32(A["cnt"]).reshape(A["nq"], A["nk"])
    full = qts is None
    qts = np.arange(A["nq"]) if qts is None else np.asarray(qts)
    ocnt, ocls = oracle.tile_counts(route, w.layout, w.frames, w.frame_size, w.frame_window, w.spatial_band,
                                    w.sink_frames, bq, bk, qts=qts)
    area = oracle.tile_areas(N, bq, bk)
    if variant == syn.MASK_ROUNDED:
        ocls = oracle.rounded_classes(ocnt, area[qts])
    assert np.array_equal(cnt[qts], ocnt)
    assert np.array_equal(cls[qts], ocls)
    # totals: exact count of the whole map equals the closed form of the mask
    if route == 0:
        closed = closed_form_spatial(w.frames, w.frame_size, w.frame_window, w.sink_frames)
    else:
        closed = closed_form_temporal(w.frames, w.frame_size, w.spatial_band, w.sink_frames)
    assert summ.retained_exact == closed == int(cnt.astype(np.int64).sum())
    assert summ.n_full == int((cls == 1).sum()) and summ.n_boundary == int((cls == 2).sum())
    assert summ.n_empty == int((cls == 0).sum())
    assert summ.visited_area == int(area[cls != 0].sum())
    if variant == syn.MASK_ROUNDED:
        assert summ.retained_map == int(area[cls == 1].sum())
    else:
        assert summ.retained_map == summ.retained_exact
    # CSR of visited tiles
    row_ptr = u32(A["row_ptr"]).astype(np.int64)
    cols = u32(A["cols"])
    for qt in (qts if not full else range(A["nq"])):
        seg = cols[row_ptr[qt]: row_ptr[qt + 1]]
        kts = np.nonzero(cls[qt])[0]
        assert np.array_equal(seg & 0x3FFFFFFF, kts)
        assert np.array_equal(seg >> 30, cls[qt, kts])
    # execution lists and scheduler orders (derived from the map, which matched the oracle)
    check_group_lists(A, summ, cls, N, bq, bk, 2)
    return summ


TINY_MAPS = [(r, lay, var, bq, bk) for r in (0, 1) for lay in (0, 1) for var in (0, 1)
             for (bq, bk) in ((64, 64), (128, 64), (256, 128))]


@pytest.mark.parametrize("route,layout,variant,bq,bk", TINY_MAPS)
def test_tilemap_tiny(S, route, layout, variant, bq, bk):
    w = syn.TINY.replace(layout=layout)
    check_tilemap(S, w, route, variant, bq, bk)


@pytest.mark.parametrize("route,variant,bq,bk", [(0, 0, 128, 128), (1, 0, 128, 128), (1, 1, 64, 64),
                                                  (0, 1, 512, 128), (1, 0, 256, 64)])
def test_tilemap_medium_ragged(S, route, variant, bq, bk):
    w = syn.Workload("m2", frames=6, grid_h=13, grid_w=17, routes=(route,), d=128, frame_window=2,
                     spatial_band=9, sink_frames=1)
    check_tilemap(S, w, route, variant, bq, bk)
    check_tilemap(S, w.replace(sink_frames=2, layout=1), route, variant, bq, bk)


@pytest.mark.parametrize("route,variant,bq,bk", [(0, 0, 128, 128), (1, 0, 128, 128), (0, 1, 256, 64),
                                                  (1, 1, 512, 128)])
def test_tilemap_pages_shape(S, route, variant, bq, bk):
    w = syn.MIXED_75K
    nq = -(-w.tokens // bq)
    qts = sorted({0, 1, 2, 27, 28, 29, nq // 3, nq // 2, nq - 3, nq - 2, nq - 1})
    summ = check_tilemap(S, w, route, variant, bq, bk, qts=qts)
    assert summ.retained_exact == (1969920000 if route == 0 else 2220817200)


def test_tilemap_1440p_totals(S):
    w = syn.P1440
    for route in (0, 1):
        nq = -(-w.tokens // 128)
        check_tilemap(S, w, route, 0, 128, 128, qts=[0, 113, nq // 2, nq - 1])


# ------------------------------------------------------------------------------ permutation
@pytest.mark.parametrize("w", [syn.TINY, MEDIUM, syn.MIXED_75K, MEDIUM.replace(layout=1, sink_frames=2)],
                         ids=lambda w: f"{w.name}-L{w.layout}-F{w.sink_frames}")
def test_permute_matches_oracle(S, w):
    g, m, _ = gp.geom_mask_tile(w)
    x = torch.randn(w.heads, w.tokens, w.d, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    xd = x.cuda()
    y = torch.empty_like(xd)
    S.svg_permute(xd, y, w.routes, g, m)
    z = torch.empty_like(xd)
    S.svg_permute(y, z, w.routes, g, m, inverse=True)
    torch.cuda.synchronize()
    yc = y.cpu()
    for h, r in enumerate(w.routes):
        pi = oracle.perm_table(r, w.layout, w.frames, w.frame_size, w.sink_frames)
        exp = torch.empty_like(x[h])
        exp[torch.as_tensor(pi)] = x[h]
        assert torch.equal(yc[h].view(torch.int16), exp.view(torch.int16))
    assert torch.equal(z.cpu().view(torch.int16), x.view(torch.int16))


# ------------------------------------------------------------------------------ attention
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("variant", [0, 1])
def test_attention_tiny(S, mode, variant):
    w = syn.TINY
    q, k, v = syn.make_qkv(w)
    out, lse, st = gp.run_path(w, q, k, v, mode=mode, variant=variant)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, lse, variant=variant)


@pytest.mark.parametrize("bq,bk", [(128, 128), (256, 64), (64, 128), (512, 64)])
@pytest.mark.parametrize("variant", [0, 1])
def test_attention_medium_ragged(S, bq, bk, variant):
    w = MEDIUM
    q, k, v = syn.make_qkv(w, seed_offset=3)
    out, lse, st = gp.run_path(w, q, k, v, variant=variant, bq=bq, bk=bk)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, lse, variant=variant, bq=bq, bk=bk)


@pytest.mark.parametrize("d,bk", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_dense_matches_oracle(S, d, bk):
    w = MEDIUM.replace(d=d, bk=bk)
    q, k, v = syn.make_qkv(w, seed_offset=5)
    out, lse, st = gp.run_path(w, q, k, v, dense=True, bk=bk)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, lse, all_kept=True)


EDGE = [
    syn.Workload("one_token", frames=1, grid_h=1, grid_w=1, routes=(0,), d=64, frame_window=0, spatial_band=0),
    syn.Workload("one_frame_ragged", frames=1, grid_h=7, grid_w=11, routes=(0, 1), d=128, frame_window=0,
                 spatial_band=3),
    syn.Workload("no_sink", frames=4, grid_h=6, grid_w=9, routes=(0, 1), d=128, frame_window=1, spatial_band=4,
                 sink_frames=0),
    syn.Workload("zero_window", frames=5, grid_h=6, grid_w=9, routes=(0, 1), d=64, frame_window=0,
                 spatial_band=0, bq=64, bk=64),
    syn.Workload("full_space_major", frames=6, grid_h=8, grid_w=10, routes=(1, 0, 1), d=128, frame_window=1,
                 spatial_band=5, layout=1),
    syn.Workload("two_sink_frames", frames=7, grid_h=5, grid_w=9, routes=(1, 0), d=128, frame_window=1,
                 spatial_band=3, sink_frames=2, bq=256, bk=64),
    syn.Workload("window_covers_all", frames=3, grid_h=9, grid_w=13, routes=(0,), d=128, frame_window=5,
                 spatial_band=0),
]


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
@pytest.mark.parametrize("variant", [0, 1])
def test_attention_edge_cases(S, w, variant):
    q, k, v = syn.make_qkv(w, seed_offset=11)
    for mode in (0, 1):
        out, lse, st = gp.run_path(w, q, k, v, mode=mode, variant=variant)
        assert st == 0
        gp.compare_rows(w, q, k, v, out, lse, variant=variant)


def test_rounded_row_without_keys_gives_zero(S):
    # band 0 over a wide frame: most temporal tiles are far below half full, so rounding
    # drops every tile of some rows; those rows must come out as O = 0, LSE = -inf.
    w = syn.Workload("sparse_rounded", frames=3, grid_h=16, grid_w=32, routes=(1,), d=64, frame_window=0,
                     spatial_band=0, sink_frames=0, variant=1, bq=128, bk=128)
    q, k, v = syn.make_qkv(w, seed_offset=2)
    out, lse, st = gp.run_path(w, q, k, v)
    assert st == 0
    stats = gp.compare_rows(w, q, k, v, out, lse, variant=1)
    assert not torch.isfinite(lse).all()  # some rows really had no key
    assert stats


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("bk", [64, 128])
def test_attention_growing_maxima(S, dense, bk):
    """Keys planted at random positions with scores up to ~9x the others: a row's running maximum
    jumps past the rescale threshold in the middle of the row, which exercises the redo of a tile
    whose exponentials were taken against the old maximum, and the O correction."""
    w = MEDIUM.replace(bk=bk)
    q, k, v = syn.make_qkv(w, seed_offset=13)
    k = k.float()
    g = torch.Generator().manual_seed(77)
    for h in range(w.heads):
        idx = torch.randperm(w.tokens, generator=g)[:24]
        k[h, idx] *= torch.linspace(2.0, 9.0, 24)[:, None]
    k = k.to(torch.bfloat16)
    out, lse, st = gp.run_path(w, q, k, v, dense=dense, bk=bk)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, lse, all_kept=dense)


def test_naive_equals_split_up_to_rounding(S):
    w = MEDIUM
    q, k, v = syn.make_qkv(w, seed_offset=7)
    a, la, _ = gp.run_path(w, q, k, v, mode=0)
    b, lb, _ = gp.run_path(w, q, k, v, mode=1)
    diff = (a.float() - b.float()).abs().max().item()
    assert diff <= 4e-3 and torch.allclose(la, lb, atol=1e-4, rtol=0)


# --- the pages' sizes: sampled rows (seeded) plus every row of the ragged last tile
# Oracle rows of the exact masks are shared between the tile shapes of one workload (the exact
# mask's result does not depend on the tiles); rounded masks are keyed by their tile shape.
_ORACLE_MEMO = {}


def _pages(w, rows=512, variant=None, bq=None, bk=None, mode=0):
    q, k, v = syn.make_qkv(w)
    out, lse, st = gp.run_path(w, q, k, v, variant=variant, bq=bq, bk=bk, mode=mode)
    assert st == 0

    def rows_of(h):
        r = syn.sample_rows(w.replace(sample_rows=rows), h)
        return np.unique(np.concatenate([r.numpy(), gp.tail_rows(w, h, 96)]))

    var = w.variant if variant is None else variant
    key = (w.name, "exact") if var == syn.MASK_EXACT else (w.name, "rounded", bq or w.bq, bk or w.bk)
    stats = gp.compare_rows(w, q, k, v, out, lse, rows_per_head=rows_of, variant=variant, bq=bq, bk=bk,
                            cache=_ORACLE_MEMO, cache_key=key)
    assert all(s["rows"] >= min(rows, w.tokens) for s in stats)
    return stats


def test_attention_pages_spatial(S):
    _pages(syn.SPATIAL_75K, rows=2048)


def test_attention_pages_temporal(S):
    _pages(syn.TEMPORAL_75K, rows=2048)


@pytest.mark.parametrize("bq,bk", syn.TILE_SWEEP)
@pytest.mark.parametrize("variant", [0, 1])
def test_attention_pages_mixed_sweep(S, bq, bk, variant):
    """The tile sweep of the mixed workload: 2,048 seeded rows per head for the 128 x 128 tiles of both
    masks, 512 per head for the other shapes (plus the ragged tail)."""
    _pages(syn.MIXED_75K, rows=2048 if (bq, bk) == (128, 128) else 512, variant=variant, bq=bq, bk=bk)


def test_attention_pages_mixed_naive(S):
    _pages(syn.MIXED_75K, rows=512, mode=1)


def test_attention_1440p(S):
    """302,400 tokens, 5 spatial + 5 temporal heads: 2,048 seeded rows per head plus the tail."""
    _pages(syn.P1440, rows=2048)


def test_dense_pages_shape(S):
    """The dense baseline at the pages' 75,600 tokens (2 heads, d = 128, 128-key tiles) against the
    oracle's all-kept attention on 2,048 seeded rows per head plus the tail."""
    w = syn.SPATIAL_75K.replace(routes=(0, 0))
    q, k, v = syn.make_qkv(w, seed_offset=7)
    out, lse, st = gp.run_path(w, q, k, v, dense=True, bk=128)
    assert st == 0

    def rows_of(h):
        r = syn.sample_rows(w.replace(sample_rows=2048), h)
        return np.unique(np.concatenate([r.numpy(), np.arange(w.tokens - 96, w.tokens)]))

    gp.compare_rows(w, q, k, v, out, lse, rows_per_head=rows_of, all_kept=True)


# ----------------------------------------------------------------------------- head routing
def _route_case(S, w, q, k, v, rows):
    g, m, _ = gp.geom_mask_tile(w)
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rd = torch.as_tensor(np.asarray(rows), dtype=torch.int32, device=dev)
    route = torch.full((w.heads,), 255, dtype=torch.uint8, device=dev)
    err = torch.full((w.heads, 2), -1.0, dtype=torch.float32, device=dev)
    work = torch.empty(S.svg_route_work_bytes(w.heads, w.tokens, w.d, len(rows)), dtype=torch.uint8, device=dev)
    S.svg_route_heads(qd, kd, vd, g, m, rd, route, err, work=work)
    torch.cuda.synchronize()
    assert S.svg_read_status(work) == 0
    valid = [r for r in np.asarray(rows).tolist() if 0 <= r < w.tokens]
    want_err, want_route = [], []
    for h in range(w.heads):
        es, et, ed = oracle.route_errors(q[h], k[h], v[h], valid, T=w.frames, S=w.frame_size,
                                         frame_window=w.frame_window, band=w.spatial_band, F0=w.sink_frames)
        want_err.append((es / ed, et / ed))
        want_route.append(0 if es <= et else 1)
    return route.cpu().numpy(), err.cpu().numpy().astype(np.float64), np.array(want_route), np.array(want_err)


def _check_routes(got_r, got_e, want_r, want_e):
    # fp32 accumulation against fp64: relative errors within 1e-3 of their own size
    assert np.allclose(got_e, want_e, rtol=2e-3, atol=1e-6), (got_e, want_e)
    for h in range(len(want_r)):
        es, et = want_e[h]
        if abs(es - et) > 1e-2 * max(es, et):
            assert got_r[h] == want_r[h], (h, got_r, want_r)
        else:  # a near tie may go either way; the decision must match the device's own errors
            assert got_r[h] == (0 if got_e[h][0] <= got_e[h][1] else 1)


@pytest.mark.parametrize("d", [64, 128])
def test_route_planted_structure(S, d):
    w = syn.Workload("route_medium", frames=6, grid_h=8, grid_w=12, routes=(0, 1, 1, 0, 1, 0), d=d,
                     frame_window=1, spatial_band=2)
    kinds = list(w.routes)
    q, k, v = syn.make_routed_qkv(w, kinds, seed_offset=d)
    rows = np.arange(0, w.tokens, 3)  # 192 rows: a ragged last block of sampled rows
    got_r, got_e, want_r, want_e = _route_case(S, w, q, k, v, rows)
    _check_routes(got_r, got_e, want_r, want_e)
    assert list(got_r) == kinds == list(want_r)


def test_route_random_heads_and_rows_outside(S):
    """Unstructured heads (decisions follow the oracle's errors) and sampled rows that fall outside
    the sequence, which contribute nothing."""
    w = MEDIUM
    q, k, v = syn.make_qkv(w, seed_offset=11)
    rows = np.concatenate([np.arange(0, w.tokens, 13), [-1, w.tokens, w.tokens + 5]])
    got_r, got_e, want_r, want_e = _route_case(S, w, q, k, v, rows)
    _check_routes(got_r, got_e, want_r, want_e)


def test_route_pages_shape(S):
    """Routing at 75,600 tokens with 64 sampled rows per head, planted spatial and temporal heads."""
    w = syn.MIXED_75K.replace(routes=(0, 1, 0, 1))
    kinds = list(w.routes)
    q, k, v = syn.make_routed_qkv(w, kinds, strength=1.0, seed_offset=3)
    rows = syn.sample_rows(w.replace(sample_rows=64), 0).numpy()
    got_r, got_e, want_r, want_e = _route_case(S, w, q, k, v, rows)
    _check_routes(got_r, got_e, want_r, want_e)
    assert list(got_r) == kinds


def test_route_many_rows_several_row_blocks(S):
    """300 sampled rows per head: three 128-row blocks of the tensor-core kernel, the last ragged."""
    w = syn.Workload("route_rows", frames=6, grid_h=10, grid_w=16, routes=(0, 1), d=128, frame_window=1,
                     spatial_band=12)
    q, k, v = syn.make_routed_qkv(w, list(w.routes), strength=1.2, seed_offset=5)
    rows = np.sort(np.random.default_rng(3).choice(w.tokens, 300, replace=False))
    got_r, got_e, want_r, want_e = _route_case(S, w, q, k, v, rows)
    _check_routes(got_r, got_e, want_r, want_e)
    assert list(got_r) == list(w.routes)


@pytest.mark.parametrize("d", [64, 128])
def test_route_several_key_chunks(S, d):
    """4,620 keys: three key chunks of 1,600 (the last ragged), 100 sampled rows (a ragged row block)."""
    w = syn.Workload("route_chunks", frames=7, grid_h=20, grid_w=33, routes=(1, 0, 1), d=d,
                     frame_window=1, spatial_band=40)
    q, k, v = syn.make_routed_qkv(w, list(w.routes), strength=1.2, seed_offset=9)
    rows = np.sort(np.random.default_rng(5).choice(w.tokens, 100, replace=False))
    got_r, got_e, want_r, want_e = _route_case(S, w, q, k, v, rows)
    _check_routes(got_r, got_e, want_r, want_e)
    assert list(got_r) == list(w.routes)


# ----------------------------------------------------------------------------- host-buffer entry
@pytest.mark.parametrize("chunk", [1, 3, 4, 9])
@pytest.mark.parametrize("routes", [(0, 1, 0, 1), (0, 0, 0, 0), (1, 1, 0, 1), (0, 1, 1, 0, 0, 1, 0)])
def test_host_entry_matches_device_path(S, chunk, routes):
    """svg_attention_fwd_host (pinned host buffers, chunked pipeline) gives exactly the bytes of
    the device-buffer path, and so the oracle's values."""
    w = MEDIUM.replace(routes=routes)
    q, k, v = syn.make_qkv(w, seed_offset=17)
    want, lse, st = gp.run_path(w, q, k, v)
    assert st == 0
    g, m, t = gp.geom_mask_tile(w)
    maps = gp.build_maps(w, g, m, t, list(routes))
    qh, kh, vh = (x.contiguous().pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    buf = torch.empty(S.svg_attention_host_buffer_bytes(w.tokens, w.d, min(chunk, w.heads)), dtype=torch.uint8,
                      device="cuda")
    S.svg_attention_fwd_host(qh, kh, vh, oh, list(routes), maps[0], maps[1], g, m, t, buf, chunk_heads=chunk)
    assert torch.equal(oh.view(torch.int16), want.view(torch.int16))
    gp.compare_rows(w, q, k, v, oh, None)


# ----------------------------------------------------------------------------- fused token order
FUSED_CASES = [
    (syn.TINY, {}),
    (MEDIUM, {}),
    (MEDIUM, {"bq": 256, "bk": 64}),
    (MEDIUM.replace(variant=1), {}),
    (syn.Workload("fused_space_major", frames=6, grid_h=8, grid_w=10, routes=(1, 0, 1), d=128, frame_window=1,
                  spatial_band=5, layout=1), {}),
    (syn.Workload("fused_two_sinks", frames=7, grid_h=5, grid_w=9, routes=(1, 0), d=128, frame_window=1,
                  spatial_band=3, sink_frames=2, bq=256, bk=64), {}),
    (syn.Workload("fused_d64_ragged", frames=5, grid_h=6, grid_w=9, routes=(1, 1, 0), d=64, frame_window=0,
                  spatial_band=2, bq=64, bk=64), {}),
    # runs of one patch's frames longer than a tile (256 rows: boxes never fit, every group gathered),
    # longer than a box may be (259 rows: the box maps are not built), and of a single frame
    (syn.Workload("fused_run_256", frames=257, grid_h=2, grid_w=3, routes=(1, 0), d=128, frame_window=2,
                  spatial_band=1), {}),
    (syn.Workload("fused_run_259", frames=260, grid_h=2, grid_w=3, routes=(1,), d=128, frame_window=2,
                  spatial_band=1), {}),
    (syn.Workload("fused_run_1", frames=2, grid_h=16, grid_w=20, routes=(1, 0), d=128, frame_window=1,
                  spatial_band=7), {}),
]


@pytest.mark.parametrize("w,kw", FUSED_CASES, ids=lambda x: getattr(x, "name", str(x)))
@pytest.mark.parametrize("mode", [0, 1])
def test_fused_order_equals_permuted_path(S, w, kw, mode):
    """Q/K/V/O in original order with temporal rows gathered in-kernel: bitwise the same O (and
    LSE, mapped to original order) as permute + attention + inverse permute, and the oracle's."""
    q, k, v = syn.make_qkv(w, seed_offset=21)
    want, want_lse, st = gp.run_path(w, q, k, v, mode=mode, **kw)
    assert st == 0
    got, got_lse, st = gp.run_fused(w, q, k, v, mode=mode, **kw)
    assert st == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert torch.equal(got_lse, gp.lse_to_original(w, want_lse))
    gp.compare_rows(w, q, k, v, got, None, variant=w.variant, bq=kw.get("bq", w.bq), bk=kw.get("bk", w.bk))


def test_fused_order_pages_mixed(S):
    """75,600 tokens, 5 spatial + 5 temporal heads: fused equals the permuted path bit for bit."""
    w = syn.MIXED_75K
    q, k, v = syn.make_qkv(w)
    want, _, st = gp.run_path(w, q, k, v, lse=False)
    assert st == 0
    got, _, st = gp.run_fused(w, q, k, v, lse=False)
    assert st == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


# ----------------------------------------------------------------------------- scheduling order
def _run_ordered(S, w, qp, kp, vp, maps, g, m, t, order, mode=0):
    o = torch.empty_like(qp)
    ls = torch.empty(qp.shape[:2], dtype=torch.float32, device=qp.device)
    sc = S.alloc_scratch()
    n = torch.cuda.get_device_properties(0).multi_processor_count
    tr = torch.full((n + 3, 4), -1, dtype=torch.int64, device=qp.device)
    S.svg_attention_fwd_ex(qp, kp, vp, o, list(w.routes), maps[0], maps[1], g, m, t, mode=mode, scratch=sc, lse=ls,
                           order=order, cta_trace=tr)
    assert S.svg_read_status(sc) == 0
    return o, ls, tr.cpu()


@pytest.mark.parametrize("w,variant", [(MEDIUM, 0), (MEDIUM.replace(routes=(1, 1, 0, 1, 0, 0, 1)), 1),
                                       (syn.MIXED_75K, 0)], ids=["medium", "medium7_rounded", "mixed_75600"])
def test_work_order_gives_the_same_bytes_and_a_complete_trace(S, w, variant):
    """The work-ordered scheduler (longest processing time first over all heads) computes exactly the
    head-major order's bytes; the per-CTA trace accounts for every item and half-tile once."""
    g, m, t = gp.geom_mask_tile(w, variant)
    routes = list(w.routes)
    q, k, v = (x.cuda() for x in syn.make_qkv(w, seed_offset=71))
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for a, b in ((q, qp), (k, kp), (v, vp)):
        S.svg_permute(a, b, routes, g, m)
    maps = gp.build_maps(w, g, m, t, routes)
    summ = {c: S.svg_tilemap_summary(maps[c]) for c in (0, 1) if maps[c] is not None}
    o0, l0, tr0 = _run_ordered(S, w, qp, kp, vp, maps, g, m, t, S.SVG_ORDER_HEAD_MAJOR)
    o1, l1, tr1 = _run_ordered(S, w, qp, kp, vp, maps, g, m, t, S.SVG_ORDER_WORK)
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(l0, l1)
    npairs = -(-w.tokens // 256)
    want_tiles = sum(summ[r].pair_half_tiles for r in routes)
    n = torch.cuda.get_device_properties(0).multi_processor_count
    for tr in (tr0, tr1):
        ran = tr[:n][tr[:n, 2] > 0]
        assert int(tr[:n, 2].sum()) == w.heads * npairs and int(tr[:n, 3].sum()) == want_tiles
        assert (ran[:, 1] >= ran[:, 0]).all() and (ran[:, 0] > 0).all()
        assert (tr[n:] == 0).all()  # entries past the grid are cleared and never written
    if w.tokens > 10000:  # and against the oracle on sampled rows
        out = torch.empty_like(o1)
        S.svg_permute(o1, out, routes, g, m, inverse=True)
        q0, k0, v0 = syn.make_qkv(w, seed_offset=71)
        gp.compare_rows(w.replace(sample_rows=128), q0, k0, v0, out.cpu(), None)


def test_ablation_ordering_naive_slower_than_split_and_rounded_without_boundary(S):
    """The pages' ablation ordering on spatial_75600: masking every visited tile (naive) is slower than
    the full / boundary split, and the tile-aligned (rounded) map has no boundary tile while the exact
    map has some."""
    w = syn.SPATIAL_75K
    dev = torch.device("cuda")
    g, m, t = gp.geom_mask_tile(w)
    routes = list(w.routes)
    q, k, v = (x.to(dev) for x in syn.make_qkv(w))
    maps = gp.build_maps(w, g, m, t, routes)
    o = torch.empty_like(q)
    sc = S.alloc_scratch()

    def ms(mode):
        for _ in range(2):
            S.svg_attention_fwd(q, k, v, o, routes, maps[0], maps[1], g, m, t, mode=mode, scratch=sc)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record()
        for _ in range(3):
            S.svg_attention_fwd(q, k, v, o, routes, maps[0], maps[1], g, m, t, mode=mode, scratch=sc)
        b_.record()
        torch.cuda.synchronize()
        return a_.elapsed_time(b_) / 3

    split, naive = ms(S.SVG_MODE_SPLIT), ms(S.SVG_MODE_NAIVE)
    assert S.svg_read_status(sc) == 0
    assert naive > 1.2 * split, (naive, split)
    exact = S.svg_tilemap_summary(maps[0])
    gr, mr, tr = gp.geom_mask_tile(w, variant=syn.MASK_ROUNDED)
    rounded = S.svg_tilemap_summary(gp.build_maps(w, gr, mr, tr, routes)[0])
    assert rounded.n_boundary == 0 < exact.n_boundary


def test_fused_order_1440p_equals_permuted_path_and_oracle(S):
    """302,400 tokens (21 frames, 20-frame runs as boxes), 5 spatial + 5 temporal heads: the fused order
    gives the permuted path's bytes, and the oracle's values on 256 seeded rows per head."""
    w = syn.P1440
    q, k, v = syn.make_qkv(w, seed_offset=91)
    want, _, st = gp.run_path(w, q, k, v, lse=False)
    assert st == 0
    got, _, st = gp.run_fused(w, q, k, v, lse=False)
    assert st == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    del want
    gp.compare_rows(w.replace(sample_rows=256), q, k, v, got, None)


# ----------------------------------------------------------------------------- limits
def test_max_heads_small_geometry(S):
    """4,096 heads (the ABI's limit) of a one-frame 8 x 8 geometry, alternating routes: the route bit
    set, the work counter and the permutation at their largest head index; sampled heads checked."""
    routes = tuple(h % 2 for h in range(4096))
    w = syn.Workload("max_heads", frames=2, grid_h=4, grid_w=8, routes=routes, d=64, frame_window=0,
                     spatial_band=3, bq=64, bk=64)
    q, k, v = syn.make_qkv(w, seed_offset=51)
    out, lse, st = gp.run_path(w, q, k, v)
    assert st == 0
    heads = [0, 1, 2047, 2048, 4094, 4095]
    for h in heads:
        rows = np.arange(w.tokens)
        ref, _ = gp.oracle_rows(w, q, k, v, h, rows)
        got = out[h].to(torch.float64).numpy()
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= gp.REL_L2_TOL, h


def test_smoke_entry_point(S):
    import __graft_entry__
    __graft_entry__.smoke()


# ----------------------------------------------------------------------------- e4m3 QK^T
@pytest.mark.parametrize("bq,bk", [(128, 128), (256, 64)])
@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_qk8_matches_oracle_on_quantised_inputs(S, bq, bk, variant, mode):
    """QK^T on the 8-bit path: the oracle sees the same e4m3 values (exact in bf16), so parity holds
    with the bf16 path's tolerance."""
    w = MEDIUM.replace(bq=bq, bk=bk, variant=variant)
    q, k, v = syn.make_qkv(w, seed_offset=61)
    q, k = gp.quantize_e4m3(q), gp.quantize_e4m3(k)
    out, st = gp.run_qk8(w, q, k, v, mode=mode)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, None, variant=variant, bq=bq, bk=bk)


def test_qk8_pages_temporal_and_growing_maxima(S):
    w = syn.TEMPORAL_75K.replace(sample_rows=256)
    q, k, v = syn.make_qkv(w)
    q, k = gp.quantize_e4m3(q), gp.quantize_e4m3(k)
    out, st = gp.run_qk8(w, q, k, v)
    assert st == 0
    gp.compare_rows(w, q, k, v, out, None)
    wm = MEDIUM
    q, k, v = syn.make_qkv(wm, seed_offset=13)
    k = k.float()
    g = torch.Generator().manual_seed(77)
    for h in range(wm.heads):
        idx = torch.randperm(wm.tokens, generator=g)[:24]
        k[h, idx] *= torch.linspace(2.0, 9.0, 24)[:, None]
    q, k = gp.quantize_e4m3(q), gp.quantize_e4m3(k.to(torch.bfloat16))
    out, st = gp.run_qk8(wm, q, k, v)
    assert st == 0
    gp.compare_rows(wm, q, k, v, out, None)
