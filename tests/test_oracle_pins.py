"""Pins for the fp64 oracle: every routine is checked against something other than itself.

* retained counts against closed forms counted per frame pair / per patch pair;
* tile classes against an interval derivation over frame or patch ranges, and against
  hand-derived class totals for the tiny grid;
* attention against special cases with a known answer (Q = 0 gives the mean of the kept
  values and LSE = ln #kept; V = 1 gives O = 1; an all-kept mask gives textbook softmax
  attention computed with numpy), and a numpy brute force with an explicit N x N mask;
* the token order against closed-form positions and the bijection property;
* the pages' kept share (~38.87% at 75,600 tokens) for the temporal band reading, and the pages'
  38.87% and 27.55% as the spatial mask's visited and boundary tile shares at TPU tile sizes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_spatio_flash_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers
def closed_form_spatial(T, S, k, F0):
    """Sum over query frames f of |{g : |f-g| <= k} U {g < F0}| frames, times S*S tokens."""
    total = 0
    for f in range(T):
        kept = {g for g in range(T) if abs(f - g) <= k} | set(range(min(F0, T)))
        total += len(kept)
    return total * S * S


def closed_form_temporal(T, S, b, F0):
    """Per query: (T-F0) * #{s' : |s-s'| <= b} band keys outside the sink + F0*S sink keys.
    Summed over s, #{(s,s') : |s-s'| <= b} = S(2b+1) - b(b+1) for b < S."""
    assert b < S
    band_pairs = S * (2 * b + 1) - b * (b + 1)
    return T * ((T - F0) * band_pairs + F0 * S * S)


def token_fs(T, S):
    i = np.arange(T * S)
    return i // S, i % S


def s_of_position(layout, route, T, S, F0, p):
    """Patch index of the token sitting at position p (layout definition, solved for s)."""
    p = np.asarray(p)
    if route == syn.ROUTE_SPATIAL:
        return p % S
    if layout == syn.LAYOUT_FULL_SPACE_MAJOR:
        return p // T
    return np.where(p < F0 * S, p % S, (p - F0 * S) // max(T - F0, 1))


def t_of_position(layout, route, T, S, F0, p):
    p = np.asarray(p)
    if route == syn.ROUTE_SPATIAL:
        return p // S
    if layout == syn.LAYOUT_FULL_SPACE_MAJOR:
        return p % T
    return np.where(p < F0 * S, p // S, F0 + (p - F0 * S) % max(T - F0, 1))


def interval_classes(route, layout, T, S, k, b, F0, bq, bk, qts=None):
    """Tile classes from frame / patch ranges instead of element-by-element tests.

    Spatial: keep depends only on the (query frame, key frame) pair, and every frame that
    a tile touches owns at least one of its rows/columns, so the tile is full iff every
    touched frame pair is kept and empty iff none is. Temporal: sink columns are always
    kept; for the others keep depends only on |s_q - s_k|, so the tile is full iff the
    largest patch distance is <= b and empty iff it has no sink column and the smallest
    patch distance is > b."""
    N = T * S
    nq, nk = -(-N // bq), -(-N // bk)
    qts = range(nq) if qts is None else qts
    out = np.zeros((len(qts), nk), dtype=np.uint8)
    for a, qt in enumerate(qts):
        rp = np.arange(qt * bq, min(N, (qt + 1) * bq))
        for kt in range(nk):
            cp = np.arange(kt * bk, min(N, (kt + 1) * bk))
            if route == syn.ROUTE_SPATIAL:
                fq = np.unique(t_of_position(layout, route, T, S, F0, rp))
                fk = np.unique(t_of_position(layout, route, T, S, F0, cp))
                kept = (np.abs(fq[:, None] - fk[None, :]) <= k) | (fk[None, :] < F0)
                out[a, kt] = 1 if kept.all() else (0 if not kept.any() else 2)
            else:
                sq = np.unique(s_of_position(layout, route, T, S, F0, rp))
                tk = t_of_position(layout, route, T, S, F0, cp)
                sk = np.unique(s_of_position(layout, route, T, S, F0, cp)[tk >= F0])
                has_sink = bool((tk < F0).any())
                if len(sk) == 0:
                    out[a, kt] = 1
                    continue
                maxd = max(sq.max() - sk.min(), sk.max() - sq.min())
                pos = np.searchsorted(sk, sq)
                lo = np.abs(sq - sk[np.clip(pos - 1, 0, len(sk) - 1)])
                hi = np.abs(sq - sk[np.clip(pos, 0, len(sk) - 1)])
                mind = min(lo.min(), hi.min())
                if maxd <= b:
                    out[a, kt] = 1
                elif mind > b and not has_sink:
                    out[a, kt] = 0
                else:
                    out[a, kt] = 2
    return out


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def f64(x):
    return x.to(torch.float64).numpy()


# ----------------------------------------------------------------------------- retained counts
@pytest.mark.parametrize("T,H,W,k,F0", [(4, 8, 16, 1, 1), (5, 3, 4, 0, 1), (7, 2, 5, 2, 2), (6, 3, 3, 9, 0)])
def test_retained_spatial_closed_form(T, H, W, k, F0):
    S = H * W
    assert oracle.retained_pairs(syn.ROUTE_SPATIAL, T, S, k, 0, F0) == closed_form_spatial(T, S, k, F0)


@pytest.mark.parametrize("T,H,W,b,F0", [(4, 8, 16, 16, 1), (5, 3, 4, 0, 1), (7, 2, 5, 3, 2), (3, 4, 4, 15, 0)])
def test_retained_temporal_closed_form(T, H, W, b, F0):
    S = H * W
    assert oracle.retained_pairs(syn.ROUTE_TEMPORAL, T, S, 0, b, F0) == closed_form_temporal(T, S, b, F0)


def test_retained_tiny_values():
    # 12 of 16 frame pairs kept (frames {0,1},{0,1,2},{0,1,2,3},{0,2,3}) x 128^2 tokens.
    assert oracle.retained_pairs(syn.ROUTE_SPATIAL, 4, 128, 1, 16, 1) == 12 * 128 * 128 == 196608
    assert oracle.retained_pairs(syn.ROUTE_TEMPORAL, 4, 128, 1, 16, 1) == 112960


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, val = line.split()
                vals[key] = float(val)
    return vals


def test_pages_shape_and_budget():
    """The pages' workload: 75,600 tokens; ~38.87% of query-key pairs kept.

    The temporal band reading b = 715 is the integer band whose exact kept share is closest
    to the printed 38.87%; the oracle's brute-force count must land there. The spatial mask
    as read (+-3 frames, frame-0 sink) keeps 152/441 of pairs, which does NOT reproduce the
    printed share; that mismatch is a reading recorded in the design notes, pinned here."""
    g = read_golden("pages_workload.txt")
    w = syn.TEMPORAL_75K
    T, S, N = w.frames, w.frame_size, w.tokens
    assert N == g["tokens"] and w.heads == g["heads"] and w.d == g["head_dim"]
    target = g["kept_pairs_percent"] / 100.0
    shares = {b: closed_form_temporal(T, S, b, 1) / N ** 2 for b in range(600, 800)}
    best = min(shares, key=lambda b: abs(shares[b] - target))
    assert best == w.spatial_band == 715
    got = oracle.retained_pairs(syn.ROUTE_TEMPORAL, T, S, 0, 715, 1)
    assert got == 2220817200
    assert abs(got / N ** 2 - target) < 2e-4
    sp = oracle.retained_pairs(syn.ROUTE_SPATIAL, T, S, 3, 0, 1)
    assert sp == 152 * S * S == 1969920000
    # 1440p: four times the tokens of 720p at the same frame count
    assert syn.P1440.tokens == g["resolution_scale_tokens"] * N


def test_pages_tile_shares_at_tpu_scale_tiles():
    """The pages' 38.87% and 27.55% are tile-level shares of the spatial mask at TPU tile sizes.

    The pages give no tile shape. Classified element by element by the oracle at 75,600 tokens
    (+-3 frames, frame-0 sink), the share of (query tile, key tile) pairs that are visited at
    2048 x 2048 tiles is 38.86% (the pages print 38.87% as the kept share), and the share of
    visited tiles that are boundary tiles at 2304 x 2048 is 27.56% (the pages print 27.55%);
    at B200's 128 x 128 tiles it is 1.7%. No single shape gives both printed values, so the
    reading is recorded and pinned here, not used to choose the kernel's tiles; the pages'
    2.22% after tile-aligned traversal stays unpinned (the rounded map's ragged-tail tiles are
    3.2-3.7% of its visited tiles at these shapes)."""
    g = read_golden("pages_workload.txt")
    w = syn.SPATIAL_75K
    T, S = w.frames, w.frame_size

    def shares(bq, bk):
        _, cls = oracle.tile_counts(syn.ROUTE_SPATIAL, syn.LAYOUT_SINK_PREFIX, T, S, w.frame_window, 0,
                                    w.sink_frames, bq, bk)
        full, bnd = int((cls == 1).sum()), int((cls == 2).sum())
        return (full + bnd) / cls.size, bnd / (full + bnd)

    visited, _ = shares(2048, 2048)
    assert abs(visited - g["kept_pairs_percent"] / 100.0) < 2e-4
    _, boundary = shares(2304, 2048)
    assert abs(boundary - g["boundary_tiles_percent"] / 100.0) < 2e-4
    assert g["boundary_tiles_aligned_percent"] < g["boundary_tiles_percent"]


# ----------------------------------------------------------------------------- token order
@pytest.mark.parametrize("layout", [syn.LAYOUT_SINK_PREFIX, syn.LAYOUT_FULL_SPACE_MAJOR])
@pytest.mark.parametrize("T,S,F0", [(4, 128, 1), (21, 30, 1), (5, 7, 2), (3, 4, 0)])
def test_permutation_bijection_and_corners(layout, T, S, F0):
    pi = oracle.perm_table(syn.ROUTE_TEMPORAL, layout, T, S, F0)
    inv = oracle.inverse_table(syn.ROUTE_TEMPORAL, layout, T, S, F0)
    N = T * S
    assert np.array_equal(np.sort(pi), np.arange(N))
    assert np.array_equal(inv[pi], np.arange(N))
    pos = lambda t, s: oracle.position(syn.ROUTE_TEMPORAL, layout, T, S, F0, t, s)
    if layout == syn.LAYOUT_FULL_SPACE_MAJOR or F0 == 0:
        assert pos(0, 0) == 0 and pos(T - 1, 0) == T - 1 and pos(0, 1) == T
    else:
        assert pos(0, S - 1) == S - 1                # frame 0 first, in patch order
        assert pos(F0, 0) == F0 * S                  # first non-sink token right after
        assert pos(F0 + 1, 0) == F0 * S + 1          # same patch, next frame: adjacent
        assert pos(F0, 1) == F0 * S + (T - F0)       # next patch after T-F0 frames
    assert pos(T - 1, S - 1) == N - 1
    sp = oracle.perm_table(syn.ROUTE_SPATIAL, layout, T, S, F0)
    assert np.array_equal(sp, np.arange(N))          # spatial heads keep frame-major order


# ----------------------------------------------------------------------------- tile classes
def class_totals(cls):
    return int((cls == 1).sum()), int((cls == 2).sum()), int((cls == 0).sum())


def test_tiny_tile_class_totals():
    """Hand-derived totals, 64x64 tiles on 4 x (8x16):
    spatial: frames are 2 tiles wide and 12 of 16 frame pairs are kept -> 48 full, 16 empty.
    temporal, frame-0 prefix: the 2 sink key tiles are full for all 8 query tiles (16); each
      other key tile spans ~21 patch indices > b = 16, so none is full; 24 are within
      distance 16 of the query tile's patch range (boundary) and 24 are not (empty).
    temporal, fully space-major: every key tile holds frame-0 keys (never empty); a tile
      spans 16 patches, so only the 8 diagonal tiles are full."""
    w = syn.TINY
    T, S = w.frames, w.frame_size
    cnt, cls = oracle.tile_counts(syn.ROUTE_SPATIAL, 0, T, S, 1, 16, 1, 64, 64)
    assert class_totals(cls) == (48, 0, 16)
    assert int(cnt.sum()) == 196608
    _, cls = oracle.tile_counts(syn.ROUTE_TEMPORAL, syn.LAYOUT_SINK_PREFIX, T, S, 1, 16, 1, 64, 64)
    assert class_totals(cls) == (16, 24, 24)
    _, cls = oracle.tile_counts(syn.ROUTE_TEMPORAL, syn.LAYOUT_FULL_SPACE_MAJOR, T, S, 1, 16, 1, 64, 64)
    assert class_totals(cls) == (8, 56, 0)


CASES = [
    # route, layout, T, H, W, k, b, F0, bq, bk
    (0, 0, 4, 8, 16, 1, 16, 1, 64, 64),
    (1, 0, 4, 8, 16, 1, 16, 1, 64, 64),
    (1, 1, 4, 8, 16, 1, 16, 1, 64, 64),
    (0, 0, 5, 3, 7, 1, 4, 1, 16, 8),      # frames not aligned with tiles, ragged tail
    (1, 0, 5, 3, 7, 1, 4, 1, 16, 8),
    (1, 1, 5, 3, 7, 1, 2, 1, 8, 16),
    (0, 0, 6, 4, 5, 2, 3, 2, 24, 16),     # two sink frames
    (1, 0, 6, 4, 5, 2, 3, 2, 24, 16),
]


@pytest.mark.parametrize("case", CASES)
def test_tile_classes_match_interval_derivation(case):
    route, layout, T, H, W, k, b, F0, bq, bk = case
    S = H * W
    cnt, cls = oracle.tile_counts(route, layout, T, S, k, b, F0, bq, bk)
    ref = interval_classes(route, layout, T, S, k, b, F0, bq, bk)
    assert np.array_equal(cls, ref)
    # class is consistent with the count, and the counts add up to the retained pairs
    area = oracle.tile_areas(T * S, bq, bk)
    assert np.array_equal(cls == 1, cnt == area) and np.array_equal(cls == 0, cnt == 0)
    assert int(cnt.sum()) == oracle.retained_pairs(route, T, S, k, b, F0)


@pytest.mark.parametrize("route,bq,bk", [(0, 128, 128), (1, 128, 128), (1, 256, 64)])
def test_tile_classes_pages_shape_sampled_rows(route, bq, bk):
    """Pages' 75,600-token shape: sampled q-tile rows (first, ragged last, frame-straddling)."""
    w = syn.MIXED_75K
    T, S, N = w.frames, w.frame_size, w.tokens
    nq = -(-N // bq)
    qts = [0, 1, 27, 28, nq // 2, nq - 2, nq - 1]
    cnt, cls = oracle.tile_counts(route, 0, T, S, 3, 715, 1, bq, bk, qts=qts)
    ref = interval_classes(route, 0, T, S, 3, 715, 1, bq, bk, qts=qts)
    assert np.array_equal(cls, ref)


def test_layout_preserves_budget():
    """The exact mask keeps the same pairs whatever the token order: the per-tile counts of
    each layout add up to the same total."""
    T, S, b = 5, 21, 3
    tot = []
    for layout in (0, 1):
        cnt, _ = oracle.tile_counts(1, layout, T, S, 0, b, 1, 16, 16)
        tot.append(int(cnt.sum()))
    assert tot[0] == tot[1] == closed_form_temporal(T, S, b, 1)


def test_rounded_rule():
    f = oracle.lib().or_rounded_class
    assert f(8, 16) == 1 and f(7, 16) == 0 and f(0, 16) == 0 and f(16, 16) == 1 and f(3, 5) == 1
    # tiles aligned with frames: no boundary tiles, so rounding changes nothing
    cnt, cls = oracle.tile_counts(0, 0, 4, 128, 1, 0, 1, 64, 64)
    r = oracle.rounded_classes(cnt, oracle.tile_areas(512, 64, 64))
    assert np.array_equal(r, cls)


# ----------------------------------------------------------------------------- attention
def numpy_masked_attention(q, k, v, mask, scale):
    """Textbook attention with an explicit [N, N] boolean mask (numpy, fp64)."""
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p = np.where(mask, p, 0.0)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v) / l, (m + np.log(l))[:, 0]


def explicit_mask(route, T, S, k, b, F0):
    t, s = token_fs(T, S)
    if route == 0:
        m = np.abs(t[:, None] - t[None, :]) <= k
    else:
        m = np.abs(s[:, None] - s[None, :]) <= b
    return m | (t[None, :] < F0)


@pytest.mark.parametrize("route", [0, 1])
def test_attention_brute_force_tiny(route):
    w = syn.TINY
    T, S, N, d = w.frames, w.frame_size, w.tokens, w.d
    q, k, v = syn.make_qkv(w)
    h = route
    rows = np.arange(N)
    out, lse = oracle.attention_rows(q[h], k[h], v[h], rows, route=route, layout=0, T=T, S=S,
                                     frame_window=1, band=16, F0=1)
    ref, ref_lse = numpy_masked_attention(f64(q[h]), f64(k[h]), f64(v[h]),
                                          explicit_mask(route, T, S, 1, 16, 1), 1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_q_zero_gives_mean_of_kept_values():
    T, H, W, d = 5, 3, 4, 16
    S, N = H * W, T * H * W
    g = torch.Generator().manual_seed(5)
    v = bf16(torch.randn(N, d, generator=g))
    q = bf16(torch.zeros(N, d))
    k = bf16(torch.randn(N, d, generator=g))
    for route, kk, b in [(0, 1, 0), (1, 0, 2)]:
        out, lse = oracle.attention_rows(q, k, v, np.arange(N), route=route, layout=0, T=T, S=S,
                                         frame_window=kk, band=b, F0=1)
        vv = f64(v)
        for i in range(N):
            ti, si = divmod(i, S)
            if route == 0:
                frames = {g_ for g_ in range(T) if abs(g_ - ti) <= kk} | {0}
                kept = [j for j in range(N) if j // S in frames]
            else:
                kept = [j for j in range(N) if j // S == 0 or abs(j % S - si) <= b]
            np.testing.assert_allclose(out[i], vv[kept].mean(axis=0), rtol=1e-12, atol=1e-12)
            assert abs(lse[i] - math.log(len(kept))) < 1e-12


def test_attention_all_kept_is_dense_softmax_and_rows_sum_to_one():
    T, H, W, d = 3, 4, 4, 32
    S, N = H * W, T * H * W
    g = torch.Generator().manual_seed(11)
    q, k, v = (bf16(torch.randn(N, d, generator=g) * 2) for _ in range(3))
    scale = 0.3
    rows = np.arange(N)
    dense, _ = oracle.attention_rows(q, k, v, rows, route=0, layout=0, T=T, S=S, frame_window=0,
                                     band=0, F0=0, scale=scale, mask_kind=oracle.MASK_ALL)
    s = f64(q) @ f64(k).T * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ f64(v)
    np.testing.assert_allclose(dense, ref, rtol=1e-11, atol=1e-12)
    # a spatial window covering every frame keeps every pair
    wide, _ = oracle.attention_rows(q, k, v, rows, route=0, layout=0, T=T, S=S, frame_window=T,
                                    band=0, F0=1, scale=scale)
    np.testing.assert_allclose(wide, dense, rtol=0, atol=0)
    ones = bf16(torch.ones(N, d))
    o1, _ = oracle.attention_rows(q, k, ones, rows, route=1, layout=0, T=T, S=S, frame_window=0,
                                  band=1, F0=1, scale=scale)
    np.testing.assert_allclose(o1, 1.0, rtol=1e-13)


def test_sink_always_kept():
    rng = np.random.default_rng(3)
    T, S = 7, 13
    for _ in range(500):
        i, s = rng.integers(0, T * S), rng.integers(0, S)
        for route in (0, 1):
            assert oracle.keep(route, S, 0, 0, 1, int(i), int(s)) == 1   # key in frame 0


def test_rounded_mask_attention_matches_explicit_tile_mask():
    T, H, W, d, bq, bk = 5, 3, 7, 16, 16, 8
    S, N = H * W, T * H * W
    g = torch.Generator().manual_seed(2)
    q, k, v = (bf16(torch.randn(N, d, generator=g)) for _ in range(3))
    for route, layout in [(0, 0), (1, 0), (1, 1)]:
        cnt, _ = oracle.tile_counts(route, layout, T, S, 1, 4, 1, bq, bk)
        rc = oracle.rounded_classes(cnt, oracle.tile_areas(N, bq, bk))
        out, _ = oracle.attention_rows(q, k, v, np.arange(N), route=route, layout=layout, T=T, S=S,
                                       frame_window=1, band=4, F0=1, mask_kind=oracle.MASK_ROUNDED,
                                       rcls=rc, bq=bq, bk=bk)
        pi = oracle.perm_table(route, layout, T, S, 1)
        mask = rc[(pi // bq)[:, None], (pi // bk)[None, :]] == 1
        has = mask.any(axis=1)
        ref, _ = numpy_masked_attention(f64(q)[has], f64(k), f64(v), mask[has], 1 / math.sqrt(d))
        np.testing.assert_allclose(out[has], ref, rtol=1e-10, atol=1e-12)
        assert np.all(out[~has] == 0)


# ----------------------------------------------------------------------------- head routing
def test_route_masks_equal_to_dense_have_zero_error():
    """A spatial window covering every frame keeps every pair, so E_spatial = 0 exactly; a
    patch band covering every patch does the same for E_temporal."""
    w = syn.Workload("r", frames=4, grid_h=4, grid_w=6, routes=(0,), d=32, frame_window=1, spatial_band=2)
    q, k, v = syn.make_qkv(w, seed_offset=4)
    rows = np.arange(0, w.tokens, 5)
    es, et, ed = oracle.route_errors(q[0], k[0], v[0], rows, T=4, S=24, frame_window=4, band=2, F0=1)
    assert es == 0.0 and et > 0.0 and ed > 0.0
    es, et, ed = oracle.route_errors(q[0], k[0], v[0], rows, T=4, S=24, frame_window=1, band=24, F0=1)
    assert et == 0.0 and es > 0.0
    assert oracle.route(q[0], k[0], v[0], rows, T=4, S=24, frame_window=1, band=24, F0=1) == syn.ROUTE_TEMPORAL


def test_route_constant_values_and_ties():
    w = syn.Workload("r", frames=3, grid_h=4, grid_w=4, routes=(0,), d=16, frame_window=0, spatial_band=1)
    q, k, _ = syn.make_qkv(w, seed_offset=6)
    v = bf16(torch.full((w.tokens, w.d), 0.75))
    es, et, ed = oracle.route_errors(q[0], k[0], v, np.arange(w.tokens), T=3, S=16, frame_window=0, band=1, F0=1)
    # every mask averages the same constant: both errors are rounding noise only
    assert es < 1e-20 and et < 1e-20 and abs(ed - w.tokens * w.d * 0.5625) < 1e-9
    # both masks keep every pair: the errors are exactly equal (zero) and the tie goes spatial
    es, et, _ = oracle.route_errors(q[0], k[0], v, np.arange(w.tokens), T=3, S=16, frame_window=3, band=16, F0=1)
    assert es == et == 0.0
    assert oracle.route(q[0], k[0], v, np.arange(w.tokens), T=3, S=16, frame_window=3, band=16, F0=1) == 0


def test_route_recovers_planted_structure():
    w = syn.Workload("r", frames=6, grid_h=8, grid_w=8, routes=(0, 1, 1, 0), d=64, frame_window=1, spatial_band=2)
    kinds = [0, 1, 1, 0]
    q, k, v = syn.make_routed_qkv(w, kinds)
    rows = np.arange(0, w.tokens, 7)
    for h, kind in enumerate(kinds):
        kw = dict(T=w.frames, S=w.frame_size, frame_window=1, band=2, F0=1)
        es, et, _ = oracle.route_errors(q[h], k[h], v[h], rows, **kw)
        assert oracle.route(q[h], k[h], v[h], rows, **kw) == kind, (h, es, et)
        assert (es < 0.5 * et) if kind == 0 else (et < 0.5 * es)
