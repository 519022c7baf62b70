"""Copy plans of the fused token order, restated on the CPU and checked against the token order.

In fused order a temporal head's tile of ROWS positions [p0, p0 + ROWS) is read where its rows lie in
the original frame-major order ("Sparse Attention Patterns" of "Accelerating Spatio-Temporal Attention
for Video Diffusion on TPUs": temporal heads attend within one patch across frames, so their tokens
are reordered patch-major). Past the sink prefix
the order runs through one patch's frames at a time, so the kernel copies each run of R = T - F0 frames
(T in the fully space-major order) that lies wholly inside the tile as one strided box, and gathers the
4-row groups that hold the partial runs at the tile's edges; a tile that starts inside the sink prefix,
or a run length outside [4, 256], is gathered group by group. The rules below are the ones the kernel
follows (first whole run u_a = ceil(q0 / R), runs [u_a, u_end) with u_end = floor((q0 + ROWS) / R),
a group gathered unless it lies inside the boxes' rows); this test checks, for many geometries and
both token orders, that they place in every row of every tile exactly the token of that position:
boxes disjoint, in range and inside the tile, a group written by a gather and a box twice only with the
same token. The GPU tests check the kernel itself (fused order bitwise equal to the permuted path)."""
import itertools

import pytest


def orig_index(T, S, F0, space_major, p):
    """Original (frame-major) index of the token at position p of a temporal head's order."""
    if space_major:
        s, t = divmod(p, T)
        return t * S + s
    pre = F0 * S
    if p < pre:
        return p
    s, r = divmod(p - pre, T - F0)
    return (F0 + r) * S + s


def plan_tile(T, S, F0, space_major, p0, rows):
    """(boxes, gathered groups) of the tile at position p0: boxes as (first tile row, patch, run)."""
    N = T * S
    pre = 0 if space_major else F0 * S
    run = T if space_major else T - F0
    R = run if 4 <= run <= 256 else 0
    if p0 + rows <= pre:
        return "prefix", [], []
    if p0 < pre or R == 0:
        return "gather", [], list(range(rows // 4))
    q0 = p0 - pre
    runs = (N - pre) // R
    u_a = (q0 + R - 1) // R
    u_end = min((q0 + rows) // R, runs)
    n_box = max(0, u_end - u_a)
    c0 = u_a * R - q0 if n_box else 0
    c1 = u_end * R - q0 if n_box else 0
    boxes = [(pre + u * R - p0, u, R) for u in range(u_a, u_end)]
    groups = [g for g in range(rows // 4) if not (4 * g >= c0 and 4 * g + 4 <= c1)]
    return "runs", boxes, groups


def check_geometry(T, H, W, F0, space_major, rows):
    S = H * W
    N = T * S
    t0 = 0 if space_major else F0
    n_boxes = n_groups = 0
    for p0 in range(0, N, rows):
        kind, boxes, groups = plan_tile(T, S, F0, space_major, p0, rows)
        if kind == "prefix":  # one tiled copy: positions there are the original indices
            assert all(orig_index(T, S, F0, space_major, p) == p for p in range(p0, min(p0 + rows, N)))
            continue
        cover = [None] * rows
        for row, u, R in boxes:
            assert 0 <= row and row + R <= rows, "box outside the tile"
            assert 0 <= u < S and t0 + R <= T, "box outside the tensor"
            for i in range(R):
                assert cover[row + i] is None, "boxes overlap"
                cover[row + i] = (t0 + i) * S + u  # frame t0 + i of patch u
            n_boxes += 1
        for g in groups:
            for i in range(4):
                src = orig_index(T, S, F0, space_major, min(p0 + 4 * g + i, N - 1))
                assert cover[4 * g + i] in (None, src), "a gather and a box write different tokens"
                cover[4 * g + i] = src
            n_groups += 1
        for r in range(rows):  # rows past the end repeat the last token (they are masked)
            assert cover[r] == orig_index(T, S, F0, space_major, min(p0 + r, N - 1)), (p0, r)
    return n_boxes, n_groups


GEOMETRIES = [(4, 8, 16, 1), (5, 12, 20, 1), (6, 8, 10, 1), (7, 5, 9, 2), (5, 6, 9, 1), (21, 45, 80, 1),
              (6, 13, 17, 2), (3, 16, 32, 0), (4, 6, 9, 0), (2, 4, 8, 1), (1, 7, 11, 1), (257, 2, 3, 1),
              (260, 2, 3, 1), (2, 16, 20, 1), (33, 3, 5, 1)]


@pytest.mark.parametrize("geom", GEOMETRIES, ids=lambda g: "x".join(map(str, g)))
def test_plans_place_every_token(geom):
    T, H, W, F0 = geom
    for space_major, rows in itertools.product((False, True), (64, 128)):
        check_geometry(T, H, W, F0, space_major, rows)


def test_pages_shape_uses_boxes_for_most_rows():
    """21 x 45 x 80 with a frame-0 sink: runs of 20 frames, so a 128-row tile is about six boxes
    and the groups of the two partial runs at its edges."""
    n_boxes, n_groups = check_geometry(21, 45, 80, 1, False, 128)
    tiles = (21 * 3600 - 3600) // 128
    assert 5.0 < n_boxes / tiles < 6.5
    assert n_groups / tiles < 8


def test_long_runs_are_gathered():
    """Runs of 256 frames never fit a 128-row tile, and runs past 256 have no box map: gathers only."""
    for T in (257, 260):
        n_boxes, n_groups = check_geometry(T, 2, 3, 1, False, 128)
        assert n_boxes == 0 and n_groups > 0
