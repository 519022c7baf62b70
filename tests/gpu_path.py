"""Test-side driver of the CUDA path and its comparison with the oracle.

run_path() pushes original-order Q/K/V through the product's public calls exactly as a user
would: svg_permute (temporal heads to their order), svg_build_tilemap per route class,
svg_attention_fwd (or svg_dense_attention_fwd), svg_permute inverse on O. compare_rows()
checks sampled rows of every head against the fp64 oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_spatio_flash_b200 import synthetic as syn

REL_L2_TOL = 1e-2   # relative L2 error of O per head
MAX_ABS_TOL = 2e-2  # max |O_gpu - O_oracle|
LSE_ABS_TOL = 5e-3  # LSE is accumulated in fp32 from fp32 probabilities


def svg():
    from block_sparse_spatio_flash_b200 import svg as mod
    return mod


def geom_mask_tile(w: syn.Workload, variant=None, bq=None, bk=None):
    S = svg()
    g = S.make_geom(w.frames, w.grid_h, w.grid_w)
    m = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames,
                    w.variant if variant is None else variant, w.layout)
    t = S.make_tile(w.bq if bq is None else bq, w.bk if bk is None else bk)
    return g, m, t


def build_maps(w, g, m, t, routes):
    S = svg()
    maps = [None, None]
    for c in (0, 1):
        if c in routes:
            ws = S.alloc_workspace(g, t)
            S.svg_build_tilemap(g, m, t, c, ws)
            maps[c] = ws
    return maps


def run_path(w: syn.Workload, q, k, v, *, mode=0, variant=None, bq=None, bk=None, dense=False, lse=True,
             stall=False):
    """Returns (O [H, N, d] bf16 CPU in original order, LSE [H, N] fp32 CPU in POSITION order, status).
    stall: run the launch through the test hook whose wait runs out (svg_test_attention_fwd_stall)."""
    S = svg()
    dev = torch.device("cuda")
    g, m, t = geom_mask_tile(w, variant, bq, bk)
    routes = list(w.routes)
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    if not dense and any(routes):
        qp, kp, vp = (torch.empty_like(x) for x in (qd, kd, vd))
        for src, dst in ((qd, qp), (kd, kp), (vd, vp)):
            S.svg_permute(src, dst, routes, g, m, inverse=False)
    else:
        qp, kp, vp = qd, kd, vd
    o = torch.empty_like(qp)
    ls = torch.empty(qp.shape[:2], dtype=torch.float32, device=dev) if lse else None
    scratch = S.alloc_scratch()
    if dense:
        S.svg_dense_attention_fwd(qp, kp, vp, o, bk=t.bk, scratch=scratch, lse=ls)
    else:
        maps = build_maps(w, g, m, t, routes)
        fwd = S.svg_test_attention_fwd_stall if stall else S.svg_attention_fwd
        fwd(qp, kp, vp, o, routes, maps[0], maps[1], g, m, t, mode=mode, scratch=scratch, lse=ls)
    status = S.svg_read_status(scratch)
    if not dense and any(routes):
        out = torch.empty_like(o)
        S.svg_permute(o, out, routes, g, m, inverse=True)
    else:
        out = o
    torch.cuda.synchronize()
    return out.cpu(), (ls.cpu() if lse else None), status


def oracle_rows(w, q, k, v, h, rows, *, variant=None, bq=None, bk=None, all_kept=False):
    route = w.routes[h]
    var = w.variant if variant is None else variant
    bq = w.bq if bq is None else bq
    bk = w.bk if bk is None else bk
    kw = dict(route=route, layout=w.layout, T=w.frames, S=w.frame_size, frame_window=w.frame_window,
              band=w.spatial_band, F0=w.sink_frames)
    if all_kept:
        return oracle.attention_rows(q[h], k[h], v[h], rows, mask_kind=oracle.MASK_ALL, **kw)
    if var == syn.MASK_EXACT:
        return oracle.attention_rows(q[h], k[h], v[h], rows, **kw)
    # rounded: brute-force counts of the q-tiles these rows fall in, then the rounding rule
    N = w.tokens
    pi = oracle.perm_table(route, w.layout, w.frames, w.frame_size, w.sink_frames)
    qts = np.unique(pi[rows] // bq)
    cnt, _ = oracle.tile_counts(route, w.layout, w.frames, w.frame_size, w.frame_window, w.spatial_band,
                                w.sink_frames, bq, bk, qts=qts)
    rc_rows = oracle.rounded_classes(cnt, oracle.tile_areas(N, bq, bk, qts))
    nq, nk = -(-N // bq), -(-N // bk)
    rcls = np.zeros((nq, nk), dtype=np.uint8)
    rcls[qts] = rc_rows
    return oracle.attention_rows(q[h], k[h], v[h], rows, mask_kind=oracle.MASK_ROUNDED, rcls=rcls, bq=bq, bk=bk,
                                 **kw)


def oracle_rows_cached(cache, key, w, q, k, v, h, rows, **kw):
    """oracle_rows through a per-row memo: `key` names the inputs and the mask (the same key must
    mean the same q / k / v and the same mask), so that checks of one workload under several tile
    shapes of the exact mask share the oracle's rows."""
    store = cache.setdefault(tuple(key) + (h,), {})
    missing = np.array([r for r in rows.tolist() if r not in store], dtype=np.int64)
    if len(missing):
        o, l = oracle_rows(w, q, k, v, h, missing, **kw)
        for i, r in enumerate(missing.tolist()):
            store[r] = (o[i], l[i])
    return (np.stack([store[r][0] for r in rows.tolist()]),
            np.array([store[r][1] for r in rows.tolist()], dtype=np.float64))


def compare_rows(w, q, k, v, out, lse, rows_per_head=None, cache=None, cache_key=None, **kw):
    """Check every head on its sampled rows; returns a list of per-head stats. With `cache` (a dict)
    and `cache_key`, oracle rows are memoised across calls (see oracle_rows_cached)."""
    # LSE rows are in each head's token order, except on the dense path (never permuted)
    permuted = not kw.get("all_kept", False)
    stats = []
    for h in range(w.heads):
        rows = syn.sample_rows(w, h) if rows_per_head is None else rows_per_head(h)
        rows = np.asarray(rows, dtype=np.int64)
        if cache is not None:
            ref, ref_lse = oracle_rows_cached(cache, cache_key, w, q, k, v, h, rows, **kw)
        else:
            ref, ref_lse = oracle_rows(w, q, k, v, h, rows, **kw)
        got = out[h, torch.as_tensor(rows)].to(torch.float64).numpy()
        diff = got - ref
        rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))
        mx = float(np.abs(diff).max())
        st = {"head": h, "rows": len(rows), "rel_l2": rel, "max_abs": mx}
        assert rel <= REL_L2_TOL and mx <= MAX_ABS_TOL, st
        if lse is not None:
            pi = (oracle.perm_table(w.routes[h], w.layout, w.frames, w.frame_size, w.sink_frames)
                  if permuted else np.arange(w.tokens))
            got_l = lse[h, torch.as_tensor(pi[rows])].to(torch.float64).numpy()
            fin = np.isfinite(ref_lse)
            assert np.array_equal(fin, np.isfinite(got_l)), st
            if fin.any():
                dl = float(np.abs(got_l[fin] - ref_lse[fin]).max())
                st["lse_max_abs"] = dl
                assert dl <= LSE_ABS_TOL, st
        stats.append(st)
    return stats


def tail_rows(w, h, extra=64):
    """Original rows whose POSITIONS are the last `extra` of the sequence (the ragged tile)."""
    pi = oracle.perm_table(w.routes[h], w.layout, w.frames, w.frame_size, w.sink_frames)
    inv = np.empty_like(pi)
    inv[pi] = np.arange(len(pi))
    return inv[max(0, len(pi) - extra):]


def scale_for(d):
    return 1.0 / math.sqrt(d)


def run_fused(w: syn.Workload, q, k, v, *, mode=0, variant=None, bq=None, bk=None, lse=True):
    """svg_attention_fwd_fused on original-order tensors. Returns (O [H, N, d] bf16 CPU, LSE [H, N]
    fp32 CPU, both in ORIGINAL order, status)."""
    S = svg()
    dev = torch.device("cuda")
    g, m, t = geom_mask_tile(w, variant, bq, bk)
    routes = list(w.routes)
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o = torch.empty_like(qd)
    ls = torch.empty(qd.shape[:2], dtype=torch.float32, device=dev) if lse else None
    scratch = S.alloc_scratch()
    maps = build_maps(w, g, m, t, routes)
    S.svg_attention_fwd_fused(qd, kd, vd, o, routes, maps[0], maps[1], g, m, t, mode=mode, scratch=scratch, lse=ls)
    status = S.svg_read_status(scratch)
    torch.cuda.synchronize()
    return o.cpu(), (ls.cpu() if lse else None), status


def lse_to_original(w: syn.Workload, lse):
    """LSE rows from each head's position order to the original order."""
    out = torch.empty_like(lse)
    for h in range(w.heads):
        pi = oracle.perm_table(w.routes[h], w.layout, w.frames, w.frame_size, w.sink_frames)
        out[h] = lse[h, torch.as_tensor(pi)]
    return out


def quantize_e4m3(x):
    """bf16 -> e4m3 (round to nearest) -> bf16: the values the 8-bit QK^T path sees, exactly."""
    return x.to(torch.float8_e4m3fn).to(torch.bfloat16)


def run_qk8(w: syn.Workload, q, k, v, *, mode=0, variant=None, bq=None, bk=None):
    """svg_attention_fwd_qk8 on e4m3 copies of q and k (q and k must already hold e4m3 values in bf16,
    see quantize_e4m3). Returns (O [H, N, d] bf16 CPU in original order, status)."""
    S = svg()
    dev = torch.device("cuda")
    g, m, t = geom_mask_tile(w, variant, bq, bk)
    routes = list(w.routes)
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    qp, kp, vp = (torch.empty_like(x) for x in (qd, kd, vd))
    for src, dst in ((qd, qp), (kd, kp), (vd, vp)):
        S.svg_permute(src, dst, routes, g, m, inverse=False)
    q8, k8 = (x.to(torch.float8_e4m3fn).contiguous() for x in (qp, kp))  # exact: the values are e4m3
    o = torch.empty_like(vp)
    scratch = S.alloc_scratch()
    maps = build_maps(w, g, m, t, routes)
    S.svg_attention_fwd_qk8(q8, k8, vp, o, routes, maps[0], maps[1], g, m, t, mode=mode, scratch=scratch)
    status = S.svg_read_status(scratch)
    out = torch.empty_like(o)
    S.svg_permute(o, out, routes, g, m, inverse=True)
    torch.cuda.synchronize()
    return out.cpu(), status
