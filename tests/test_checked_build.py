"""The checked build (libsvgattn_checked.so, -DSVG_CHECKED=1): every kernel checks the indexes it
computes for global memory, tile-map arrays and TMA coordinates, counts a failed check and skips or
clamps the access instead of trapping. compute-sanitizer is closed on this machine; this build is the
race / out-of-range detector of the small cases.

CPU: both libraries export the same entry points, and each reports which build it is.
GPU (a child process with SVG_CHECKED=1): the small cases of every entry point run with zero failed
checks and match the oracle; a tile map with one corrupted entry (a key tile past the map) is
caught by the checks, counted, and does not fault."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libs():
    from block_sparse_spatio_flash_b200 import build
    return build.build(), build.build(checked=True)


def test_both_builds_export_the_same_symbols_and_name_themselves(libs):
    from tests.test_abi import declared_functions
    release, checked = (ctypes.CDLL(p) for p in libs)
    for lib in (release, checked):
        missing = [n for n in declared_functions() if not hasattr(lib, n)]
        assert not missing, missing
    assert release.svg_checked_build() == 0 and checked.svg_checked_build() == 1
    n = ctypes.c_uint32(7)
    assert release.svg_checks_failed(ctypes.byref(n), 1) == 0 and n.value == 0  # no device work
    assert release.svg_checks_failed(None, 1) == -1


CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import numpy as np
import torch
from block_sparse_spatio_flash_b200 import synthetic as syn
from block_sparse_spatio_flash_b200 import svg as S
from tests import gpu_path as gp
assert S.svg_checked_build()
S.svg_checks_failed(reset=True)
medium = syn.Workload("medium_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 0, 1), d=128, frame_window=1,
                      spatial_band=20)
cases = [
    (syn.TINY, dict()),
    (medium, dict()),
    (medium, dict(bq=256, bk=64)),
    (medium.replace(variant=1), dict()),
    (syn.Workload("two_sinks_fsm", frames=7, grid_h=5, grid_w=9, routes=(1, 0), d=128, frame_window=1,
                  spatial_band=3, sink_frames=2, layout=1, bq=256, bk=64), dict()),
    (syn.Workload("d64_ragged", frames=5, grid_h=6, grid_w=9, routes=(1, 1, 0), d=64, frame_window=0,
                  spatial_band=2, bq=64, bk=64), dict()),
]
for w, kw in cases:
    q, k, v = syn.make_qkv(w, seed_offset=81)
    for mode in (0, 1):
        out, lse, st = gp.run_path(w, q, k, v, mode=mode, **kw)
        assert st == 0, st
        gp.compare_rows(w, q, k, v, out, lse, variant=w.variant, **kw)
    out, _, st = gp.run_fused(w, q, k, v, lse=False, **kw)
    assert st == 0, st
    gp.compare_rows(w, q, k, v, out, None, variant=w.variant, **kw)
    out, lse, st = gp.run_path(w, q, k, v, dense=True, bk=kw.get("bk", w.bk))
    assert st == 0, st
    gp.compare_rows(w, q, k, v, out, lse, all_kept=True)
    n = S.svg_checks_failed(reset=True)
    assert n == 0, (w.name, n)
# the work-ordered scheduler and the e4m3 call
w = medium
q, k, v = syn.make_qkv(w, seed_offset=83)
g, m, t = gp.geom_mask_tile(w)
dev = torch.device("cuda")
qp, kp, vp = (torch.empty_like(x) for x in (x_.to(dev) for x_ in (q, k, v)))
for a, b in zip((q, k, v), (qp, kp, vp)):
    S.svg_permute(a.to(dev), b, list(w.routes), g, m)
maps = gp.build_maps(w, g, m, t, list(w.routes))
o = torch.empty_like(qp)
sc = S.alloc_scratch()
S.svg_attention_fwd_ex(qp, kp, vp, o, list(w.routes), maps[0], maps[1], g, m, t, scratch=sc, order=S.SVG_ORDER_WORK)
assert S.svg_read_status(sc) == 0
q8, k8 = gp.quantize_e4m3(q), gp.quantize_e4m3(k)
out, st = gp.run_qk8(w, q8, k8, v)
assert st == 0
gp.compare_rows(w, q8, k8, v, out, None)
assert S.svg_checks_failed(reset=True) == 0
# a corrupted tile map: the first entry of the first item names a key tile past the map
A = S.tilemap_arrays(maps[0], g, t)
ptr0 = int(A["pair_ptr"][0].item())
ent = A["pair_ent"][ptr0: ptr0 + 1]
flags = int(ent.item()) & ~0x0FFFFFFF  # a signed int32: the flag bits keep their two's-complement sign
ent.fill_(flags | (A["nk"] + 5))
S.svg_attention_fwd(qp, kp, vp, o, list(w.routes), maps[0], maps[1], g, m, t, scratch=sc)
assert S.svg_read_status(sc) == 0
n = S.svg_checks_failed(reset=True)
assert n > 0, n
print("ok", n)
"""


@pytest.mark.gpu
def test_checked_build_runs_clean_and_catches_a_corrupted_map(libs):
    env = dict(os.environ, SVG_CHECKED="1")
    env.pop("SVG_KERNEL", None)
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "ok" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])
