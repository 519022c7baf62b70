"""The selectable schedule (SVG_KERNEL=ps: the attention kernel with P staged in shared memory)
against the oracle, on every entry the option reaches: sparse (both modes, both masks), dense,
d = 64, fused token order (bitwise equal to the permuted path under the same schedule), e4m3
QK^T and the bounded-wait path. The choice is read once per process, so it runs in a child
process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import torch
from block_sparse_spatio_flash_b200 import synthetic as syn
from tests import gpu_path as gp
cases = [
    (syn.Workload("medium_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 0, 1), d=128, frame_window=1,
                  spatial_band=20), dict()),
    (syn.Workload("medium_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 0, 1), d=128, frame_window=1,
                  spatial_band=20), dict(bq=256, bk=64)),
    (syn.Workload("rounded_1200", frames=5, grid_h=12, grid_w=20, routes=(1, 0), d=128, frame_window=1,
                  spatial_band=20, variant=1), dict()),
    (syn.Workload("sparse_rounded", frames=3, grid_h=16, grid_w=32, routes=(1,), d=128, frame_window=0,
                  spatial_band=0, sink_frames=0, variant=1), dict()),
]
for w, kw in cases:
    for mode in (0, 1):
        q, k, v = syn.make_qkv(w, seed_offset=41)
        out, lse, st = gp.run_path(w, q, k, v, mode=mode, **kw)
        assert st == 0, st
        gp.compare_rows(w, q, k, v, out, lse, variant=w.variant, **kw)
    q, k, v = syn.make_qkv(w, seed_offset=43)
    out, lse, st = gp.run_path(w, q, k, v, dense=True, bk=kw.get("bk", 128))
    assert st == 0, st
    gp.compare_rows(w, q, k, v, out, lse, all_kept=True)
# every other entry the option reaches: d = 64, fused token order, e4m3 QK^T, the bounded-wait path
w64 = syn.Workload("d64_ragged", frames=5, grid_h=6, grid_w=9, routes=(1, 1, 0), d=64, frame_window=0,
                   spatial_band=2, bq=64, bk=64)
for bk in (64, 128):
    q, k, v = syn.make_qkv(w64, seed_offset=47)
    out, lse, st = gp.run_path(w64, q, k, v, bk=bk)
    assert st == 0, st
    gp.compare_rows(w64, q, k, v, out, lse, bk=bk)
wf = cases[0][0]
q, k, v = syn.make_qkv(wf, seed_offset=53)
want, _, st = gp.run_path(wf, q, k, v, lse=False)
got, _, st2 = gp.run_fused(wf, q, k, v, lse=False)
assert st == 0 and st2 == 0, (st, st2)
assert (got.view(torch.int16) == want.view(torch.int16)).all()
gp.compare_rows(wf, q, k, v, got, None)
q8, k8 = gp.quantize_e4m3(q), gp.quantize_e4m3(k)
out, st = gp.run_qk8(wf, q8, k8, v)
assert st == 0, st
gp.compare_rows(wf, q8, k8, v, out, None)
_, _, st = gp.run_path(wf, q, k, v, stall=True)
assert st == -4, st
out, lse, st = gp.run_path(wf, q, k, v)
assert st == 0, st
gp.compare_rows(wf, q, k, v, out, lse)
print("ok")
"""


def test_p_in_shared_memory_schedule_matches_oracle():
    env = dict(os.environ, SVG_KERNEL="ps")
    child = CHILD.format(root=ROOT)
    r = subprocess.run([sys.executable, "-c", child], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), (r.stdout[-2000:], r.stderr[-4000:])
