"""The allocation-free attention entry point (svg_attention_fwd_noalloc).

It serves callers that cannot allocate device memory themselves -- a plugin inside a host
framework that only hands over its input and output buffers, or a server that forbids device
allocation after start-up -- by keeping its scratch in a static device array inside the
library. This test calls it through the C ABI twice in a row (the second call reuses the
array the first one left behind) and checks both outputs against the regular entry point,
with the tolerances of the other parity tests. The file sorts last so that a run stopping at
the first failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest
import torch

from block_sparse_spatio_flash_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

REL_L2_TOL = 1e-2
MAX_ABS_TOL = 2e-2

WORKLOAD = syn.Workload("noalloc_mixed", frames=5, grid_h=12, grid_w=20, routes=(0, 1, 1, 0), d=128,
                        frame_window=1, spatial_band=20, bq=128, bk=128)


def _close(a, b):
    a64, b64 = a.double(), b.double()
    rel = float((a64 - b64).norm() / b64.norm().clamp_min(1e-30))
    mx = float((a64 - b64).abs().max())
    return rel <= REL_L2_TOL and mx <= MAX_ABS_TOL, rel, mx


def test_noalloc_matches_regular_entry_point_twice():
    from block_sparse_spatio_flash_b200 import build
    build.build()
    from block_sparse_spatio_flash_b200 import svg as S

    w = WORKLOAD
    dev = torch.device("cuda")
    g = S.make_geom(w.frames, w.grid_h, w.grid_w)
    m = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, w.variant, w.layout)
    t = S.make_tile(w.bq, w.bk)
    routes = list(w.routes)
    q, k, v = (x.to(dev) for x in syn.make_qkv(w, seed_offset=21))
    qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
    for a, b in ((q, qp), (k, kp), (v, vp)):
        S.svg_permute(a, b, routes, g, m)
    ws = [None, None]
    for c in (0, 1):
        ws[c] = S.alloc_workspace(g, t)
        S.svg_build_tilemap(g, m, t, c, ws[c])

    ref = torch.empty_like(qp)
    ref_lse = torch.empty(qp.shape[:2], dtype=torch.float32, device=dev)
    scratch = S.alloc_scratch()
    S.svg_attention_fwd(qp, kp, vp, ref, routes, ws[0], ws[1], g, m, t, scratch=scratch, lse=ref_lse)
    assert S.svg_read_status(scratch) == 0

    status = torch.full((1,), 12345, dtype=torch.int32, device=dev)
    outs = [torch.full_like(qp, float("nan")) for _ in range(3)]
    lses = [torch.full_like(ref_lse, float("nan")) for _ in range(3)]
    for call in range(2):
        o, lse = outs[call], lses[call]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        S.svg_attention_fwd_noalloc(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, lse=lse, status=status)
        torch.cuda.synchronize()
        if call == 1:  # the library is loaded and its array resident: a call allocates no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        ok, rel, mx = _close(o.float(), ref.float())
        assert ok, (call, rel, mx)
        assert torch.isfinite(o.float()).all()
        assert float((lse - ref_lse).abs().max()) <= 5e-3
    # without a status pointer the status word inside the library's own array is used
    S.svg_attention_fwd_noalloc(qp, kp, vp, outs[2], routes, ws[0], ws[1], g, m, t, lse=lses[2])
    torch.cuda.synchronize()
    ok, rel, mx = _close(outs[2].float(), ref.float())
    assert ok, ("no status pointer", rel, mx)


def test_noalloc_rejects_bad_arguments_without_touching_the_device():
    import ctypes
    from block_sparse_spatio_flash_b200 import svg as S
    lib = ctypes.CDLL(S.LIB_PATH)
    f = lib.svg_attention_fwd_noalloc
    f.argtypes = S._sig["svg_attention_fwd_noalloc"][1]
    g, m, t = S.make_geom(4, 8, 16), S.make_mask(1, 16), S.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    p = ctypes.c_void_p(1 << 20)
    assert f(None, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, None, None) == S.SVG_ERR_ARG
    assert f(p, p, p, p, None, 2, 512, 96, 0.0, routes, p, p, g, m, t, 0, None, None) == S.SVG_ERR_UNSUPPORTED
    assert np.int32(S.svg_attention_scratch_bytes()) <= 256
