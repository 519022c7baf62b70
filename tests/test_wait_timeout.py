"""Failure detection on the GPU without a fault: a launch whose softmax warps wait on a barrier that
nothing completes (the test entry point svg_test_attention_fwd_stall) must give up after the bounded wait, report
SVG_ERR_TIMEOUT through the status word, drain its copies and MMAs, free TMEM and return; the next
launch in the same context must then run normally and match the oracle."""
import pytest

from block_sparse_spatio_flash_b200 import synthetic as syn
from tests import gpu_path as gp

pytestmark = pytest.mark.gpu

W = syn.Workload("timeout_1200", frames=5, grid_h=12, grid_w=20, routes=(0, 1), d=128, frame_window=1,
                 spatial_band=20)


@pytest.fixture(scope="module")
def S():
    from block_sparse_spatio_flash_b200 import build
    build.build()
    return gp.svg()


def test_stalled_wait_reports_timeout_and_context_survives(S):
    q, k, v = syn.make_qkv(W, seed_offset=31)
    _, _, st = gp.run_path(W, q, k, v, stall=True)
    assert st == S.SVG_ERR_TIMEOUT
    out, lse, st = gp.run_path(W, q, k, v)
    assert st == 0
    gp.compare_rows(W, q, k, v, out, lse)
