import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


def pytest_collection_modifyitems(config, items):
    if _has_gpu():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    """With SVG_CHECKED=1 the suite runs on the checked build (device-side bounds checks): every check
    that failed anywhere in the session fails the run."""
    if os.environ.get("SVG_CHECKED") != "1" or not _has_gpu():
        return
    import sys as _sys
    mod = _sys.modules.get("block_sparse_spatio_flash_b200.svg")
    if mod is None:
        return
    n = mod.svg_checks_failed(reset=False)
    if n:
        print(f"\nchecked build: {n} device-side bounds checks failed during the session")
        session.exitstatus = 1
