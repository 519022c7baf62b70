"""Host-side parts of bench.py's JSON contract (CPU): the captured DRAM traffic is reported only for
the kernel sources, workload and launch shape it was captured on, and both arms print the same
`config` object apart from how the work is spread."""
import argparse

import bench
from block_sparse_spatio_flash_b200 import synthetic as syn


def _args(**kw):
    base = dict(bq=128, bk=128, mode="split")
    base.update(kw)
    return argparse.Namespace(**base)


def test_traffic_only_for_the_captured_kernel_and_workload(monkeypatch):
    c = bench.CAPTURED_TRAFFIC
    monkeypatch.delenv("SVG_KERNEL", raising=False)
    w = syn.WORKLOADS[c["workload"]]
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: c["sources_sha256"])
    assert bench.captured_traffic(w, _args()) == c["bytes_per_head"] * w.heads
    # per-launch bytes grow with the heads processed
    w3 = w.replace(routes=w.routes[:3])
    assert bench.captured_traffic(w3, _args()) == c["bytes_per_head"] * 3
    # another tile shape, mode or workload: no figure
    assert bench.captured_traffic(w, _args(bk=64)) is None
    assert bench.captured_traffic(w, _args(mode="naive")) is None
    assert bench.captured_traffic(syn.TINY, _args()) is None
    # another kernel option selected: no figure
    monkeypatch.setenv("SVG_KERNEL", "ps")
    assert bench.captured_traffic(w, _args()) is None
    monkeypatch.delenv("SVG_KERNEL")
    assert bench.captured_traffic(w, _args()) == c["bytes_per_head"] * w.heads
    # changed kernel sources: no figure
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: "0" * 16)
    assert bench.captured_traffic(w, _args()) is None


def test_both_arms_share_the_config_keys():
    w = syn.SPATIAL_75K
    a = bench.workload_config(w, _args(), "replicas x1", "no flush")
    b = bench.workload_config(w, _args(), "oracle on the host cores of rank 0 of 1", "n/a (host memory)")
    assert a.keys() == b.keys()
    assert {k: v for k, v in a.items() if k not in ("parallelism", "l2")} == \
        {k: v for k, v in b.items() if k not in ("parallelism", "l2")}
    assert a["workload"] == "spatial_75600" and a["tokens"] == 75600 and a["heads"] == 10
    assert a["routes"] == "S" * 10 and a["bq"] == 128 and a["bk"] == 128
