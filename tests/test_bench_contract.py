"""Host-side parts of bench.py's JSON contract (CPU): the captured DRAM traffic is reported only for
the kernel sources, workload and launch shape it was captured on, and both arms print the same
`config` object."""
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


def test_both_arms_print_the_same_config():
    w = syn.SPATIAL_75K
    a = bench.workload_config(w, _args())
    b = bench.workload_config(w, _args())
    assert a == b
    assert "parallelism" not in a and "l2" not in a
    assert a["workload"] == "spatial_75600" and a["tokens"] == 75600 and a["heads"] == 10
    assert a["routes"] == "S" * 10 and a["bq"] == 128 and a["bk"] == 128


def test_reference_arm_line_carries_the_workload_config(capsys):
    """The reference arm's JSON line (rank 0, a tiny bounded sample) prints the same config object as
    the GPU arm builds for that workload, with the spread of the work outside it."""
    import json
    args = argparse.Namespace(steps=1, warmup=3, ref_rows=4, bq=64, bk=64, mode="split")
    assert bench.run_reference(args, syn.TINY, 1, 0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"] == bench.workload_config(syn.TINY, args)
    assert "parallelism" in line and "parallelism" not in line["config"]


def test_clock_sampler_writes_outside_the_repository(tmp_path):
    c = bench.ClockSampler(0)
    assert not c.path.startswith(bench.ROOT)
    c2 = bench.ClockSampler(0, str(tmp_path))
    assert c2.path.startswith(str(tmp_path))


def test_trace_stats_of_a_synthetic_trace():
    import torch
    # three CTAs: busy 4, 6 and 10 ms from a common start; a fourth entry never ran (zeros)
    t0 = 1_000_000_000
    tr = torch.tensor([[t0, t0 + 4_000_000, 3, 30], [t0, t0 + 6_000_000, 4, 40], [t0, t0 + 10_000_000, 5, 50],
                       [0, 0, 0, 0]], dtype=torch.int64)
    s = bench.trace_stats(tr)
    assert s["ctas"] == 3 and abs(s["span_ms"] - 10.0) < 1e-9
    assert abs(s["busy_max_ms"] - 10.0) < 1e-9 and abs(s["busy_mean_ms"] - 20.0 / 3) < 1e-9
    assert abs(s["tail_ms"] - 4.0) < 1e-9  # last end 10 ms, median end 6 ms
    assert abs(s["idle_frac"] - (1 - 20.0 / 30.0)) < 1e-9
    assert (s["tiles_max"], s["tiles_min"], s["items_max"], s["items_min"]) == (50, 30, 5, 3)
    assert bench.trace_stats(torch.zeros((2, 4), dtype=torch.int64)) is None
