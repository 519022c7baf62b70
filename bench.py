"""Benchmark of the block-sparse spatio-temporal attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload spatial_75600|temporal_75600|mixed_75600|p1440_302400]
                    [--bq 128 --bk 128] [--mode split|naive] [--fused] [--no-extras]

A step is one call of svg_attention_fwd (split mode: full tiles unmasked, boundary tiles
masked) over the whole workload, Q/K/V/O resident in HBM (774 MB at 75,600 tokens, larger
than the 126 MB L2, so no flush is needed between steps). With --fused a step is one call of
svg_attention_fwd_fused on original-order tensors instead (temporal heads' token permutation
inside the kernel). Tile maps are built once per
geometry (the design caches them) and timed separately, as are the token permutation, the
dense baseline, the naive and the rounded modes. Multi-GPU runs are independent replicas
(the path has no exchange step): every rank runs the same workload; the step time is the
max over ranks and `value` sums the work of all ranks.

Rank 0 prints one JSON line. `--impl reference` times the fp64 CPU oracle instead (rank 0
only, bounded row sample per step, full-call time extrapolated by rows).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_spatio_flash_b200 import synthetic as syn  # noqa: E402

METRIC = "ms/call & effective TFLOP/s, 75,600-tok 10-head d128 bf16 sparse attention"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, log_dir: str = ""):
        import tempfile
        self.dev = device_index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(), f"svg_bench_clocks_rank{device_index}.csv")

    def __enter__(self):
        try:
            if os.path.dirname(self.path):
                os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


def aggregate_over_ranks(local_ms: float, local_flop: float, world: int, device=None):
    """Step time of the job = max over ranks (device-timed); value = all ranks' FLOP over it.

    Every rank calls this at the same point (it is a collective when world > 1)."""
    ms = float(local_ms)
    flop = float(local_flop)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms, flop], dtype=torch.float64, device=device)
        tmax = t[:1].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        tsum = t[1:].clone()
        dist.all_reduce(tsum, op=dist.ReduceOp.SUM)
        ms, flop = float(tmax.item()), float(tsum.item())
    return ms, flop / (ms * 1e-3) / 1e12


def time_events(fn, iters, stream):
    """Mean ms per call over `iters` calls, CUDA events on the launching stream."""
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(iters):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / iters


def time_interleaved(fns, iters, rounds, stream):
    """Median over `rounds` of the mean ms per call over `iters` calls, for each callable of `fns`
    (a dict), after one untimed call each; the callables take turns within every round, so that
    clock and power changes during the measurement fall on all of them alike."""
    for fn in fns.values():
        fn()
    times = {k: [] for k in fns}
    for _ in range(rounds):
        for k, fn in fns.items():
            times[k].append(time_events(fn, iters, stream))
    return {k: statistics.median(v) for k, v in times.items()}


def workload_flops(w, summaries):
    """(effective, visited, executed) FLOP per call: 4*d*pairs; retained / in-range visited area /
    MMA work actually issued (128-row halves x bk key tiles)."""
    eff = vis = exe = 0
    for r in w.routes:
        s = summaries[r]
        eff += 4 * w.d * s.retained_map
        vis += 4 * w.d * s.visited_area
        exe += 4 * w.d * s.pair_half_tiles * 128 * w.bk
    return eff, vis, exe


def oracle_sample(w, q, k, v, rows_per_head):
    """Time the fp64 oracle on a seeded row sample of every head; return (seconds, rows, threads)."""
    import oracle
    t0 = time.perf_counter()
    nrows = 0
    for h in range(w.heads):
        rows = syn.sample_rows(w.replace(sample_rows=rows_per_head), h).numpy()
        rows = rows[:rows_per_head]
        oracle.attention_rows(q[h], k[h], v[h], rows, route=w.routes[h], layout=w.layout, T=w.frames,
                              S=w.frame_size, frame_window=w.frame_window, band=w.spatial_band, F0=w.sink_frames)
        nrows += len(rows)
    return time.perf_counter() - t0, nrows, oracle.num_threads()


def oracle_full_call_seconds(w, sec, nrows, fixed):
    """Full-call oracle time from a row sample: the once-per-head part (widening K and V to fp64,
    measured with one row per head) plus the per-row part of the sample scaled to every row."""
    per_row = max(sec - fixed, 0.0) / nrows
    return fixed + per_row * (w.tokens * w.heads)


def closed_form_effective_flops(w):
    """4*d*retained for the exact masks, from the oracle's closed-form-pinned brute force is
    too slow here; the tile-map summary gives the same number on the GPU path. For the CPU
    arm the retained count is computed by the oracle once (exact)."""
    import oracle
    tot = 0
    for r in set(w.routes):
        n = oracle.retained_pairs(r, w.frames, w.frame_size, w.frame_window, w.spatial_band, w.sink_frames)
        tot += n * sum(1 for x in w.routes if x == r)
    return 4 * w.d * tot


def workload_config(w, args):
    """The `config` object of both arms' JSON lines: the workload and the launch shape only, so that
    the two arms print identical objects; how the work is spread and the cache policy are top-level
    keys of the line."""
    return {"workload": w.name, "tokens": w.tokens, "heads": w.heads, "d": w.d,
            "routes": "".join("S" if r == 0 else "T" for r in w.routes),
            "frame_window": w.frame_window, "spatial_band": w.spatial_band, "sink_frames": w.sink_frames,
            "bq": w.bq, "bk": w.bk, "mode": args.mode,
            **({"token_order": "fused"} if getattr(args, "fused", False) else {})}


def run_reference(args, w, world, rank):
    if rank != 0:
        return 0
    q, k, v = syn.make_qkv(w)
    eff = closed_form_effective_flops(w)
    rows = args.ref_rows
    for _ in range(args.warmup if args.warmup < 1 else 1):
        oracle_sample(w, q, k, v, max(4, rows // 8))
    fixed, _, _ = oracle_sample(w, q, k, v, 1)  # the once-per-head part of a call
    times = []
    nthreads = 1
    for _ in range(args.steps):
        sec, nrows, nthreads = oracle_sample(w, q, k, v, rows)
        times.append(oracle_full_call_seconds(w, sec, nrows, fixed))
    t = statistics.mean(times)
    value = eff / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "parallelism": f"oracle on the host cores of rank 0 of {world}", "l2": "n/a (host memory)",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{rows} seeded query rows per head x {w.heads} heads per step; full-call time = "
                                   f"once-per-head part ({fixed:.2f} s, timed with one row per head) + per-row "
                                   f"part scaled to all rows"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=syn.SPATIAL_75K.name)
    ap.add_argument("--bq", type=int, default=128)
    ap.add_argument("--bk", type=int, default=128)
    ap.add_argument("--mode", default="split", choices=["split", "naive"])
    ap.add_argument("--fused", action="store_true",
                    help="time svg_attention_fwd_fused (token permutation inside the kernel) as the step")
    ap.add_argument("--chunk-heads", type=int, default=1, help="heads per chunk of the host-buffer pipeline")
    ap.add_argument("--no-extras", action="store_true", help="skip the side measurements")
    ap.add_argument("--quick", action="store_true",
                    help="only the timed steps (no side measurements, e2e or CPU baseline): for profiler runs")
    ap.add_argument("--heads", type=int, default=0, help="use only the first H heads of the workload")
    ap.add_argument("--shard-heads", action="store_true",
                    help="split one call's heads over the ranks (strong scaling) instead of running replicas")
    ap.add_argument("--cpu-rows", type=int, default=3072,
                    help="oracle rows per head for cpu_baseline (about 10 s of host work at the pages' shape)")
    ap.add_argument("--ref-rows", type=int, default=96, help="oracle rows per head per --impl reference step")
    ap.add_argument("--route-calls", type=int, default=0,
                    help="after the timed region, this many svg_route_heads calls (64 sampled rows per head) on the "
                         "workload, untimed: a fixed launch sequence for profiling the route kernel")
    ap.add_argument("--clock-log-dir", default="",
                    help="folder for the nvidia-smi clock samples of the timed region (default: the temp folder)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_env()
    w = syn.WORKLOADS[args.workload].replace(bq=args.bq, bk=args.bk)
    if args.heads > 0:
        w = w.replace(routes=w.routes[: args.heads])

    if args.impl == "reference":
        return run_reference(args, w, world, rank)

    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    from block_sparse_spatio_flash_b200 import svg as S

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    P, peak_kind = peaks()
    g = S.make_geom(w.frames, w.grid_h, w.grid_w)
    m = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, w.variant, w.layout)
    t = S.make_tile(w.bq, w.bk)
    routes = list(w.routes)
    mode = S.SVG_MODE_SPLIT if args.mode == "split" else S.SVG_MODE_NAIVE

    q_cpu, k_cpu, v_cpu = syn.make_qkv(w)
    ws = [None, None]
    summ = [None, None]
    for c in sorted(set(routes)):
        ws[c] = S.alloc_workspace(g, t, dev)
        S.svg_build_tilemap(g, m, t, c, ws[c])
        summ[c] = S.svg_tilemap_summary(ws[c])
    plan = None
    if args.shard_heads:
        # one call's heads split over the ranks by tile-map work; each rank keeps only its heads
        from block_sparse_spatio_flash_b200 import shard
        if world > w.heads:
            raise SystemExit(f"--shard-heads needs at least one head per rank ({w.heads} heads, {world} ranks)")
        plan = shard.plan_heads(shard.head_costs(routes, summ), world)
        q_cpu, k_cpu, v_cpu = (shard.local_heads(x, plan, rank) for x in (q_cpu, k_cpu, v_cpu))
        w = w.replace(routes=tuple(shard.local_routes(plan, rank, routes)))
        routes = list(w.routes)
    q, k, v = (x.to(dev) for x in (q_cpu, k_cpu, v_cpu))
    if any(routes):  # temporal heads run in their own token order (permutation timed separately)
        qp, kp, vp = (torch.empty_like(x) for x in (q, k, v))
        for a, b_ in ((q, qp), (k, kp), (v, vp)):
            S.svg_permute(a, b_, routes, g, m)
    else:
        qp, kp, vp = q, k, v
    o = torch.empty_like(qp)
    scratch = S.alloc_scratch(dev)
    eff_flop, vis_flop, exe_flop = workload_flops(w, summ)
    o_all = None
    if plan is not None and world > 1:
        o_all = torch.empty((plan.heads,) + tuple(o.shape[1:]), dtype=o.dtype, device=dev)

    o_orig = torch.empty_like(q) if args.fused else None

    def step():
        if args.fused:
            S.svg_attention_fwd_fused(q, k, v, o_orig, routes, ws[0], ws[1], g, m, t, mode=mode, scratch=scratch)
        else:
            S.svg_attention_fwd(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, mode=mode, scratch=scratch)
        if o_all is not None:  # every rank ends the step with all heads' O
            shard.gather_heads(o_orig if args.fused else o, plan, out=o_all)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = S.svg_read_status(scratch)
    if status != 0:
        raise RuntimeError(f"device status {status}: {S.svg_error_string(status)}")

    # ---------------------------------------------------------------- timed region
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local, args.clock_log_dir) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    ms, value = aggregate_over_ranks(ev[0].elapsed_time(ev[-1]) / args.steps, eff_flop, world, dev)
    status = S.svg_read_status(scratch)
    if status != 0:
        raise RuntimeError(f"device status {status}: {S.svg_error_string(status)}")
    clocks = clk.summary()

    # ---------------------------------------------------------------- roofline of the attention kernel
    peak = float(P["bf16_tflops"])
    achieved = vis_flop / (statistics.mean(per_step) * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": captured_traffic(w, args),
                "kernel": f"attn_kernel<{w.d},{args.bk}> ({args.mode}{', fused token order' if args.fused else ''}, "
                          f"{kernel_variant()} schedule)",
                "flop_definition": "4*d*(in-range area of visited tiles)", "peak_kind": f"{peak_kind} bf16 burst"}

    if args.route_calls > 0:
        rrows = torch.as_tensor(syn.sample_rows(w.replace(sample_rows=64), 0)[:64].numpy(), dtype=torch.int32,
                                device=dev)
        rt = torch.empty(w.heads, dtype=torch.uint8, device=dev)
        rwork = torch.empty(S.svg_route_work_bytes(w.heads, w.tokens, w.d, rrows.numel()), dtype=torch.uint8,
                            device=dev)
        for _ in range(args.route_calls):
            S.svg_route_heads(q, k, v, g, m, rrows, rt, work=rwork)
        torch.cuda.synchronize()
        if S.svg_read_status(rwork) != 0:
            raise RuntimeError("route kernel status")

    extras = {}
    if not (args.no_extras or args.quick):
        extras = side_measurements(S, w, g, m, t, routes, q, k, v, qp, kp, vp, o, scratch, ws, summ, P, stream,
                                   dev)

    # ---------------------------------------------------------------- end to end through host buffers
    e2e = None
    if not args.quick:
        e2e = end_to_end(S, w, g, m, t, routes, q_cpu, k_cpu, v_cpu, ws, scratch, mode, eff_flop, world, dev, stream,
                         args, attn_ms=statistics.mean(per_step))

    cpu = None
    if rank == 0 and world == 1 and not args.quick:
        fixed, _, _ = oracle_sample(w, q_cpu, k_cpu, v_cpu, 1)
        sec, nrows, nthreads = oracle_sample(w, q_cpu, k_cpu, v_cpu, args.cpu_rows)
        full = oracle_full_call_seconds(w, sec, nrows, fixed)
        cpu = {"value": eff_flop / full / 1e12, "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
               "sample": f"{args.cpu_rows} seeded query rows per head x {w.heads} heads ({nrows} rows, "
                         f"{sec:.1f} s); full-call time = once-per-head part ({fixed:.2f} s, one row per head) "
                         f"+ per-row part scaled to all rows = {full:.1f} s",
               "ms_per_call_extrapolated": full * 1e3}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong" if plan is not None else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, args),
            "parallelism": f"heads x{world} (all-gather of O in the step)" if plan is not None else f"replicas x{world}",
            "l2": "no flush: Q/K/V/O = %.0f MB > 126 MB L2" % (4 * w.heads * w.tokens * w.d * 2 / 1e6),
            "ms_per_call": ms,
            "effective_flop_per_call": eff_flop, "visited_flop_per_call": vis_flop, "executed_flop_per_call": exe_flop,
            "visited_tflops": vis_flop / (ms * 1e-3) / 1e12,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
            "clocks": clocks, "extras": extras,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


# DRAM bytes (read + write) of one attention launch from an ncu capture of the 2-head slice of
# spatial_75600 (128 x 128 tiles, split mode), scaled to the launch's heads: traffic grows with the
# heads processed. Valid only for the kernel sources that were captured (their SHA-256 prefix);
# after any change to them the field is null until the capture is repeated.
CAPTURED_TRAFFIC = {"sources_sha256": "04b08fa2470c36ca", "bytes_per_head": 145.666304e6 / 2,
                    "workload": "spatial_75600", "bq": 128, "bk": 128, "mode": "split"}


def kernel_sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_spatio_flash_b200", "csrc")
    for name in ("svg_attention.cu", "svg_common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_variant() -> str:
    """The attention kernel the library runs: its default, or the option named by SVG_KERNEL."""
    return os.environ.get("SVG_KERNEL", "") or "default"


def captured_traffic(w, args):
    c = CAPTURED_TRAFFIC
    if (kernel_sources_sha() != c["sources_sha256"] or w.name != c["workload"] or args.bq != c["bq"]
            or args.bk != c["bk"] or args.mode != c["mode"] or kernel_variant() != "default"
            or getattr(args, "fused", False)):
        return None
    return c["bytes_per_head"] * w.heads


def side_measurements(S, w, g, m, t, routes, q, k, v, qp, kp, vp, o, scratch, ws, summ, P, stream, dev):
    out = {}
    iters = 10
    hbm = float(P["hbm_gbs"])
    # tile-map build (integer, once per geometry)
    ms = time_events(lambda: [S.svg_build_tilemap(g, m, t, c, ws[c]) for c in sorted(set(routes))], 5, stream)
    out["tilemap_build_ms"] = ms
    # permutation, one [H, N, d] tensor (temporal heads reordered, spatial heads copied)
    tmp = torch.empty_like(q)
    ms = time_events(lambda: S.svg_permute(q, tmp, routes, g, m), iters, stream)
    nbytes = 2 * q.numel() * 2
    out["permute_ms_per_tensor"] = ms
    out["permute_gbs"] = nbytes / (ms * 1e-3) / 1e9
    out["permute_hbm_frac"] = out["permute_gbs"] / hbm
    # the ablation: dense baseline (same kernel, every tile full), naive mode (every visited tile
    # masked), split mode, QK^T on the 8-bit path (e4m3 copies of the permuted Q and K: an opt-in
    # variant, not the headline) and the rounded (tile-aligned) masks, taking turns after one
    # untimed call each, so that the ratios compare like with like
    mr = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, S.SVG_MASK_ROUNDED, w.layout)
    wr = [None, None]
    rs = {}
    for c in sorted(set(routes)):
        wr[c] = S.alloc_workspace(g, t, dev)
        S.svg_build_tilemap(g, mr, t, c, wr[c])
        rs[c] = S.svg_tilemap_summary(wr[c])
    q8, k8 = qp.to(torch.float8_e4m3fn), kp.to(torch.float8_e4m3fn)
    tm = time_interleaved({
        "dense": lambda: S.svg_dense_attention_fwd(qp, kp, vp, o, bk=t.bk, scratch=scratch),
        "naive": lambda: S.svg_attention_fwd(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, mode=S.SVG_MODE_NAIVE,
                                             scratch=scratch),
        "split": lambda: S.svg_attention_fwd(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, mode=S.SVG_MODE_SPLIT,
                                             scratch=scratch),
        "qk8": lambda: S.svg_attention_fwd_qk8(q8, k8, vp, o, routes, ws[0], ws[1], g, m, t, scratch=scratch),
        "rounded": lambda: S.svg_attention_fwd(qp, kp, vp, o, routes, wr[0], wr[1], g, mr, t, scratch=scratch),
    }, 2, 3, stream)
    del q8, k8
    dense_flop = 4 * w.d * w.tokens * w.tokens * w.heads
    out["dense_ms"] = tm["dense"]
    out["dense_tflops"] = dense_flop / (tm["dense"] * 1e-3) / 1e12
    out["naive_ms"] = tm["naive"]
    out["split_ms"] = tm["split"]
    out["split_vs_dense"] = tm["dense"] / tm["split"]
    out["qk8_ms"] = tm["qk8"]
    out["qk8_vs_split"] = tm["split"] / tm["qk8"]
    out["rounded_ms"] = tm["rounded"]
    for name, sm in (("exact", summ), ("rounded", rs)):
        tot_tiles = sum(sm[c].n_full + sm[c].n_boundary + sm[c].n_empty for c in sorted(set(routes)))
        vis = sum(sm[c].n_full + sm[c].n_boundary for c in sorted(set(routes)))
        bnd = sum(sm[c].n_boundary for c in sorted(set(routes)))
        kept = sum(sm[c].retained_map * sum(1 for r in routes if r == c) for c in sorted(set(routes)))
        out[f"{name}_boundary_frac_of_visited"] = bnd / max(vis, 1)
        out[f"{name}_visited_frac_of_all"] = vis / max(tot_tiles, 1)
        out[f"{name}_retained_frac"] = kept / (w.heads * w.tokens ** 2)
    # head routing from 64 sampled query rows per head (original order, dense + both sparse masks)
    rows = torch.as_tensor(syn.sample_rows(w.replace(sample_rows=64), 0)[:64].numpy(), dtype=torch.int32,
                           device=dev)
    rt = torch.empty(w.heads, dtype=torch.uint8, device=dev)
    work = torch.empty(S.svg_route_work_bytes(w.heads, w.tokens, w.d, rows.numel()), dtype=torch.uint8, device=dev)
    S.svg_route_heads(q, k, v, g, m, rows, rt, work=work)  # untimed first call (module load)
    out["route_ms"] = time_events(lambda: S.svg_route_heads(q, k, v, g, m, rows, rt, work=work), 10, stream)
    out["route_rows_per_head"] = int(rows.numel())
    rows256 = torch.as_tensor(syn.sample_rows(w.replace(sample_rows=256), 0)[:256].numpy(), dtype=torch.int32,
                              device=dev)
    work256 = torch.empty(S.svg_route_work_bytes(w.heads, w.tokens, w.d, rows256.numel()), dtype=torch.uint8,
                          device=dev)
    S.svg_route_heads(q, k, v, g, m, rows256, rt, work=work256)
    out["route_ms_256_rows"] = time_events(lambda: S.svg_route_heads(q, k, v, g, m, rows256, rt, work=work256), 10,
                                           stream)
    out["route_status"] = S.svg_read_status(work256)
    del work256
    out["scheduler"] = scheduler_compare(S, w, qp, kp, vp, o, routes, ws, g, m, t, scratch, stream, dev)
    out["workloads"] = other_workloads(S, P, stream, dev)
    out["tile_sweep_mixed_75600"] = tile_sweep(S, stream, dev)
    st = S.svg_read_status(scratch)
    out["status"] = st
    return out


def tile_sweep(S, stream, dev):
    """mixed_75600 (5 spatial + 5 temporal heads) over query tiles {128, 256, 512} x key tiles
    {64, 128}, exact and rounded masks: boundary-tile share of the visited tiles, visited share of
    all tiles, kept-pair share, and the attention time."""
    w = syn.MIXED_75K
    routes = list(w.routes)
    g = S.make_geom(w.frames, w.grid_h, w.grid_w)
    q, k, v = (x.to(dev) for x in syn.make_qkv(w))
    qp, kp, vp = (torch.empty_like(q) for _ in range(3))
    m0 = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, S.SVG_MASK_EXACT, w.layout)
    for a, b in ((q, qp), (k, kp), (v, vp)):
        S.svg_permute(a, b, routes, g, m0)
    del q, k, v
    o = torch.empty_like(qp)
    sc = S.alloc_scratch(dev)
    res = {}
    for bq, bk in syn.TILE_SWEEP:
        t = S.make_tile(bq, bk)
        for var, name in ((S.SVG_MASK_EXACT, "exact"), (S.SVG_MASK_ROUNDED, "rounded")):
            m = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, var, w.layout)
            ws, sm = [None, None], {}
            for c in (0, 1):
                ws[c] = S.alloc_workspace(g, t, dev)
                S.svg_build_tilemap(g, m, t, c, ws[c])
                sm[c] = S.svg_tilemap_summary(ws[c])
            ms = time_events(lambda: S.svg_attention_fwd(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, scratch=sc),
                             3, stream)
            vis = sum(sm[c].n_full + sm[c].n_boundary for c in (0, 1))
            tot = sum(sm[c].n_full + sm[c].n_boundary + sm[c].n_empty for c in (0, 1))
            kept = sum(sm[c].retained_map * routes.count(c) for c in (0, 1))
            res[f"{bq}x{bk}-{name}"] = {"ms": ms, "boundary_frac_of_visited": sum(sm[c].n_boundary for c in (0, 1)) / vis,
                                        "visited_frac_of_all": vis / tot,
                                        "retained_frac": kept / (w.heads * w.tokens ** 2)}
            del ws
    res["status"] = S.svg_read_status(sc)
    return res


def trace_stats(tr):
    """Balance of one traced launch from its per-CTA records (start ns, end ns, items, half-tiles):
    span of the launch, busy time per CTA (start to end of the CTA), the tail (last CTA end minus the
    median CTA end) and the spread of the work the CTAs took."""
    t = tr[tr[:, 0] > 0].to(torch.float64)
    if t.numel() == 0:
        return None
    start, end = t[:, 0], t[:, 1]
    busy = (end - start) / 1e6
    span = float(end.max() - start.min()) / 1e6
    return {"ctas": int(t.shape[0]), "span_ms": span, "busy_max_ms": float(busy.max()),
            "busy_mean_ms": float(busy.mean()), "busy_min_ms": float(busy.min()),
            "tail_ms": float(end.max() - end.median()) / 1e6,
            "idle_frac": 1.0 - float(busy.sum()) / (t.shape[0] * span) if span > 0 else 0.0,
            "tiles_max": int(t[:, 3].max()), "tiles_mean": float(t[:, 3].mean()), "tiles_min": int(t[:, 3].min()),
            "items_max": int(t[:, 2].max()), "items_min": int(t[:, 2].min())}


def scheduler_compare(S, w, qp, kp, vp, o, routes, ws, g, m, t, sc, stream, dev, iters=5):
    """Both scheduling orders of the persistent kernel on one workload: ms per call (untraced) and the
    per-CTA balance of one traced call each."""
    n = torch.cuda.get_device_properties(dev).multi_processor_count
    tr = torch.zeros((n, 4), dtype=torch.int64, device=dev)
    out = {}
    for name, order in (("head_major", S.SVG_ORDER_HEAD_MAJOR), ("work", S.SVG_ORDER_WORK)):
        ms = time_events(lambda: S.svg_attention_fwd_ex(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, scratch=sc,
                                                        order=order), iters, stream)
        S.svg_attention_fwd_ex(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, scratch=sc, order=order, cta_trace=tr)
        torch.cuda.synchronize()
        out[name] = {"ms": ms, "trace": trace_stats(tr.cpu())}
    return out


def other_workloads(S, P, stream, dev):
    """Attention time (split mode, permuted inputs, 128 x 128 tiles) of the other workloads of the
    pages' shapes: all-temporal heads at 75,600 tokens (sink-prefix and fully space-major token
    orders), mixed heads at 75,600 tokens, mixed heads at 302,400 (1440p);
    next to it the fused-order call (svg_attention_fwd_fused on original-order tensors) and the
    permuted path with its four permutation passes."""
    res = {}
    temporal_fsm = syn.TEMPORAL_75K.replace(name="temporal_75600_full_space_major", layout=syn.LAYOUT_FULL_SPACE_MAJOR)
    for w in (syn.TEMPORAL_75K, temporal_fsm, syn.MIXED_75K, syn.P1440):
        g = S.make_geom(w.frames, w.grid_h, w.grid_w)
        m = S.make_mask(w.frame_window, w.spatial_band, w.sink_frames, w.variant, w.layout)
        t = S.make_tile(w.bq, w.bk)
        routes = list(w.routes)
        q, k, v = (x.to(dev) for x in syn.make_qkv(w))
        qp, kp, vp = (torch.empty_like(q) for _ in range(3))
        for a, b in ((q, qp), (k, kp), (v, vp)):
            S.svg_permute(a, b, routes, g, m)
        o = torch.empty_like(qp)
        ws, summ = [None, None], {}
        for c in sorted(set(routes)):
            ws[c] = S.alloc_workspace(g, t, dev)
            S.svg_build_tilemap(g, m, t, c, ws[c])
            summ[c] = S.svg_tilemap_summary(ws[c])
        sc = S.alloc_scratch(dev)
        # the permuted layout's attention, the same call with the permutation inside the kernel
        # (original-order tensors) and one permutation pass, taking turns
        tm = time_interleaved({
            "attn": lambda: S.svg_attention_fwd(qp, kp, vp, o, routes, ws[0], ws[1], g, m, t, scratch=sc),
            "fused": lambda: S.svg_attention_fwd_fused(q, k, v, o, routes, ws[0], ws[1], g, m, t, scratch=sc),
            "perm": lambda: S.svg_permute(q, qp, routes, g, m)}, 2, 3, stream)
        ms, ms_fused, ms_perm = tm["attn"], tm["fused"], tm["perm"]
        eff, vis, _ = workload_flops(w, summ)
        res[w.name] = {"ms": ms, "effective_tflops": eff / (ms * 1e-3) / 1e12,
                       "visited_tflops": vis / (ms * 1e-3) / 1e12,
                       "visited_frac_of_peak": vis / (ms * 1e-3) / 1e12 / float(P["bf16_tflops"]),
                       "fused_order_ms": ms_fused, "permuted_path_ms": ms + 4 * ms_perm,
                       "scheduler": scheduler_compare(S, w, qp, kp, vp, o, routes, ws, g, m, t, sc, stream, dev),
                       "status": S.svg_read_status(sc)}
        del q, k, v, qp, kp, vp, o, ws
        torch.cuda.empty_cache()
    return res


def end_to_end(S, w, g, m, t, routes, q_cpu, k_cpu, v_cpu, ws, scratch, mode, eff_flop, world, dev, stream, args,
               attn_ms=None):
    """Same metric through the public C-ABI call on host buffers (svg_attention_fwd_host): every
    step copies Q/K/V in from pinned host memory, permutes temporal heads, runs the attention,
    permutes O back and copies it out, in chunks of heads whose copies overlap the neighbouring
    chunks' compute. The call is synchronous, so a step is timed on the host clock between two
    device synchronisations."""
    qh, kh, vh = (x.contiguous().pin_memory() for x in (q_cpu, k_cpu, v_cpu))
    oh = torch.empty_like(q_cpu).pin_memory()
    ch = max(1, min(args.chunk_heads, w.heads))
    buf = torch.empty(S.svg_attention_host_buffer_bytes(w.tokens, w.d, ch), dtype=torch.uint8, device=dev)

    def e2e_step():
        S.svg_attention_fwd_host(qh, kh, vh, oh, routes, ws[0], ws[1], g, m, t, buf, chunk_heads=ch, mode=mode)

    for _ in range(2):
        e2e_step()
    n = max(3, min(20, args.steps // 5))
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(n):
        e2e_step()
    torch.cuda.synchronize()
    ms_local = (time.perf_counter() - t0) * 1e3 / n
    ms, value = aggregate_over_ranks(ms_local, eff_flop, world, dev)
    h2d = 3 * q_cpu.numel() * 2
    d2h = q_cpu.numel() * 2
    out = {"value": value, "unit": "TFLOP/s", "ms_per_step": ms, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": n, "call": "svg_attention_fwd_host", "chunk_heads": ch,
           "clock": "host, between device synchronisations"}
    # the copies alone, one direction at a time (pinned host memory, one copy per tensor): the pipeline
    # cannot beat all of H2D plus the last chunk's attention and D2H
    dq = [torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (qh, kh, vh)]
    h2d_ms = time_events(lambda: [d.copy_(x, non_blocking=True) for d, x in zip(dq, (qh, kh, vh))], 3, stream)
    d2h_ms = time_events(lambda: oh.copy_(dq[0], non_blocking=True), 3, stream)
    out.update(h2d_ms=h2d_ms, h2d_gbs=h2d / h2d_ms / 1e6, d2h_ms=d2h_ms, d2h_gbs=d2h / d2h_ms / 1e6)
    # both directions at once, as in the pipeline: all inputs in on one stream while as many bytes as the
    # outputs go out on another; the link is shared, so this time bounds the pipeline too
    side = torch.cuda.Stream(device=dev)
    ev0, ev1, ev2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    torch.cuda.synchronize()
    ev0.record(stream)
    side.wait_event(ev0)
    with torch.cuda.stream(side):
        oh.copy_(dq[0], non_blocking=True)
        ev2.record(side)
    for d_, x in zip(dq, (qh, kh, vh)):
        d_.copy_(x, non_blocking=True)
    stream.wait_event(ev2)
    ev1.record(stream)
    torch.cuda.synchronize()
    duplex_ms = ev0.elapsed_time(ev1)
    out.update(duplex_ms=duplex_ms, duplex_gbs=(h2d + d2h) / duplex_ms / 1e6)
    if attn_ms is not None:
        chunks = -(-w.heads // ch)
        bound = max(h2d_ms + (attn_ms + d2h_ms) / chunks, duplex_ms)
        out.update(copy_bound_ms=bound, frac_of_copy_bound=bound / ms)
    del dq
    return out


if __name__ == "__main__":
    sys.exit(main())
