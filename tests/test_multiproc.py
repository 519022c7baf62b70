"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The attention path has no exchange step, so several GPUs run independent replicas; the only
cross-rank logic is the timing reduction (max over ranks) and the work sum, and the reference
arm that only rank 0 runs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms, value = bench.aggregate_over_ranks(10.0 + 5.0 * rank, 1e12 * (rank + 1), world, torch.device("cpu"))
        out[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_aggregate_over_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # every rank sees the slowest rank's time and the sum of all ranks' work
    for r in range(world):
        ms, value = res[r]
        assert ms == 15.0
        assert value == pytest.approx(3e12 / 15e-3 / 1e12)


def test_aggregate_single_rank():
    import bench
    ms, value = bench.aggregate_over_ranks(4.0, 8e12, 1)
    assert ms == 4.0 and value == pytest.approx(2000.0)


def test_reference_arm_other_ranks_exit_without_work():
    import argparse
    import bench
    from block_sparse_spatio_flash_b200 import synthetic as syn
    args = argparse.Namespace(steps=1, warmup=3, ref_rows=4)
    assert bench.run_reference(args, syn.TINY, 2, 1) == 0
