"""bench.py host logic (CPU only): flop counts, multi-rank combination over gloo
(world size 2), per-rank inputs for weak scaling, and the reference arm's
rank-0-only rule."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

import bench


def test_flop_convention():
    f, b = bench.flops(1, 16, 32768, 128, True)
    assert f == 4.0 * 16 * 32768 ** 2 * 128 / 2 and b == 2.5 * f
    f2, _ = bench.flops(2, 3, 100, 64, False)
    assert f2 == 4.0 * 6 * 100 ** 2 * 64


def test_job_tflops_is_weak_scaling():
    per_rank = 1.5e13
    assert abs(bench.job_tflops(per_rank, 1, 15.0) - 1000.0) < 1e-9
    # twice the ranks, same slowest time: twice the job throughput
    assert abs(bench.job_tflops(per_rank, 2, 15.0) - 2000.0) < 1e-9


def test_rank_seeds_differ():
    seeds = {bench.rank_seed(4, r) for r in range(8)}
    assert len(seeds) == 8


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank]
        out[rank] = bench.max_over_ranks(mine, world, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    port = 29500 + (os.getpid() % 1000)
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        assert out[0] == [11.0, 5.0] and out[1] == [11.0, 5.0]


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(type("A", (), {"steps": 2, "warmup": 3})())
    assert buf.getvalue() == ""


def test_traffic_lookup_tracks_kernel_sources(monkeypatch):
    real = bench.stored_traffic("bwd")
    if real is not None:
        monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 64)
        assert bench.stored_traffic("bwd") is None
