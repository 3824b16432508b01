"""The benchmark's multi-rank logic on CPU: two gloo ranks (no GPU).

bench.py runs one replica of the workload per GPU (the path shards by
(batch, head) with no exchange), reduces the per-rank device times with a
MAX, and reports the whole-job throughput world * flops / max time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 3.0 - rank]            # per-rank (timed ms, e2e ms)
        out[rank] = bench.max_over_ranks(mine, world, device=None)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == [11.0, 3.0] and out[1] == [11.0, 3.0]


def test_aggregate_is_weak_scaling():
    # 2 ranks, 1 TFLOP per rank per step, slowest rank 10 steps in 20 ms -> 1000 TFLOP/s
    assert bench.aggregate_tflops(1e12, 20.0, 10, 2) == pytest.approx(1000.0)
    assert bench.aggregate_tflops(1e12, 20.0, 10, 1) == pytest.approx(500.0)


def test_reference_arm_only_rank0():
    class A:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(A, bench.ALL["tiny"], rank=1) is None


def test_flop_and_byte_counts():
    w = bench.ALL["wan5b"]
    c = bench.tile_counts(w)
    assert c.size == 120 and c.sum() == w.N
    nT = c.size
    all_idx = torch.arange(nT).repeat(w.B, w.H, nT, 1).numpy()
    # every tile kept: the exact count is dense attention's 4 * d * N^2 per head
    assert bench.exact_flops(all_idx, w) == 4 * w.d * w.N * w.N * w.B * w.H
    assert bench.nominal_flops(w) == 4 * w.B * w.H * w.N * w.topk * 256 * w.d
    assert bench.select_bytes(w) == 2 * w.B * w.H * w.N * w.d * 2 + w.B * w.H * nT * w.topk * 4
