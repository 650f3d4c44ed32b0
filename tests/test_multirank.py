"""The benchmark's multi-rank timing on CPU with two gloo ranks: every rank
gets the max over ranks of the per-rank timings, and the whole-job value
counts the tokens of all ranks over the slowest rank's step time (weak
scaling, no data-path collective)."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 1.0 * (rank + 1)]
        got = bench.max_over_ranks(mine, torch.device("cpu"), world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        assert res[r] == [11.0, 5.0, 2.0]


def test_job_value_is_weak_scaling_throughput():
    # 2 ranks x 16384 tokens each, slowest step 4 ms
    assert bench.job_value(16384, 2, 4.0) == pytest.approx(2 * 16384 / 0.004)
    assert bench.max_over_ranks([1.0, 2.0], None, 1) == [1.0, 2.0]


def test_peak_follows_the_sampled_clocks():
    peaks = {"bf16_tflops": 1669.5, "bf16_tflops_sustained": 1411.1}
    # full clocks: the burst GEMM figure; power cap engaged: the sustained one
    assert bench.pick_bf16_peak(peaks, "measured", {"reasons": []})[0] == 1669.5
    p, src = bench.pick_bf16_peak(peaks, "measured", {"reasons": ["sw_power_cap"]})
    assert p == 1411.1 and "sustained" in src
    assert bench.pick_bf16_peak({"bf16_tflops": 1590.0}, "fallback", None)[0] == 1590.0
