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


def test_packed_phase2_inputs_alias_one_aligned_buffer():
    from block_sparse_long_rope_b200.configs import Workload
    from block_sparse_long_rope_b200.pipeline import phase2_calls

    w = Workload(index=70, name="pack-test", B=2, Hq=8, Hkv=2, D=64, theta=1e4, L=512,
                 block_len=128, anchor_len=128, Tq=5, Tdec=3)
    g = torch.Generator().manual_seed(5)
    new = [torch.randn(w.B, w.Tq + w.Tdec, h, w.D, generator=g).to(torch.bfloat16)
           for h in (w.Hq, w.Hkv, w.Hkv)]
    calls = phase2_calls(w, *new)
    buf, packed = bench.pack_calls(calls)
    assert buf.numel() == sum(x.numel() for c in calls for x in c[:3])
    base = buf.data_ptr()
    for pc, c in zip(packed, calls):
        assert pc[3] == c[3]
        for v, x in zip(pc[:3], c[:3]):
            assert v.shape == x.shape and v.is_contiguous()
            assert base <= v.data_ptr() < base + buf.numel() * 2
            assert (v.data_ptr() - base) % 16 == 0
            v.copy_(x)
    # one copy of the buffer carries every call's inputs
    buf2 = buf.clone()
    off = 0
    for c in calls:
        for x in c[:3]:
            assert torch.equal(buf2[off:off + x.numel()].view(x.shape), x)
            off += x.numel()


def test_host_cpu_reports_model_and_cores():
    info = bench.host_cpu()
    assert info["host_cores"] == os.cpu_count()
    assert isinstance(info["cpu_model"], str) and info["cpu_model"]


def test_multi_gpu_runs_default_to_the_sharded_deployment():
    # one GPU: a single replica; several: one sequence's blocks over the ranks
    assert bench.resolve_mode(None, 1) == "replicas"
    assert bench.resolve_mode(None, 2) == "sharded"
    assert bench.resolve_mode(None, 8) == "sharded"
    assert bench.resolve_mode("replicas", 8) == "replicas"
    assert bench.resolve_mode("sharded", 1) == "sharded"


def test_code_digest_ignores_comments_and_layout(tmp_path, monkeypatch):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    a.write_text("int f(int x) {\n  return x + 1;  // one more\n}\n/* block\ncomment */\n")
    b.write_text("int f(int x){return x+1;}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.code_digest(["a.cu"]) == bench.code_digest(["b.cu"])
    b.write_text("int f(int x){return x+2;}\n")
    assert bench.code_digest(["a.cu"]) != bench.code_digest(["b.cu"])


def test_committed_phase1_traffic_records_match_the_kernel_sources():
    """The bench line's roofline `traffic` comes from an ncu capture recorded
    under profiles/; it is reported only while the kernel sources are the
    ones captured (comments aside)."""
    for wl in ("llama8b-1m", "llama8b-16k"):
        t = bench.phase1_traffic(wl)
        assert isinstance(t, int) and t > 0, wl
