"""Benchmark of the Star Attention hot path on B200 (one attention layer).

A step is one pass of the whole hot path over one batch of synthetic input:
RoPE + Phase-1 anchor-block encoding of the context, the Phase-2 query chunk
(partials + LSE merge), then every single-token decode step (partials + LSE
merge). Inputs are resident in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl star|reference]

One JSON line on stdout (rank 0). With N > 1 (torchrun, one rank per GPU)
each rank runs its own independent sequences (weak scaling, no data-path
collective); the time is the max over ranks.

--mode sharded spreads ONE sequence's blocks over the N ranks instead (the
pages' multi-host form: Phase 1 per shard, Phase 2 with a query broadcast, an
all-gather of partials and the merge over NCCL; strong scaling), launched
eagerly. With N = 1 it runs the same code on a one-rank process group.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Phase1 context tok/s + % bf16 TC peak; Phase2 decode tok/s + HBM GB/s (1 GPU)"
DEFAULT_CONFIG = "llama8b-16k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def pick_bf16_peak(peaks, peak_src, clocks):
    """The bf16 denominator: the burst figure for kernels that ran at full
    clock, the sustained one (seconds-long GEMM under the power cap) when the
    clocks sampled during timing show the power cap engaged."""
    capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or [])
    if capped and "bf16_tflops_sustained" in peaks:
        return float(peaks["bf16_tflops_sustained"]), f"{peak_src} bf16_tflops_sustained (power cap engaged)"
    return float(peaks["bf16_tflops"]), f"{peak_src} bf16_tflops (burst)"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- oracle CPU baseline
def oracle_sample(w, budget_s=15.0, seed=0):
    """Times the fp64 oracle, as it stands, on a bounded random sample of the
    workload: Phase-1 rows, and the Phase-2 rows of one decode step.
    Returns an estimated step time (s) scaled to the whole step, and a label."""
    import numpy as np
    import torch

    from block_sparse_long_rope_b200 import inputs
    from oracle import oracle as orc

    rng = np.random.default_rng(seed)
    # Phase 1: random (head, row) pairs of sequence 0, uniform over rows
    q, k, v = inputs.make_context(1, w.L, w.Hq, w.Hkv, w.D, w.index)
    q2, k2, v2 = inputs.make_new_tokens(1, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, w.index)
    rows_done, t_p1 = 0, 0.0
    batch = 32
    while t_p1 < budget_s * 0.7:
        rows = rng.integers(0, w.L, size=batch)
        heads = rng.integers(0, w.Hq, size=batch)
        t0 = time.perf_counter()
        orc.phase1_rows(q, k, v, w.block_len, w.anchor_len, w.theta, np.zeros(batch), heads, rows)
        t_p1 += time.perf_counter() - t0
        rows_done += batch
    per_row_p1 = t_p1 / rows_done
    # Phase 2: all heads of one decode token (every split) at the end of the tail
    tail = w.Tq + w.Tdec - 1
    t0 = time.perf_counter()
    orc.phase2_rows(q2[:, tail:tail + 1], k, v, k2, v2, w.block_len, tail, w.theta,
                    np.zeros(w.Hq), np.arange(w.Hq), np.zeros(w.Hq))
    t_dec = time.perf_counter() - t0  # one decode token, all heads
    est_step = (per_row_p1 * w.L * w.Hq + t_dec * (w.Tq + w.Tdec)) * w.B
    sample = (f"{rows_done} random Phase-1 (row, head) queries of sequence 0 and one decode token "
              f"(all {w.Hq} heads, all splits); step time extrapolated to B*L*Hq Phase-1 rows and "
              f"Tq+Tdec Phase-2 tokens")
    del q, k, v, q2, k2, v2, torch
    return est_step, sample, t_p1 + t_dec


def code_digest(paths):
    """sha256 of the given sources with comments and whitespace removed, so
    that only a change of the code itself marks a capture as stale."""
    import hashlib
    import re

    h = hashlib.sha256()
    for src in paths:
        with open(os.path.join(ROOT, src)) as g:
            text = g.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()


def phase1_traffic(workload):
    """DRAM bytes (read + write) of one star_phase1_encode launch from the ncu
    capture recorded under profiles/, if the kernel code is still the code
    that was profiled; None otherwise (the counters no longer apply)."""
    path = os.path.join(ROOT, "profiles", f"phase1_traffic_{workload}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if code_digest(rec["sources"]) != rec["code_sha256"]:
            return None
        return int(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def max_over_ranks(values, device, world):
    """Element-wise max of per-rank timings (ms) over all ranks."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_value(tokens_per_rank, world, ms_per_step):
    """Whole-job throughput: tokens all ranks processed per second of the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v else (os.cpu_count() or 1)


def host_cpu():
    """The host's CPU model (first 'model name' of /proc/cpuinfo) and its
    logical core count, recorded beside the CPU baseline."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_cores": os.cpu_count()}


# --------------------------------------------------------------------------- star arm
def pack_calls(calls, device=None, pin=False):
    """The Phase-2 inputs of a step (every call's q, k, v) laid out back to
    back in one bf16 buffer, so a step uploads them with one copy: returns
    (buffer, calls whose q, k, v are views into it). Every tensor holds a
    multiple of 8 elements, so each view starts 16-byte aligned."""
    import torch

    sizes = [x.numel() for c in calls for x in c[:3]]
    buf = torch.empty(sum(sizes), dtype=torch.bfloat16, device=device)
    if pin:
        buf = buf.pin_memory()
    out, off = [], 0
    for c in calls:
        views = []
        for x in c[:3]:
            views.append(buf[off:off + x.numel()].view(x.shape))
            off += x.numel()
        out.append(tuple(views) + (c[3],))
    return buf, out


def run_star(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from block_sparse_long_rope_b200 import inputs, star
    from block_sparse_long_rope_b200.pipeline import StarLayer, phase2_calls

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peak_src = load_peaks()

    # inputs: every rank holds its own independent sequences (seeded per rank)
    cfg_index = w.index + 100 * rank
    with torch.no_grad():
        ctx = inputs.make_context(w.B, w.L, w.Hq, w.Hkv, w.D, cfg_index, device=dev)
        new = inputs.make_new_tokens(w.B, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, cfg_index, device=dev)
    calls = phase2_calls(w, *new)
    layer = StarLayer(w, device=dev)
    stream = torch.cuda.current_stream()

    def phase1():
        layer.encode(*ctx)

    def query_chunk():
        q2, k2, v2, tail = calls[0]
        layer.attend(q2, k2, v2, tail)

    def decode_loop():
        for (q2, k2, v2, tail) in calls[1:]:
            layer.attend(q2, k2, v2, tail)

    parts = [phase1, query_chunk, decode_loop]
    if args.graph:
        # every call enqueues fixed kernels on fixed buffers, so each part is
        # captured once as a CUDA graph and replayed (no per-call launch cost)
        for fn in parts:
            fn()
        torch.cuda.synchronize()
        graphs = []
        for fn in parts:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs.append(g)
        parts = [g.replay for g in graphs]
        stream = torch.cuda.current_stream()

    def step(ev=None):
        for i, fn in enumerate(parts):
            if ev is not None:
                ev[i].record(stream)
            fn()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    star.star_device_status(layer.buf.ws1)
    star.star_device_status(layer.buf.ws2)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    elapsed_ms = start.elapsed_time(end)
    p1_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    chunk_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    star.star_device_status(layer.buf.ws1)
    star.star_device_status(layer.buf.ws2)

    elapsed_ms, p1_ms, chunk_ms, dec_ms = max_over_ranks(
        [elapsed_ms, p1_ms, chunk_ms, dec_ms], dev, world)

    # ---- end to end through the public API with host buffers ----------------
    # Every step uploads its inputs from pinned host memory, runs the layer
    # and reads its results back. Steps are pipelined over three streams (as a
    # serving loop would run them): the upload of step i+1 overlaps the
    # compute of step i and the read-back of step i-1. Two layers (caches,
    # outputs) and two device input sets alternate, so no step waits on a
    # buffer another step still uses except through the events below.
    # The new tokens of all the step's calls sit back to back in one pinned
    # staging buffer (as a serving loop would batch them), so the upload is
    # one copy for them plus one per context tensor: at 55 GB/s over the
    # host link, ~200 separate small copies cost about a millisecond a step.
    host_ctx = [t.cpu().pin_memory() for t in ctx]
    host_pack, host_calls = pack_calls(calls, pin=True)
    for hc, c in zip(host_calls, calls):
        for h, x in zip(hc[:3], c[:3]):
            h.copy_(x)
    layers2 = [layer, StarLayer(w, device=dev)]
    dev_sets = [([torch.empty_like(t) for t in ctx], pack_calls(calls, device=dev)) for _ in range(2)]
    # the step's result read back is the last generated token's attention
    # output; the Phase-1 output stays on the device (a decoder's next layer
    # consumes it there)
    host_dec = torch.empty((w.B, 1, w.Hq, w.D), dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_ctx) + \
        sum(x.numel() * x.element_size() for c in host_calls for x in c[:3])
    d2h = host_dec.numel() * 2
    s_up, s_comp, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def compute(k):
        lay, (dctx, (_, dcalls)) = layers2[k], dev_sets[k]
        lay.encode(*dctx)
        out = None
        for (q2, k2, v2, tail) in dcalls:
            out = lay.attend(q2, k2, v2, tail)
        return out

    replay = [None, None]  # with --graph: the compute of each buffer set as a CUDA graph

    def e2e_step(i):
        k = i % 2
        lay, (dctx, (dpack, _)) = layers2[k], dev_sets[k]
        s_up.wait_event(ev_comp[k])        # step i-2 no longer reads these inputs
        with torch.cuda.stream(s_up):
            for d, h in zip(dctx, host_ctx):
                d.copy_(h, non_blocking=True)
            dpack.copy_(host_pack, non_blocking=True)
            ev_up[k].record(s_up)
        s_comp.wait_event(ev_up[k])
        s_comp.wait_event(ev_down[k])      # step i-2's outputs have been read back
        with torch.cuda.stream(s_comp):
            if replay[k] is not None:
                replay[k][0].replay()
                out = replay[k][1]
            else:
                out = compute(k)
            ev_comp[k].record(s_comp)
        s_down.wait_event(ev_comp[k])
        with torch.cuda.stream(s_down):
            host_dec.copy_(out[0], non_blocking=True)
            ev_down[k].record(s_down)

    for i in range(max(2, args.warmup // 2)):
        e2e_step(i)
    torch.cuda.synchronize()
    if args.graph:
        for k in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_comp):
                out_k = compute(k)
            replay[k] = (g, out_k)
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record(s_up)
    s_comp.wait_event(s2)
    s_down.wait_event(s2)
    for i in range(args.steps):
        e2e_step(i)
    s_down.wait_event(ev_comp[(args.steps - 1) % 2])
    e2.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([s2.elapsed_time(e2)], dev, world)[0]
    for lay in layers2:
        star.star_device_status(lay.buf.ws1)
        star.star_device_status(lay.buf.ws2)
    del layers2[1], dev_sets, replay

    # ---- generalised prefix: Pulsar's layout on the same workload (a side
    # measurement outside the step: sink + 12.5% chunk summaries per block)
    pulsar = None
    if args.pulsar:
        from block_sparse_long_rope_b200 import prefix as pfx
        chunks = pfx.draw_chunks(w.L, w.block_len, seed=cfg_index)
        src, pos, bounds = pfx.pulsar_table(w.L, w.block_len, chunks)
        layer.set_prefix(src, pos, bounds)
        run = lambda: layer.encode(*ctx)  # noqa: E731
        if args.graph:
            run()
            torch.cuda.synchronize()
            gp = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gp):
                layer.encode(*ctx)
            run = gp.replay
        for _ in range(args.warmup):
            run()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s3 = torch.cuda.Event(enable_timing=True)
        e3 = torch.cuda.Event(enable_timing=True)
        s3.record(stream)
        for _ in range(args.steps):
            run()
        e3.record(stream)
        torch.cuda.synchronize()
        star.star_device_status(layer.ws_phase1)
        layer.set_prefix(None, None, None)
        pul_ms = max_over_ranks([s3.elapsed_time(e3) / args.steps], dev, world)[0]
        pulsar = (pul_ms, pfx.prefix_pairs(w.L, w.block_len, bounds), int(src.size))

    # ---- a decoder stack around Star attention (a side measurement outside
    # the step): RMSNorm, Q/K/V/O projections (cuBLASLt) and Phase 1 per layer
    stack_res = None
    if args.stack_layers > 0:
        from block_sparse_long_rope_b200.stack import StarStack
        dm = w.Hq * w.D
        wts = inputs.make_stack_weights(args.stack_layers, dm, w.Hq, w.Hkv, w.D, w.index,
                                        device=dev)
        stk = StarStack(w, dm, wts, device=dev)
        x0 = inputs.make_hidden(w.B, w.L, dm, w.index, device=dev)
        xs = torch.empty_like(x0)
        for _ in range(args.warmup):
            xs.copy_(x0)
            stk.encode(xs)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i in range(args.steps):
            xs.copy_(x0)  # a fresh residual stream each pass (outside the events)
            sev[i][0].record(stream)
            stk.encode(xs)
            sev[i][1].record(stream)
        torch.cuda.synchronize()
        for ly in stk.layers:
            star.star_device_status(ly.buf.ws1)
        st_ms = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in sev) / args.steps], dev,
                               world)[0]
        stack_res = (st_ms, stk.flops_encode(), dm)
        del stk, wts, x0, xs

    if rank != 0:
        return None

    K = args.steps
    ms_step = elapsed_ms / K
    ctx_tokens = w.B * w.L * world
    value = job_value(w.B * w.L, world, ms_step)
    p1_s = p1_ms / K / 1e3
    p1_flops = w.phase1_flops()
    p1_tflops = p1_flops / p1_s / 1e12
    bf16_peak, bf16_src = pick_bf16_peak(peaks, peak_src, clocks)
    hbm_peak = float(peaks["hbm_gbs"])
    dec_s = dec_ms / K / 1e3
    # bytes of K+V cache every decode step reads (tail grows by one per step)
    dec_bytes = sum(w.decode_kv_bytes(w.Tq + s) for s in range(w.Tdec))
    dec_gbs = dec_bytes / dec_s / 1e9 if dec_s > 0 else None
    dec_tok_s = w.B * w.Tdec / dec_s if dec_s > 0 else None
    chunk_s = chunk_ms / K / 1e3
    launches = 2 + 3 + w.Tdec  # rope+attn; rope+attn+merge; one decode kernel per token

    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tok/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) bf16 Q/K/V (seeded); the pages' RULER/BABILong/InfiniteBench "
                "runs need datasets and trained weights not available here",
        "config": {
            "workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "block_len": w.block_len, "anchor_len": w.anchor_len, "theta": w.theta,
            "Tq": w.Tq, "Tdec": w.Tdec, "global_batch": w.B * world, "seq_len": w.L,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "launch": "cuda_graph (one graph per phase, replayed)" if args.graph else "eager",
            "l2": "step inputs (Q+K+V context, 192 MiB at 16K) exceed the 126 MB L2; no flush",
        },
        "phases": {
            "phase1": {"ms": round(p1_s * 1e3, 4), "ctx_tok_s": round(w.B * w.L / p1_s, 1),
                       "unmasked_tflops": round(p1_tflops, 2),
                       "frac_bf16_peak": round(p1_tflops / bf16_peak, 4),
                       "note": "star_phase1_encode call: RoPE kernel + attention kernel"},
            **({} if pulsar is None else {"phase1_pulsar_layout": {
                "ms": round(pulsar[0], 4), "ctx_tok_s": round(w.B * w.L / (pulsar[0] / 1e3), 1),
                "unmasked_tflops": round(4.0 * w.D * w.Hq * w.B * pulsar[1] / (pulsar[0] / 1e3) / 1e12, 2),
                "frac_bf16_peak": round(4.0 * w.D * w.Hq * w.B * pulsar[1] / (pulsar[0] / 1e3) / 1e12 / bf16_peak, 4),
                "table_rows": pulsar[2],
                "speedup_vs_star_phase1": round(p1_s * 1e3 / pulsar[0], 3),
                "note": "star_phase1_encode_ext: 64-token sink + per-block summaries of 32-token "
                        "chunks (12.5% of a block, seeded draw standing in for Max-IDF); block i "
                        "sees sink + summaries of blocks < i at original positions; "
                        "gather/rope + rope + attention kernels"}}),
            **({} if stack_res is None else {"stack_encode": {
                "layers": args.stack_layers, "d_model": stack_res[2],
                "ms": round(stack_res[0], 4),
                "ctx_tok_s": round(w.B * w.L / (stack_res[0] / 1e3), 1),
                "tflops": round(stack_res[1] / (stack_res[0] / 1e3) / 1e12, 2),
                "frac_bf16_peak": round(stack_res[1] / (stack_res[0] / 1e3) / 1e12 / bf16_peak, 4),
                "note": "per layer: star_rmsnorm, Q/K/V projections and the O projection with "
                        "the residual (cuBLASLt GEMMs), star_phase1_encode; random weights; "
                        "FLOPs = projections + Phase-1 unmasked attention"}}),
            "phase2_query_chunk": {"ms": round(chunk_s * 1e3, 4), "tokens": w.Tq,
                                   "tflops": round(4.0 * w.D * w.Hq * w.B * w.Tq * w.L / chunk_s / 1e12, 2)},
            "phase2_decode": {"ms": round(dec_s * 1e3, 4), "tok_s": round(dec_tok_s, 1),
                              "kv_gbs": round(dec_gbs, 1),
                              "frac_hbm": round(dec_gbs / hbm_peak, 4),
                              "note": "per decode step: one kernel (RoPE/append, split-KV "
                                      "decode, split reduce and merge); the cache was "
                                      "just written by Phase 1, so a cache smaller than L2 "
                                      "(126 MB) reads partly from L2"},
        },
        "roofline": {"bound": "tensor", "kernel": "phase1 (star_phase1_encode)",
                     "achieved": round(p1_tflops, 2), "peak": bf16_peak,
                     "unit": "TFLOP/s", "frac": round(p1_tflops / bf16_peak, 4),
                     "peak_source": bf16_src,
                     "algorithmic": "4*D*Hq*B*[n*b(b+1)/2 + (n-1)*a*b] unmasked FLOPs per launch "
                                    f"= {p1_flops:.4g}",
                     "traffic": phase1_traffic(w.name),
                     "traffic_unit": "bytes per launch (DRAM read + write, ncu)"},
        "e2e": {"value": round(job_value(w.B * w.L, world, e2e_ms / K), 1), "unit": "tok/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_ms / K, 4),
                "note": "public API (StarLayer.encode/attend; with the default graph launch "
                        "each buffer set's calls are captured once and replayed); every step "
                        "uploads all its inputs (context Q/K/V and the new tokens) from pinned "
                        "host memory and reads back its result, the last generated token's "
                        "attention output (the Phase-1 output stays on the device for the next "
                        "layer); steps pipelined over upload / compute / read-back streams"},
        "gpu_launches": launches * K,
        "clocks": clocks,
    }
    if args.cpu_baseline:
        est_step, sample, spent = oracle_sample(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(w.B * w.L / est_step, 3), "unit": "tok/s",
                                "cores": omp_threads(), "kind": "oracle", "sample": sample,
                                "seconds_spent": round(spent, 2), "extrapolated": True,
                                **host_cpu()}
    return line


def run_sharded(args, w, rank, world, local_rank):
    """One sequence over the ranks (block_sparse_long_rope_b200.sharded)."""
    import torch
    import torch.distributed as dist

    from block_sparse_long_rope_b200 import inputs, sharded, star
    from block_sparse_long_rope_b200.pipeline import phase2_calls

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peak_src = load_peaks()
    plan = sharded.shard_plan(w.L, w.block_len, world)
    sh = plan[rank]
    with torch.no_grad():
        q, k, v = inputs.make_context(w.B, w.L, w.Hq, w.Hkv, w.D, w.index, device=dev)
        rows = slice(sh.row0, sh.row0 + sh.rows)
        ctx = [t[:, rows].contiguous() for t in (q, k, v)]
        anchor = [t[:, :w.anchor_len].contiguous() for t in (k, v)]
        del q, k, v
        new = inputs.make_new_tokens(w.B, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, w.index, device=dev)
    calls = phase2_calls(w, *new)
    layer = sharded.ShardedStarLayer(w, plan, rank, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        layer.encode(*ctx, anchor_k=anchor[0], anchor_v=anchor[1])
        if ev is not None:
            ev[1].record(stream)
        out = None
        for (q2, k2, v2, tail) in calls:
            out = layer.attend(q2, k2, v2, tail)
        if ev is not None:
            ev[2].record(stream)
        return out

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    star.star_device_status(layer.ws1)
    star.star_device_status(layer.ws2)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop() if sampler else None
    p1_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    p2_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    elapsed_ms, p1_ms, p2_ms = max_over_ranks([start.elapsed_time(end), p1_ms, p2_ms], dev, world)

    # end to end: this rank's shard and the anchor rows from pinned host memory
    host_ctx = [t.cpu().pin_memory() for t in ctx + anchor]
    host_pack, host_calls = pack_calls(calls, pin=True)  # one copy for all new tokens
    for hc, c in zip(host_calls, calls):
        for h, x in zip(hc[:3], c[:3]):
            h.copy_(x)
    dev_ctx = [torch.empty_like(t) for t in ctx + anchor]
    dev_pack, dev_calls = pack_calls(calls, device=dev)
    host_dec = torch.empty((w.B, 1, w.Hq, w.D), dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_ctx) + \
        sum(x.numel() * x.element_size() for c in host_calls for x in c[:3])
    d2h = host_dec.numel() * 2  # the last generated token's attention output

    def e2e_step():
        for d, h in zip(dev_ctx, host_ctx):
            d.copy_(h, non_blocking=True)
        dev_pack.copy_(host_pack, non_blocking=True)
        layer.encode(*dev_ctx[:3], anchor_k=dev_ctx[3], anchor_v=dev_ctx[4])
        out = None
        for (q2, k2, v2, tail) in dev_calls:
            out = layer.attend(q2, k2, v2, tail)
        host_dec.copy_(out[0], non_blocking=True)

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    dist.barrier()
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([s2.elapsed_time(e2)], dev, world)[0]
    if rank != 0:
        return None

    K = args.steps
    ms_step = elapsed_ms / K
    p1_s = p1_ms / K / 1e3
    p1_tflops_gpu = w.phase1_flops() / p1_s / 1e12 / world
    bf16_peak, bf16_src = pick_bf16_peak(peaks, peak_src, clocks)
    p1_launches = 2 if sh.first_block == 0 else 3
    line = {
        "metric": METRIC,
        "value": round(w.B * w.L / (ms_step / 1e3), 1),
        "unit": "tok/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) bf16 Q/K/V (seeded), one sequence sharded by blocks",
        "config": {
            "workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "block_len": w.block_len, "anchor_len": w.anchor_len, "theta": w.theta,
            "Tq": w.Tq, "Tdec": w.Tdec, "global_batch": w.B, "seq_len": w.L,
            "parallelism": f"sequence-sharded{world}", "launch": "eager",
            "l2": "step inputs exceed the 126 MB L2 at 16K and up; no flush",
        },
        "phases": {
            "phase1": {"ms": round(p1_s * 1e3, 4),
                       "unmasked_tflops_per_gpu": round(p1_tflops_gpu, 2),
                       "note": "slowest rank's Phase 1 (star_phase1_encode or _ext on its shard)"},
            "phase2": {"ms": round(p2_ms / K, 4),
                       "note": "query chunk + decode steps: broadcast, partials, all-gather, merge"},
        },
        "roofline": {"bound": "tensor", "kernel": "phase1 (per-shard encode)",
                     "achieved": round(p1_tflops_gpu, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": round(p1_tflops_gpu / bf16_peak, 4),
                     "peak_source": bf16_src,
                     "algorithmic": "whole-sequence Phase-1 unmasked FLOPs / slowest rank / N",
                     "traffic": None},
        "e2e": {"value": round(w.B * w.L / (e2e_ms / K / 1e3), 1), "unit": "tok/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": (p1_launches + 3 + 2 * w.Tdec) * K,
        "clocks": clocks,
    }
    if args.cpu_baseline:
        est_step, sample, spent = oracle_sample(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(w.B * w.L / est_step, 3), "unit": "tok/s",
                                "cores": omp_threads(), "kind": "oracle", "sample": sample,
                                "seconds_spent": round(spent, 2), "extrapolated": True,
                                **host_cpu()}
    return line


def run_reference(args, w, rank):
    """Reference arm: the fp64 oracle as it stands, on the host cores, each step
    a bounded sample of the workload scaled to the step."""
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=0.5)
    t0 = time.perf_counter()
    est = []
    sample = ""
    for _ in range(args.steps):
        e, sample, _ = oracle_sample(w, budget_s=args.ref_budget)
        est.append(e)
    wall = time.perf_counter() - t0
    est_step = sum(est) / len(est)
    value = w.B * w.L / est_step
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "tok/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(est_step * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) bf16 Q/K/V (seeded)", "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "block_len": w.block_len, "anchor_len": w.anchor_len},
        "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": omp_threads(),
                         "kind": "oracle", "sample": sample, "extrapolated": True,
                         **host_cpu()},
        "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }


def _free_port():
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="star", choices=["star", "reference"])
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--eager", dest="graph", action="store_false",
                    help="launch every call directly instead of replaying CUDA graphs")
    ap.add_argument("--no-pulsar", dest="pulsar", action="store_false",
                    help="skip the side measurement of Phase 1 with Pulsar's prefix layout")
    ap.add_argument("--stack-layers", type=int, default=2,
                    help="layers of the side measurement of a decoder stack (0 skips it)")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "sharded"],
                    help="replicas: independent sequences per rank; sharded: one sequence's "
                         "blocks spread over the ranks")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=8.0)
    args = ap.parse_args()

    from block_sparse_long_rope_b200.configs import BY_NAME
    w = BY_NAME[args.config]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host cores; other ranks exit 0
        line = run_reference(args, w, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    use_pg = world > 1 or args.mode == "sharded"
    if use_pg:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(_free_port()))
        dist.init_process_group(backend="nccl", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run = run_sharded if args.mode == "sharded" else run_star
        line = run(args, w, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if use_pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
