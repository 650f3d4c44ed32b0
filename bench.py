"""Benchmark of the Star Attention hot path on B200 (one attention layer).

A step is one pass of the whole hot path over one batch of synthetic input:
RoPE + Phase-1 anchor-block encoding of the context, the Phase-2 query chunk
(partials + LSE merge), then every single-token decode step (partials + LSE
merge). Inputs are resident in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl star|reference]

One JSON line on stdout (rank 0). With N > 1 (torchrun, one rank per GPU)
the default spreads ONE sequence's blocks over the N ranks (the pages'
multi-host form: Phase 1 per shard, Phase 2 with a query broadcast, an
all-gather of partials and the merge over NCCL; strong scaling), launched
eagerly; the time is the max over ranks. --mode sharded runs the same code
on a one-rank process group at N = 1. --mode replicas gives every rank its
own independent sequences instead (weak scaling, no data-path collective).
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
DEFAULT_CONFIG = "llama8b-1m"     # the largest single-GPU workload: the headline
SIDE_CONFIG = "llama8b-16k"       # Pulsar layout and decoder stack side measurements
PHASE2_CONFIG = "llama70b-128k"   # Phase 2 at 128K context (query chunk, decode)
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
def _host_inputs(w, seed):
    """Sequence 0's pre-RoPE K and V [1, L, Hkv, D] and the Phase-2 tokens,
    drawn on the host for the CPU timing: N(0, 1) in fp32 cast to bf16, like
    the GPU inputs (other values: only the sample's time is used). Long
    contexts are drawn in row chunks on several threads."""
    from concurrent.futures import ThreadPoolExecutor

    import torch

    from block_sparse_long_rope_b200 import inputs

    def draw(rows, H, sid):
        out = torch.empty((1, rows, H, w.D), dtype=torch.bfloat16)
        step = 1 << 16

        def part(i):
            lo = i * step
            g = torch.Generator().manual_seed(seed * 100003 + sid * 10007 + i)
            n = min(step, rows - lo)
            out[0, lo:lo + n] = torch.randn((n, H, w.D), generator=g).to(torch.bfloat16)

        with ThreadPoolExecutor(max_workers=omp_threads()) as ex:
            list(ex.map(part, range(-(-rows // step))))
        return out

    k = draw(w.L, w.Hkv, 1)
    v = draw(w.L, w.Hkv, 2)
    new = inputs.make_new_tokens(1, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, w.index)
    return k, v, new


def oracle_sample(w, budget_s=15.0, seed=0, host=None):
    """Times the fp64 oracle, as it stands, on a bounded random sample of the
    workload: Phase-1 rows (random rows and heads of sequence 0), and the
    Phase-2 rows of one decode token. `host` = (k, v, new tokens) of
    sequence 0 on the host, drawn by _host_inputs if not given.
    Returns an estimated step time (s) scaled to the whole step, a label, and
    the seconds of oracle work timed."""
    import numpy as np
    import torch

    from oracle import oracle as orc

    rng = np.random.default_rng(seed)
    k, v, (q2, k2, v2) = host if host is not None else _host_inputs(w, seed)
    g = w.Hq // w.Hkv
    rows_done, t_p1 = 0, 0.0
    batch = 256
    gq = torch.Generator().manual_seed(seed + 7)
    while rows_done == 0 or t_p1 < budget_s * 0.6:
        # one call = 256 random rows of the query heads of one KV group (the
        # oracle rotates that group's keys once per call)
        kvh = int(rng.integers(0, w.Hkv))
        rows = rng.integers(0, w.L, size=batch)
        heads = kvh * g + rng.integers(0, g, size=batch)
        q_sel = torch.randn((batch, w.D), generator=gq).to(torch.bfloat16)
        t0 = time.perf_counter()
        orc.phase1_rows_selected(q_sel, k, v, w.block_len, w.anchor_len, w.theta,
                                 np.zeros(batch), heads, rows, w.Hq)
        t_p1 += time.perf_counter() - t0
        rows_done += batch
    per_row_p1 = t_p1 / rows_done
    # Phase 2: the g heads of one KV group for one decode token (every
    # split) at the end of the tail, scaled to all Hkv groups
    tail = w.Tq + w.Tdec - 1
    kvh = int(rng.integers(0, w.Hkv))
    heads = kvh * g + np.arange(g)
    t0 = time.perf_counter()
    orc.phase2_rows(q2[:, tail:tail + 1], k, v, k2, v2, w.block_len, tail, w.theta,
                    np.zeros(g), heads, np.zeros(g))
    t_dec = (time.perf_counter() - t0) * w.Hkv  # one decode token, all heads
    est_step = (per_row_p1 * w.L * w.Hq + t_dec * (w.Tq + w.Tdec)) * w.B
    sample = (f"{rows_done} random Phase-1 (row, head) queries of sequence 0 in calls of {batch} "
              f"rows of one KV group, and the {g} heads of one KV group for one decode token "
              "(all splits, scaled by Hkv); step time extrapolated to B*L*Hq Phase-1 rows and "
              "Tq+Tdec Phase-2 tokens")
    return est_step, sample, t_p1 + t_dec / w.Hkv


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


def layer_launches(w):
    """Kernels one step of workload w launches: Phase 1 (RoPE + attention),
    the query chunk (RoPE + attention + the sub-split reduction with the
    merge, or the merge alone), one decode kernel per token (which also
    merges)."""
    chunk = 0
    if w.Tq > 0:
        chunk = 1 if w.Tq * (w.Hq // w.Hkv) <= 16 else 3
    return 2 + chunk + w.Tdec


def flush_l2(buf):
    """Evicts the 126 MB L2 by reading a 256 MiB buffer that is never written
    (its lines stay clean, so the timed call that follows pays no write-back
    of dirty lines, as zeroing a buffer would leave it to)."""
    buf.sum()


def cold_decode(layer, call, reps, dev, world):
    """Mean device time (ms) of one decode call with L2 evicted before each
    repetition (events around the call alone), max over ranks."""
    import torch

    q2, k2, v2, tail = call
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)  # 256 MiB
    for _ in range(2):
        layer.attend(q2, k2, v2, tail)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        # a spin of ~0.5 ms puts the host ahead of the device, so the events
        # time the call's kernels and not the host's Python between them
        torch.cuda._sleep(1_000_000)
        flush_l2(flush)
        a.record(stream)
        layer.attend(q2, k2, v2, tail)
        b.record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / reps
    del flush
    return max_over_ranks([ms], dev, world)[0], tail


def side_pulsar(args, w, dev, world):
    """Phase 1 with Pulsar's prefix layout (sink + 12.5% chunk summaries per
    block) on workload w, against the Star anchor in the same run."""
    import torch

    from block_sparse_long_rope_b200 import inputs, star
    from block_sparse_long_rope_b200 import prefix as pfx
    from block_sparse_long_rope_b200.pipeline import StarLayer

    ctx = inputs.make_context(w.B, w.L, w.Hq, w.Hkv, w.D, w.index, device=dev)
    layer = StarLayer(w, device=dev)
    stream = torch.cuda.current_stream()

    def timed(run):
        run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks([a.elapsed_time(b) / args.steps], dev, world)[0]

    star_ms = timed(lambda: layer.encode(*ctx))
    chunks = pfx.draw_chunks(w.L, w.block_len, seed=w.index)
    src, pos, bounds = pfx.pulsar_table(w.L, w.block_len, chunks)
    layer.set_prefix(src, pos, bounds)
    pul_ms = timed(lambda: layer.encode(*ctx))
    star.star_device_status(layer.ws_phase1)
    layer.set_prefix(None, None, None)
    star.star_device_status(layer.buf.ws1)
    res = {"workload": w.name, "ms": pul_ms, "star_anchor_ms": star_ms,
           "pairs": pfx.prefix_pairs(w.L, w.block_len, bounds), "rows": int(src.size)}
    del layer, ctx
    torch.cuda.empty_cache()
    return res


def side_stack(args, w, dev, world):
    """A decoder stack (RMSNorm, Q/K/V/O projections, Star Phase 1 per layer)
    on workload w: mean ms per encode of args.stack_layers layers."""
    import torch

    from block_sparse_long_rope_b200 import inputs, star
    from block_sparse_long_rope_b200.stack import StarStack

    dm = w.Hq * w.D
    wts = inputs.make_stack_weights(args.stack_layers, dm, w.Hq, w.Hkv, w.D, w.index, device=dev)
    stk = StarStack(w, dm, wts, device=dev)
    x0 = inputs.make_hidden(w.B, w.L, dm, w.index, device=dev)
    xs = torch.empty_like(x0)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        xs.copy_(x0)
        stk.encode(xs)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i in range(args.steps):
        xs.copy_(x0)  # a fresh residual stream each pass (outside the events)
        sev[i][0].record(stream)
        stk.encode(xs)
        sev[i][1].record(stream)
    torch.cuda.synchronize()
    for ly in stk.layers:
        star.star_device_status(ly.buf.ws1)
    st_ms = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in sev) / args.steps], dev, world)[0]
    res = {"workload": w.name, "ms": st_ms, "flops": stk.flops_encode(), "d_model": dm,
           "proj_flops": stk.flops_encode() - args.stack_layers * w.phase1_flops()}
    del stk, wts, x0, xs
    torch.cuda.empty_cache()
    return res


def side_phase2(args, w, dev, world, peaks):
    """Phase 2 of workload w after one Phase-1 encode: the query chunk (mean
    of replays, L2 evicted before each), the decode loop of all Tdec tokens
    as one graph (consecutive steps overlap), and one decode step in
    isolation with L2 evicted before it."""
    import torch

    from block_sparse_long_rope_b200 import inputs, star
    from block_sparse_long_rope_b200.pipeline import StarLayer, phase2_calls

    ctx = inputs.make_context(w.B, w.L, w.Hq, w.Hkv, w.D, w.index, device=dev)
    new = inputs.make_new_tokens(w.B, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, w.index, device=dev)
    calls = phase2_calls(w, *new)
    layer = StarLayer(w, device=dev)
    layer.encode(*ctx)
    del ctx
    stream = torch.cuda.current_stream()
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)  # 256 MiB
    res = {"workload": w.name}
    if w.Tq > 0:
        q2, k2, v2, tail = calls[0]
        layer.attend(q2, k2, v2, tail)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.attend(q2, k2, v2, tail)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for _ in range(args.warmup):
            g.replay()
        for a, b in evs:
            flush_l2(flush)
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in evs) / args.steps], dev, world)[0]
        res["query_chunk"] = {"ms": ms, "tokens": w.Tq,
                              "flops": 4.0 * w.D * w.Hq * w.B * w.Tq * w.L}
    if w.Tdec > 0:
        dec = calls[1:] if w.Tq > 0 else calls
        for (q2, k2, v2, tail) in dec:
            layer.attend(q2, k2, v2, tail)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for (q2, k2, v2, tail) in dec:
                layer.attend(q2, k2, v2, tail)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        loop_ms = max_over_ranks([a.elapsed_time(b) / args.steps], dev, world)[0]
        res["decode_loop"] = {"ms": loop_ms, "steps": w.Tdec,
                              "bytes": sum(w.decode_kv_bytes(w.Tq + s) for s in range(w.Tdec))}
        del g
        cold_ms, tail = cold_decode(layer, dec[-1], args.cold_decode_steps, dev, world)
        res["decode_cold"] = {"ms": cold_ms, "bytes": w.decode_kv_bytes(tail)}
    star.star_device_status(layer.buf.ws2)
    del layer, new, calls, flush
    torch.cuda.empty_cache()
    return res



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

    # one decode step in isolation, L2 evicted before it (the cache of the
    # main workload holds every row from the last step)
    cold_main = cold_decode(layer, calls[-1], args.cold_decode_steps, dev, world) \
        if args.cold_decode_steps > 0 and w.Tdec > 0 else None
    launches_step = layer_launches(w)
    del layers2[0], layer, ctx, new, calls, host_ctx, host_pack, host_calls, host_dec, parts
    if args.graph:
        del graphs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- side measurements outside the step, each on its own workload ------
    from block_sparse_long_rope_b200.configs import BY_NAME
    w_side = BY_NAME[args.side_config]
    pulsar = side_pulsar(args, w_side, dev, world) if args.pulsar else None
    stack_res = side_stack(args, w_side, dev, world) if args.stack_layers > 0 else None
    p2 = None
    if args.phase2_config:
        p2 = side_phase2(args, BY_NAME[args.phase2_config], dev, world, peaks)

    if rank != 0:
        return None

    K = args.steps
    ms_step = elapsed_ms / K
    ctx_bytes = w.B * w.L * (w.Hq + 2 * w.Hkv) * w.D * 2
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
    launches = launches_step
    burst = float(peaks["bf16_tflops"])
    L2_BYTES = 126e6

    def decode_entry(ms, nbytes, steps, cache_bytes, how):
        gbs = nbytes / (ms / 1e3) / 1e9
        key = "frac_hbm" if cache_bytes > L2_BYTES else "frac_hbm_effective"
        return {"ms_per_token": round(ms / steps, 5), "kv_gbs": round(gbs, 1),
                key: round(gbs / hbm_peak, 4), "how": how}

    phases = {
        "phase1": {"ms": round(p1_s * 1e3, 4), "ctx_tok_s": round(w.B * w.L / p1_s, 1),
                   "unmasked_tflops": round(p1_tflops, 2),
                   "frac_bf16_peak": round(p1_tflops / bf16_peak, 4),
                   "note": "star_phase1_encode call: RoPE kernel + attention kernel"},
    }
    if w.Tq > 0:
        phases["phase2_query_chunk"] = {
            "ms": round(chunk_s * 1e3, 4), "tokens": w.Tq,
            "tflops": round(4.0 * w.D * w.Hq * w.B * w.Tq * w.L / chunk_s / 1e12, 2),
            "frac_bf16_peak": round(4.0 * w.D * w.Hq * w.B * w.Tq * w.L / chunk_s / 1e12 / burst, 4)}
    if w.Tdec > 0:
        cache = w.decode_kv_bytes(w.Tq + w.Tdec - 1)
        d = decode_entry(dec_s * 1e3, dec_bytes, w.Tdec, cache,
                         "the step's decode loop (consecutive steps overlap)")
        d["tok_s"] = round(dec_tok_s, 1)
        phases["phase2_decode"] = d
        if cold_main is not None:
            c = decode_entry(cold_main[0], w.decode_kv_bytes(cold_main[1]), 1, cache,
                             "one decode call alone, L2 evicted before it (256 MiB read)")
            c["tok_s"] = round(w.B / (cold_main[0] / 1e3), 1)
            phases["phase2_decode_cold_step"] = c
    if p2 is not None:
        w2 = BY_NAME[p2["workload"]]
        e = {"workload": w2.name}
        if "query_chunk" in p2:
            qc = p2["query_chunk"]
            tf = qc["flops"] / (qc["ms"] / 1e3) / 1e12
            e["query_chunk"] = {"ms": round(qc["ms"], 4), "tokens": qc["tokens"],
                                "tflops": round(tf, 2), "frac_bf16_peak": round(tf / burst, 4),
                                "how": "one query-chunk call, L2 evicted before each (256 MiB read)"}
        if "decode_loop" in p2:
            dl, dc = p2["decode_loop"], p2["decode_cold"]
            cache2 = w2.decode_kv_bytes(w2.Tq + w2.Tdec - 1)
            e["decode_loop"] = decode_entry(dl["ms"], dl["bytes"], dl["steps"], cache2,
                                            "all decode steps as one graph; consecutive steps "
                                            "overlap and part of the cache stays in L2")
            e["decode_loop"]["tok_s"] = round(w2.B * dl["steps"] / (dl["ms"] / 1e3), 1)
            e["decode_cold_step"] = decode_entry(dc["ms"], dc["bytes"], 1, cache2,
                                                 "one decode call alone, L2 evicted before it (256 MiB read)")
            e["decode_cold_step"]["tok_s"] = round(w2.B / (dc["ms"] / 1e3), 1)
        phases["phase2_" + w2.name.replace("-", "_")] = e
    if pulsar is not None:
        ws = BY_NAME[pulsar["workload"]]
        tf = 4.0 * ws.D * ws.Hq * ws.B * pulsar["pairs"] / (pulsar["ms"] / 1e3) / 1e12
        phases["phase1_pulsar_layout"] = {
            "workload": ws.name, "ms": round(pulsar["ms"], 4),
            "unmasked_tflops": round(tf, 2), "frac_bf16_peak": round(tf / burst, 4),
            "table_rows": pulsar["rows"], "star_anchor_ms": round(pulsar["star_anchor_ms"], 4),
            "speedup_vs_star_anchor": round(pulsar["star_anchor_ms"] / pulsar["ms"], 3),
            "note": "star_phase1_encode_ext: 64-token sink + per-block summaries of 32-token "
                    "chunks (12.5% of a block, seeded draw standing in for Max-IDF); block i "
                    "sees sink + summaries of blocks < i at original positions"}
    if stack_res is not None:
        ws = BY_NAME[stack_res["workload"]]
        tf = stack_res["flops"] / (stack_res["ms"] / 1e3) / 1e12
        phases["stack_encode"] = {
            "workload": ws.name, "layers": args.stack_layers, "d_model": stack_res["d_model"],
            "ms": round(stack_res["ms"], 4), "tflops": round(tf, 2),
            "frac_bf16_peak": round(tf / burst, 4),
            "note": "per layer: star_rmsnorm, Q/K/V projections and the O projection with the "
                    "residual, star_phase1_encode; random weights; FLOPs = projections + "
                    "Phase-1 unmasked attention"}

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
            "l2": f"step inputs (Q+K+V context, {ctx_bytes / 2**20:.0f} MiB) "
                  + ("exceed the 126 MB L2; no flush" if ctx_bytes > L2_BYTES
                     else "fit in the 126 MB L2: decode figures are labelled effective"),
        },
        "phases": phases,
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


def run_reference(args, w, rank, world=1):
    """Reference arm: the fp64 oracle as it stands, on the host cores. A full
    step of a long-context workload would take hours to days on a CPU, so
    each of the K steps times a bounded random sample of that step's work
    (Phase-1 rows and one decode token), and the step time is extrapolated
    from the sample; the line says so (`extrapolated`, `sample`,
    `seconds_timed`). The per-step budget keeps the whole run within a few
    minutes."""
    if rank != 0:
        return None
    # the oracle runs on all the host's cores: a torchrun launch sets
    # OMP_NUM_THREADS=1 for every rank, and the other ranks do no work here
    # (read by the oracle's OpenMP runtime when the oracle library loads)
    os.environ["OMP_NUM_THREADS"] = str(os.cpu_count() or 1)
    per_step = max(1.0, min(args.ref_budget, 150.0 / max(1, args.steps + args.warmup)))
    host = _host_inputs(w, 0)
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=min(0.5, per_step), host=host)
    t0 = time.perf_counter()
    est = []
    sample = ""
    spent = 0.0
    for _ in range(args.steps):
        e, sample, sp = oracle_sample(w, budget_s=per_step, host=host)
        est.append(e)
        spent += sp
    wall = time.perf_counter() - t0
    est_step = sum(est) / len(est)
    value = w.B * w.L / est_step
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(est_step * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) bf16 Q/K/V (seeded)", "impl": "reference",
        "extrapolated": True,
        "ran": (f"{args.steps} timed samples of about {per_step:.1f} s each ({spent:.1f} s of "
                f"oracle work, {wall:.1f} s wall) on rank 0's host cores (the launch's "
                f"{world} rank(s); no GPU work); ms_per_step is the step time extrapolated "
                "from the samples, not a timed step"),
        "seconds_timed": round(spent, 2),
        "config": {"workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "block_len": w.block_len, "anchor_len": w.anchor_len},
        "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": omp_threads(),
                         "kind": "oracle", "sample": sample, "extrapolated": True,
                         **host_cpu()},
        "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }


def resolve_mode(mode, world):
    """The run's multi-GPU mode: as asked, else one sequence's blocks over the
    ranks when there are several (the pages' hosts: query broadcast, local
    partials, gather and merge), and a single replica on one GPU."""
    if mode is not None:
        return mode
    return "sharded" if world > 1 else "replicas"


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
    ap.add_argument("--mode", default=None, choices=["replicas", "sharded"],
                    help="replicas: independent sequences per rank; sharded: one sequence's "
                         "blocks spread over the ranks (the pages' deployment; the default "
                         "with more than one GPU)")
    ap.add_argument("--side-config", default=SIDE_CONFIG,
                    help="workload of the side measurements (Pulsar layout, decoder stack)")
    ap.add_argument("--phase2-config", default=PHASE2_CONFIG,
                    help="workload of the Phase-2 side measurement (query chunk, decode loop "
                         "and cold decode step); '' skips it")
    ap.add_argument("--cold-decode-steps", type=int, default=16,
                    help="repetitions of the isolated decode step timed with L2 evicted")
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
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    args.mode = resolve_mode(args.mode, world)
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
