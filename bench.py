"""Benchmark of the paged decode hot path on B200: one JSON line on rank 0.

A step is one pass of the whole path over one batch of the workload: the cache
write of every sequence's new token(s) (reshape_and_cache), the copy-on-write
block copies where the workload has them (copy_blocks), and the paged decode
attention (decode kernel, plus the log-sum-exp reduce for sequences longer than
one partition).  Inputs are resident in HBM when the timed region starts.

Metric: achieved HBM GB/s of algorithmic bytes (K/V read + Q read + output write
+ block tables + sequence lengths for the decode; read + written bytes for the
cache writes and copies), whole job, plus decode tokens/s and context tokens/s
per layer.  The working set (over 1 GB for the default workload) is far larger
than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU: the path shards with no exchange, so N ranks run N independent
replicas (weak scaling); timing is the max over ranks of CUDA-event time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_413_b200 import workloads as W  # noqa: E402

METRIC = "paged-attn decode: achieved HBM GB/s (% of B200 peak), seq-tokens/s per layer"
DEFAULT_CONFIG = "llama2_7b"
FALLBACK_HBM_GBS = 6650.0
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}

PREFILL = {"chunked_prefill_70b": dict(num_seqs=16, context=(2048, 4096), chunk=(512, 512),
                                       num_heads=64, num_kv_heads=8, dtype="bf16", seed=6)}

DESCR = {
    "chunked_prefill_70b": "Llama-2-70B layer, chunked prefill: 16 seqs, context U[2048,4096], "
                           "512-token chunks, 64 q / 8 kv heads, d128, bf16, causal",
    "tiny": "4 seqs L={1,17,33,100}, 4 heads MHA, d64, fp16, pool 64 blocks",
    "llama2_7b": "Llama-2-7B layer: 64 seqs, 32 heads MHA, d128, L~U[128,2048], fp16 KV, "
                 "block 16, shuffled pool 1.1x",
    "llama2_70b_gqa": "Llama-2-70B layer: 256 seqs, 64 q heads / 8 kv heads, d128, "
                      "L~U[512,768], bf16 KV, block 16, shuffled pool 1.1x",
    "long_splitk": "8 seqs x 32768 tokens, 32 q / 8 kv heads, d128, bf16 KV, 512-token "
                   "partitions + LSE reduce",
    "beam_cow_fp8": "64 prompts x 4 beams, 1032 shared tokens + 4 own, 32 q / 8 kv heads, "
                    "d128, FP8 E4M3 KV, copy-on-write copies per step",
}


# ---------------------------------------------------------------- bytes model
def decode_bytes(wl: W.Workload, out_dtype: str) -> int:
    cfg = wl.cfg
    L = wl.seq_lens.numpy().astype(np.int64)
    kv = int(L.sum()) * cfg.num_kv_heads * cfg.head_dim * 2 * W.ELT_BYTES[cfg.cache_dtype]
    qo = len(L) * cfg.num_heads * cfg.head_dim * (W.ELT_BYTES[cfg.q_dtype] +
                                                   W.ELT_BYTES[out_dtype])
    tables = int(np.ceil(L / cfg.block_size).sum()) * 4 + 4 * len(L)
    return kv + qo + tables


def shared_decode_bytes(wl: W.Workload, out_dtype: str) -> int:
    """Shared-prefix decode: each distinct K/V block once, plus Q, out, tables, lengths."""
    cfg = wl.cfg
    L = wl.seq_lens.numpy().astype(np.int64)
    qo = len(L) * cfg.num_heads * cfg.head_dim * (W.ELT_BYTES[cfg.q_dtype] +
                                                   W.ELT_BYTES[out_dtype])
    tables = int(np.ceil(L / cfg.block_size).sum()) * 4 + 4 * len(L)
    groups = 4 * (2 * wl.prefix_lens.numel() + 1)
    return unique_kv_bytes(wl) + qo + tables + groups


def unique_kv_bytes(wl: W.Workload) -> int:
    """K/V bytes of distinct physical blocks the decode reads (shared prefixes once)."""
    cfg = wl.cfg
    bt = wl.block_tables.numpy()
    L = wl.seq_lens.numpy()
    slots = set()
    for i, n in enumerate(L):
        for pos_blk in range(int(math.ceil(n / cfg.block_size))):
            b = int(bt[i, pos_blk])
            used = min(cfg.block_size, int(n) - pos_blk * cfg.block_size)
            slots.add((b, used))
    per_tok = cfg.num_kv_heads * cfg.head_dim * 2 * W.ELT_BYTES[cfg.cache_dtype]
    best = {}
    for b, used in slots:
        best[b] = max(best.get(b, 0), used)
    return sum(best.values()) * per_tok


def cache_write_bytes(wl: W.Workload) -> int:
    cfg = wl.cfg
    t = wl.slot_mapping.numel()
    per = cfg.num_kv_heads * cfg.head_dim * 2
    return t * per * (W.ELT_BYTES[wl.src_dtype] + W.ELT_BYTES[cfg.cache_dtype]) + 8 * t


def copy_bytes(wl: W.Workload) -> int:
    if wl.block_mapping is None or wl.block_mapping.numel() == 0:
        return 0
    cfg = wl.cfg
    block = cfg.block_size * cfg.num_kv_heads * cfg.head_dim * W.ELT_BYTES[cfg.cache_dtype]
    return wl.block_mapping.shape[0] * (2 * 2 * block + 16)


# ---------------------------------------------------------------- helpers
def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(step_bytes: int, world: int, steps: int, elapsed_ms: float) -> float:
    """Replicas: every rank processes its own batch, so the job moves world x the bytes."""
    return step_bytes * world * steps / (elapsed_ms * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("pa_decode.cu", "pa_kernels.cuh", "pa_common.cuh", "pa_internal.h")
PREFILL_SOURCES = ("pa_prefill.cu", "pa_tcgen05.cuh", "pa_kernels.cuh", "pa_common.cuh",
                   "pa_internal.h")
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def source_sha(names=DECODE_SOURCES) -> str:
    """sha256 prefix over a kernel's sources, in a fixed order."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "paged_kv_cache_413_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes (read + written) per launch of the workload's hot kernel, from the
    ncu capture recorded in profiles/traffic.json; None unless the sources it
    lists still hash to the value recorded with the capture."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f)["workloads"][workload]
        if source_sha(tuple(rec["sources"])) == rec["sources_sha256_16"]:
            return int(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        pass
    return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(wl: W.Workload, seqs, out_dtype: str):
    """Run the oracle (cache write of the sampled sequences' tokens + decode of them).
    Returns (seconds, algorithmic bytes of the sample)."""
    import oracle

    cfg = wl.cfg
    seqs = np.asarray(seqs)
    T = cfg.new_tokens_per_seq
    new = np.concatenate([np.arange(s * T, (s + 1) * T) for s in seqs])
    nt = torch.as_tensor(new)
    t0 = time.perf_counter()
    kc, vc = oracle.reshape_and_cache(wl.new_key[nt], wl.new_value[nt], wl.key_cache,
                                      wl.value_cache, wl.slot_mapping.numpy()[new],
                                      src_dtype=wl.src_dtype, cache_dtype=cfg.cache_dtype,
                                      k_scale=wl.k_scale, v_scale=wl.v_scale, inplace=True)
    idx = torch.as_tensor(seqs)
    oracle.paged_attention_decode(wl.query[idx], kc, vc, wl.block_tables.numpy()[seqs],
                                  wl.seq_lens.numpy()[seqs], scale=wl.scale,
                                  q_dtype=cfg.q_dtype, cache_dtype=cfg.cache_dtype,
                                  k_scale=wl.k_scale, v_scale=wl.v_scale)
    dt = time.perf_counter() - t0
    L = wl.seq_lens.numpy()[seqs].astype(np.int64)
    b = int(L.sum()) * cfg.num_kv_heads * cfg.head_dim * 2 * W.ELT_BYTES[cfg.cache_dtype]
    b += len(seqs) * cfg.num_heads * cfg.head_dim * (W.ELT_BYTES[cfg.q_dtype] +
                                                      W.ELT_BYTES[out_dtype])
    b += int(np.ceil(L / cfg.block_size).sum()) * 4 + 4 * len(seqs)
    b += len(new) * cfg.num_kv_heads * cfg.head_dim * 2 * (W.ELT_BYTES[wl.src_dtype] +
                                                          W.ELT_BYTES[cfg.cache_dtype])
    return dt, b


def cpu_baseline(wl: W.Workload, out_dtype: str, budget_s: float = 12.0):
    """The oracle timed on a bounded sample of the workload's sequences, with all the
    host's OpenMP threads and then with one thread on the same sample (or on a
    prefix of it when one thread would exceed the budget)."""
    import oracle

    n = wl.seq_lens.numel()
    order = np.random.default_rng(0).permutation(n)
    dt1, _ = oracle_sample(wl, order[:1], out_dtype)              # calibration
    k = int(max(1, min(n, budget_s / max(dt1, 1e-4))))
    dt, b = oracle_sample(wl, order[:k], out_dtype)
    # the whole workload in well under the budget: time it repeatedly (the cache
    # writes are idempotent) so that the figure rests on seconds of CPU work
    reps = 1
    if dt < 0.8 * budget_s:
        more = min(1000, int((budget_s - dt) / max(dt, 1e-4)))
        for _ in range(more):
            dti, bi = oracle_sample(wl, order[:k], out_dtype)
            dt += dti
            b += bi
        reps += more
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        k1 = int(max(1, min(k, k * reps * budget_s / max(dt * cores, 1e-4))))
        dt_1, b_1 = oracle_sample(wl, order[:k1], out_dtype)
    finally:
        oracle.set_num_threads(cores)
    return {"value": b / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"{k} of {n} sequences of the workload (cache write of their new "
                      f"tokens + fp64 decode)" + (f", {reps} times" if reps > 1 else "") +
                      f", {dt:.1f} s",
            "single_thread": {"value": b_1 / dt_1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"{k1} of the same sequences, {dt_1:.1f} s"}}


def prefill_oracle_sample(wl: W.Workload, seqs):
    """Run the oracle (cache write of the sampled sequences' chunks + their causal
    multi-query attention).  Returns (seconds, useful FLOPs of the sample)."""
    import oracle

    cfg = wl.cfg
    seqs = np.asarray(seqs)
    qs = wl.query_start.numpy().astype(np.int64)
    rows = np.concatenate([np.arange(qs[s], qs[s + 1]) for s in seqs])
    nt = torch.as_tensor(rows)
    sub_qs = np.concatenate([[0], np.cumsum([qs[s + 1] - qs[s] for s in seqs])]).astype(np.int32)
    t0 = time.perf_counter()
    kc, vc = oracle.reshape_and_cache(wl.new_key[nt], wl.new_value[nt], wl.key_cache,
                                      wl.value_cache, wl.slot_mapping.numpy()[rows],
                                      src_dtype=wl.src_dtype, cache_dtype=cfg.cache_dtype,
                                      inplace=True)
    oracle.paged_attention_prefill(wl.query[nt], kc, vc, wl.block_tables.numpy()[seqs],
                                   wl.seq_lens.numpy()[seqs], sub_qs, scale=wl.scale,
                                   q_dtype=cfg.q_dtype, cache_dtype=cfg.cache_dtype)
    dt = time.perf_counter() - t0
    L = wl.seq_lens.numpy().astype(np.int64)
    pairs = sum(int((L[s] - (qs[s + 1] - qs[s]) + np.arange(qs[s + 1] - qs[s]) + 1).sum())
                for s in seqs)
    return dt, pairs * cfg.num_heads * cfg.head_dim * 4


def prefill_cpu_baseline(wl: W.Workload, budget_s: float = 15.0):
    """The oracle timed on a bounded sample of the workload's sequences (all threads,
    then one thread on the same sample or a prefix of it)."""
    import oracle

    n = wl.seq_lens.numel()
    order = np.random.default_rng(0).permutation(n)
    dt1, _ = prefill_oracle_sample(wl, order[:1])              # calibration
    k = int(max(1, min(n, budget_s / max(dt1, 1e-4))))
    dt, fl = prefill_oracle_sample(wl, order[:k])
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        k1 = int(max(1, min(k, k * budget_s / max(dt * cores, 1e-4))))
        dt_1, fl_1 = prefill_oracle_sample(wl, order[:k1])
    finally:
        oracle.set_num_threads(cores)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"{k} of {n} sequences of the workload (cache write of their chunks + "
                      f"fp64 causal attention), {dt:.1f} s",
            "single_thread": {"value": fl_1 / dt_1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                              "sample": f"{k1} of the same sequences, {dt_1:.1f} s"}}


def pipelined_e2e(dev, stream, inputs, host_src, out, run_step, steps, world):
    """End to end through the public API with host buffers.

    Every step uploads its inputs from page-locked host memory (packed in one
    buffer, one copy) and downloads its output.  Uploads run on one copy stream
    and downloads on another, with two device buffers of each, so step k+1's
    upload and step k-1's download overlap step k's compute, as a serving loop
    would run them.  Timed from the first upload to the last download, on the
    device.  Before timing, the output must equal `out` (the device-timed
    result of the same inputs) bit for bit.  Returns (ms, h2d bytes, d2h bytes)
    per step."""
    layout, off = {}, 0
    for name, t in inputs.items():
        layout[name] = (off, t.numel() * t.element_size(), t.dtype, tuple(t.shape))
        off += (layout[name][1] + 255) // 256 * 256
    h_in = torch.zeros(off, dtype=torch.uint8).pin_memory()
    for name, (o, n, dt, shape) in layout.items():
        h_in[o:o + n].copy_(host_src[name].contiguous().view(torch.uint8).reshape(-1))
    d_in = [torch.empty(off, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_views = [{name: buf[o:o + n].view(dt).view(shape)
                for name, (o, n, dt, shape) in layout.items()} for buf in d_in]
    d_out = [torch.empty_like(out) for _ in range(2)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]  # also: d_in[b] free again
    downloaded = [torch.cuda.Event() for _ in range(2)]  # d_out[b] free again

    def e2e_step(k):
        b = k & 1
        if k >= 2:
            up.wait_event(computed[b])
        with torch.cuda.stream(up):
            d_in[b].copy_(h_in, non_blocking=True)
        uploaded[b].record(up)
        stream.wait_event(uploaded[b])
        if k >= 2:
            stream.wait_event(downloaded[b])
        run_step(d_views[b], d_out[b])
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            h_out[b].copy_(d_out[b], non_blocking=True)
        downloaded[b].record(down)

    for k in range(3):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    if not torch.equal(h_out[0].to(dev), out):  # same inputs, deterministic kernels
        raise RuntimeError("the end-to-end output differs from the device-timed output")
    if world > 1:
        torch.distributed.barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(up)  # every timed operation follows it: uploads on `up`, the rest waits on them
    for k in range(steps):
        e2e_step(k)
    a1.record(down)
    torch.cuda.synchronize(dev)
    return a0.elapsed_time(a1), off, h_out[0].numel() * h_out[0].element_size()


# ---------------------------------------------------------------- GPU arm
def timed_loop(step, launches, steps, warmup, dev, stream, world, rank, writes_step=None):
    """`warmup` untimed steps, then exactly `steps` timed ones bracketed by a
    barrier and a device synchronize on both sides, with clocks sampled meanwhile
    on rank 0.  With writes_step (CUDA-graph steps) a second region of `steps`
    replays of the step's cache writes alone follows, bracketed the same way, and a
    hot launch's time is the difference of the two regions' per-step times;
    otherwise step(timed) appends its hot launch's (start, end) events to
    `launches` when timed.  Returns (max-over-ranks elapsed ms, launch ms, clock
    summary or None)."""
    import paged_kv_cache_413_b200 as pa

    def region(fn, sampled):
        sampler = ClockSampler(dev.index) if (rank == 0 and sampled) else None
        if sampler:
            sampler.__enter__()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            fn(True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        if sampler:
            sampler.__exit__(None, None, None)
        if pa.pa_get_device_error() != 0:
            raise RuntimeError("device error bits set during the timed steps")
        return t0.elapsed_time(t1), (sampler.summary() if sampler else None)

    for _ in range(warmup):
        step(False)
        if writes_step is not None:
            writes_step(False)
    torch.cuda.synchronize(dev)
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error bits set during warm-up")
    launches.clear()
    elapsed_ms, clocks = region(step, True)
    if writes_step is not None:
        writes_ms, _ = region(writes_step, False)
        launch_ms = max(elapsed_ms - writes_ms, 0.0) / steps
    else:
        pairs = {id(e0): (e0, e1) for e0, e1 in launches}
        launch_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in pairs.values())
    elapsed_ms, launch_ms = max_over_ranks([elapsed_ms, launch_ms], world, dev)
    return elapsed_ms, launch_ms, clocks


def timing_note(args) -> str:
    if args.no_graphs:
        return ("each timed step calls the library from Python (host launch overhead "
                "included); the launch time brackets the hot kernels with CUDA events")
    return ("each timed step replays one CUDA graph of the library's calls (cache writes, then "
            "the hot kernels), bracketed as a whole by CUDA events on the stream; the launch "
            "time is the step time minus that of as many replays of a graph of the writes "
            "alone (timing events inside a graph would add ~4 us to what they bracket)")


def graph_step(writes, hot, run_step, inputs, out, ev, dev, stream, args):
    """The steps the timed loop runs: (step, writes_step).  By default the step
    replays one CUDA graph captured from the same library calls -- the cache writes
    (and copies), then the hot kernel(s) -- so host-side call overhead never idles
    the GPU inside the timed region, and writes_step replays a graph of the writes
    alone, which the timed loop subtracts to get the hot launches' time (an event
    record node inside a graph adds ~4 us to the interval it brackets, which is why
    the graph holds none).  With --no-graphs the step calls the library directly
    (run_step, events around the hot call) and writes_step is None."""
    if args.no_graphs:
        return (lambda timed: run_step(inputs, out, timed)), None
    run_step(inputs, out, False)          # warm: every kernel attribute set, maps encoded
    torch.cuda.synchronize(dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    g_step, g_writes = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=side):
        writes()
        hot()
    with torch.cuda.graph(g_writes, stream=side):
        writes()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    graphs = (g_step, g_writes)  # kept alive with the closures
    return (lambda timed: graphs[0].replay()), (lambda timed: graphs[1].replay())


def decode_case(cfg, dev, args, world, rank, decode_mode="auto", partition=None,
                with_e2e=True, with_cpu=False):
    """One decode workload, resident in HBM: W + K steps of (copy-on-write copies,
    cache write, decode), timed as a whole and per decode launch; optionally end to
    end through the public API with host buffers, and the CPU oracle baseline."""
    import paged_kv_cache_413_b200 as pa

    wl = W.make_workload(cfg, seed=cfg.seed + 1000 * rank) if rank else W.make_workload(cfg)
    out_dtype = cfg.out_dtype
    f = lambda t: None if t is None else t.to(dev)
    kc, vc = f(wl.key_cache), f(wl.value_cache)
    q, bt, sl = f(wl.query), f(wl.block_tables), f(wl.seq_lens)
    nk, nv, sm = f(wl.new_key), f(wl.new_value), f(wl.slot_mapping)
    bm = f(wl.block_mapping) if wl.block_mapping is not None and wl.block_mapping.numel() else None
    max_len = int(wl.seq_lens.max())
    part = partition if partition is not None else cfg.partition_size
    ws_n = pa.pa_paged_attention_workspace_size(q.shape[0], cfg.num_heads, cfg.num_kv_heads,
                                                cfg.head_dim, max_len, part)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
    out = torch.empty(q.shape, dtype=TORCH_DT[out_dtype], device=dev)
    stream = torch.cuda.current_stream(dev)
    if wl.prefix_key is not None:  # copy-on-write workload: fill the shared prefix once
        pa.pa_reshape_and_cache(f(wl.prefix_key), f(wl.prefix_value), kc, vc,
                                f(wl.prefix_slot_mapping), k_scale=wl.k_scale,
                                v_scale=wl.v_scale)
    part_eff = pa.pa_paged_attention_partition_size(q.shape[0], cfg.num_heads, cfg.num_kv_heads,
                                                    max_len, part)
    reduce_runs = max_len > part_eff
    shared = wl.group_starts is not None and decode_mode in ("auto", "shared")
    launches = 1 + 1 + (1 if bm is not None else 0) + (1 if reduce_runs and not shared else 0)
    gs = pl = None
    if shared:
        gs, pl = f(wl.group_starts), f(wl.prefix_lens)
        max_group = int((wl.group_starts[1:] - wl.group_starts[:-1]).max())
    ev = []
    # the step's inputs: what a serving loop hands over every step
    inputs = {"q": q, "nk": nk, "nv": nv, "sm": sm, "bt": bt, "sl": sl}
    if bm is not None:
        inputs["bm"] = bm
    if shared:
        inputs.update(gs=gs, pl=pl)

    def writes(t):
        if "bm" in t:
            pa.pa_copy_blocks([kc], [vc], t["bm"])
        pa.pa_reshape_and_cache(t["nk"], t["nv"], kc, vc, t["sm"], k_scale=wl.k_scale,
                                v_scale=wl.v_scale)

    def decode(t, out_t):
        if shared:
            pa.pa_paged_attention_decode_shared_prefix(
                out_t, t["q"], kc, vc, t["bt"], t["sl"], t["gs"], t["pl"], max_seq_len=max_len,
                max_group_size=max_group, scale=wl.scale, k_scale=wl.k_scale,
                v_scale=wl.v_scale)
        else:
            pa.pa_paged_attention_decode(out_t, t["q"], kc, vc, t["bt"], t["sl"],
                                         max_seq_len=max_len, scale=wl.scale,
                                         k_scale=wl.k_scale, v_scale=wl.v_scale,
                                         partition_size=part, workspace=ws)

    def run_step(t, out_t, timed: bool = False):
        writes(t)
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        decode(t, out_t)
        if timed:
            e1.record(stream)
            ev.append((e0, e1))

    step, writes_step = graph_step(lambda: writes(inputs), lambda: decode(inputs, out),
                                   run_step, inputs, out, ev, dev, stream, args)
    elapsed_ms, decode_ms, clocks = timed_loop(step, ev, args.steps, args.warmup, dev, stream,
                                               world, rank, writes_step)
    dec_b = shared_decode_bytes(wl, out_dtype) if shared else decode_bytes(wl, out_dtype)
    step_bytes = dec_b + cache_write_bytes(wl) + copy_bytes(wl)
    res = {"wl": wl, "shared": shared, "part_eff": part_eff, "dec_b": dec_b,
           "step_bytes": step_bytes, "elapsed_ms": elapsed_ms, "decode_ms": decode_ms,
           "clocks": clocks, "launches": launches, "out_dtype": out_dtype}
    if with_e2e:
        host_src = {"q": wl.query, "nk": wl.new_key, "nv": wl.new_value, "sm": wl.slot_mapping,
                    "bt": wl.block_tables, "sl": wl.seq_lens, "bm": wl.block_mapping,
                    "gs": wl.group_starts, "pl": wl.prefix_lens}
        e2e_steps = max(10, args.steps // 4)
        e2e_ms, h2d, d2h = pipelined_e2e(dev, stream, inputs, host_src, out, run_step,
                                         e2e_steps, world)
        res["e2e"] = (max_over_ranks([e2e_ms], world, dev)[0], e2e_steps, h2d, d2h)
    if with_cpu and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(wl, out_dtype)
    return res


def decode_roofline(r, peak, peak_kind, traffic):
    achieved = r["dec_b"] / (r["decode_ms"] * 1e-3) / 1e9
    return {"bound": "hbm",
            "kernel": ("paged_attention_decode_shared_prefix" if r["shared"] else
                       "paged_attention_decode (+ LSE reduce)"),
            "achieved": round(achieved, 2), "peak": peak,
            "peak_kind": f"{peak_kind} (hbm_gbs, copy burst)", "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "algorithmic_bytes_per_launch": r["dec_b"],
            "launch_ms": round(r["decode_ms"], 5)}


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = W.CONFIGS[args.config]
    if args.block_size:
        cfg = cfg.scaled(block_size=args.block_size)
    part = args.partition if args.partition is not None else cfg.partition_size
    r = decode_case(cfg, dev, args, world, rank, args.decode, part, with_e2e=True,
                    with_cpu=(rank == 0))
    extra = {}
    if args.config == DEFAULT_CONFIG and not args.no_configs and not args.block_size and \
            args.partition is None:
        extra = other_configs(dev, args, world, rank)
    if rank != 0:
        return None
    wl, out_dtype = r["wl"], r["out_dtype"]
    peak, peak_kind = measured_peak()
    ms_per_step = r["elapsed_ms"] / args.steps
    value = whole_job_gbs(r["step_bytes"], world, args.steps, r["elapsed_ms"])
    e2e_ms, e2e_steps, h2d, d2h = r["e2e"]
    L = wl.seq_lens.numpy().astype(np.int64)
    n_seqs = len(L)
    traffic_key = args.config if args.decode != "standard" or wl.group_starts is None \
        else args.config + "_per_sequence"
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "kv_dtype": cfg.cache_dtype, "data": "synthetic",
        "config": {"workload": f"{args.config}: {DESCR[args.config]}",
                   "block_size": cfg.block_size,
                   "partition_tokens": r["part_eff"], "out_dtype": out_dtype,
                   "l2": "no flush: inputs larger than L2 (%.2f GB read per step vs 126 MB L2)"
                         % (r["dec_b"] / 1e9),
                   "parallelism": f"replicas x{world}",
                   "timing": timing_note(args)},
        "pct_of_peak": round(100.0 * value / peak, 2),
        "decode_tokens_per_s_per_layer": round(n_seqs * world / (ms_per_step * 1e-3), 1),
        "context_tokens_per_s_per_layer": round(int(L.sum()) * world / (ms_per_step * 1e-3), 1),
        "roofline": decode_roofline(r, peak, peak_kind,
                                    None if args.block_size or args.partition is not None
                                    else recorded_traffic(traffic_key)),
        "e2e": {"value": round(whole_job_gbs(r["step_bytes"], world, e2e_steps, e2e_ms), 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": round(e2e_ms / e2e_steps, 5)},
        "gpu_launches": r["launches"] * args.steps,
        "clocks": r["clocks"],
    }
    if wl.prefix_key is not None:
        logical = decode_bytes(wl, out_dtype)
        line["decode_bytes"] = {"distinct": r["dec_b"] if r["shared"] else
                                shared_decode_bytes(wl, out_dtype),
                                "per_sequence": logical,
                                "per_sequence_gbs": round(logical / (r["decode_ms"] * 1e-3) / 1e9,
                                                          2)}
        line["config"]["decode"] = "shared-prefix" if r["shared"] else "per-sequence"
    if "cpu_baseline" in r:
        line["cpu_baseline"] = r["cpu_baseline"]
    if extra:
        line["configs"] = extra
    return line


def decode_entry(name, r, steps, world, peak, peak_kind, traffic_key):
    """The `configs` map entry of one decode workload (rank 0)."""
    wl = r["wl"]
    ms_per_step = r["elapsed_ms"] / steps
    L = wl.seq_lens.numpy().astype(np.int64)
    roof = decode_roofline(r, peak, peak_kind, recorded_traffic(traffic_key))
    e = {"workload": f"{name}: {DESCR[name]}",
         "decode": ("shared-prefix" if r["shared"] else "per-sequence"),
         "launch_ms": roof["launch_ms"], "algorithmic_bytes_per_launch": r["dec_b"],
         "achieved_gbs": roof["achieved"], "frac": roof["frac"], "peak": peak,
         "peak_kind": roof["peak_kind"], "traffic": roof["traffic"],
         "step_value": round(whole_job_gbs(r["step_bytes"], world, steps, r["elapsed_ms"]), 2),
         "unit": "GB/s", "ms_per_step": round(ms_per_step, 5), "steps": steps,
         "partition_tokens": r["part_eff"],
         "decode_tokens_per_s_per_layer": round(len(L) * world / (ms_per_step * 1e-3), 1),
         "context_tokens_per_s_per_layer": round(int(L.sum()) * world / (ms_per_step * 1e-3), 1),
         "gpu_launches": r["launches"] * steps, "clocks": r["clocks"]}
    if wl.prefix_key is not None:
        logical = decode_bytes(wl, r["out_dtype"])
        e["per_sequence_bytes"] = logical
        e["per_sequence_gbs"] = round(logical / (r["decode_ms"] * 1e-3) / 1e9, 2)
        e["distinct_bytes"] = r["dec_b"] if r["shared"] else shared_decode_bytes(wl, r["out_dtype"])
    return e


def other_configs(dev, args, world, rank):
    """Every other workload of the benchmark set, each resident in HBM and timed the
    same way (W warm-up + K timed steps, per-launch CUDA events, clocks): the
    70B-shaped GQA decode, the long-context split-K decode, the beam-search
    copy-on-write FP8 step (shared-prefix decode, and the per-sequence decode of
    the same step), the chunked prefill, and the beam pool's block swaps."""
    peak, peak_kind = measured_peak()
    out = {}
    for name, mode, key in (("llama2_70b_gqa", "auto", "llama2_70b_gqa"),
                            ("long_splitk", "auto", "long_splitk"),
                            ("beam_cow_fp8", "shared", "beam_cow_fp8"),
                            ("beam_cow_fp8", "standard", "beam_cow_fp8_per_sequence")):
        r = decode_case(W.CONFIGS[name], dev, args, world, rank, mode, None, with_e2e=False)
        if rank == 0:
            out[key] = decode_entry(name, r, args.steps, world, peak, peak_kind, key)
        del r
        torch.cuda.empty_cache()
    p = prefill_case("chunked_prefill_70b", dev, args, world, rank, with_e2e=False)
    if rank == 0:
        out["chunked_prefill_70b"] = prefill_entry("chunked_prefill_70b", p, args.steps, world)
    del p
    torch.cuda.empty_cache()
    sw = swap_case(dev, args, world, rank)
    if rank == 0:
        out["swap_blocks_beam"] = sw
    torch.cuda.empty_cache()
    return out


def swap_case(dev, args, world, rank):
    """swap_blocks on the beam workload's pool: the 192 copy-on-write blocks of one
    layer (K and V) out to page-locked host memory and back, one launch each way
    (the kernel reads and writes host memory through its mapping), against one
    cudaMemcpyAsync per block and pool; then the swaps on a second stream while the
    shared-prefix decode runs, and the decode's slowdown."""
    import paged_kv_cache_413_b200 as pa

    cfg = W.CONFIGS["beam_cow_fp8"]
    wl = W.make_workload(cfg, seed=cfg.seed + 1000 * rank) if rank else W.make_workload(cfg)
    f = lambda t: t.to(dev)
    kc, vc = f(wl.key_cache), f(wl.value_cache)
    pa.pa_reshape_and_cache(f(wl.prefix_key), f(wl.prefix_value), kc, vc,
                            f(wl.prefix_slot_mapping), k_scale=wl.k_scale, v_scale=wl.v_scale)
    pa.pa_copy_blocks([kc], [vc], f(wl.block_mapping))
    pa.pa_reshape_and_cache(f(wl.new_key), f(wl.new_value), kc, vc, f(wl.slot_mapping),
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    # out: the beams' own blocks (the decode reads them too); in: as many blocks that
    # no sequence owns, so that the swaps never write what the decode reads
    blocks = wl.block_mapping[:, 1].clone()
    n = blocks.numel()
    owned = set(int(b) for b in wl.block_tables.flatten().tolist() if b >= 0)
    free = torch.tensor([b for b in range(wl.num_blocks) if b not in owned][:n])
    if free.numel() < n:
        raise RuntimeError("the beam pool has too few free blocks for the swap measurement")
    host_k = torch.empty((n,) + tuple(kc.shape[1:]), dtype=kc.dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    out_map = torch.stack([blocks, torch.arange(n)], 1).contiguous().to(dev)   # dev -> host
    in_map = torch.stack([torch.arange(n), free], 1).contiguous().to(dev)      # host -> dev
    blocks_d, free_d = blocks.to(dev), free.to(dev)
    block_bytes = kc[0].numel() * kc.element_size()
    moved = 2 * n * block_bytes                                  # K + V, one direction
    side = torch.cuda.Stream(dev)
    main = torch.cuda.current_stream(dev)
    reps = max(5, min(args.steps, 200))

    def swap_pair():
        pa.pa_swap_blocks([host_k], [host_v], [kc], [vc], out_map, stream=side)
        pa.pa_swap_blocks([kc], [vc], [host_k], [host_v], in_map, stream=side)

    src_ids, dst_ids = blocks.tolist(), free.tolist()

    def memcpy_pair():
        with torch.cuda.stream(side):
            for i, b in enumerate(src_ids):
                host_k[i].copy_(kc[b], non_blocking=True)
                host_v[i].copy_(vc[b], non_blocking=True)
            for i, b in enumerate(dst_ids):
                kc[b].copy_(host_k[i], non_blocking=True)
                vc[b].copy_(host_v[i], non_blocking=True)

    def time_on_side(fn, k):
        for _ in range(3):
            fn()
        side.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(side)
        for _ in range(k):
            fn()
        e1.record(side)
        side.synchronize()
        return e0.elapsed_time(e1) / k

    swap_ms = time_on_side(swap_pair, reps)
    kb, vb = kc.view(torch.uint8), vc.view(torch.uint8)
    kb[free_d] = 0x7F                                           # E4M3 NaN: the swap-in must
    vb[free_d] = 0x7F                                           # rewrite every byte
    torch.cuda.synchronize(dev)
    swap_pair()
    side.synchronize()
    if not (torch.equal(kb[free_d], kb[blocks_d]) and torch.equal(vb[free_d], vb[blocks_d])):
        raise RuntimeError("the blocks swapped out and back in differ from the originals")
    memcpy_reps = max(3, min(reps, 20))
    memcpy_ms = time_on_side(memcpy_pair, memcpy_reps)
    torch.cuda.synchronize(dev)

    # overlap: the shared-prefix decode on the main stream, alone and with swaps
    gs, pl = f(wl.group_starts), f(wl.prefix_lens)
    q, bt, sl = f(wl.query), f(wl.block_tables), f(wl.seq_lens)
    outd = torch.empty(q.shape, dtype=TORCH_DT[cfg.out_dtype], device=dev)
    max_len = int(wl.seq_lens.max())
    max_group = int((wl.group_starts[1:] - wl.group_starts[:-1]).max())

    def decode():
        pa.pa_paged_attention_decode_shared_prefix(
            outd, q, kc, vc, bt, sl, gs, pl, max_seq_len=max_len, max_group_size=max_group,
            scale=wl.scale, k_scale=wl.k_scale, v_scale=wl.v_scale)

    def decode_ms(k):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for _ in range(k):
            decode()
        e1.record(main)
        return e0, e1

    for _ in range(3):
        decode()
    torch.cuda.synchronize(dev)
    k_dec = 4 * reps
    a0, a1 = decode_ms(k_dec)
    torch.cuda.synchronize(dev)
    alone = a0.elapsed_time(a1) / k_dec
    # swaps for as long as the decodes run: start them together
    start = torch.cuda.Event()
    start.record(main)
    side.wait_event(start)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(side)
    n_swaps = max(1, int(k_dec * alone / max(swap_ms, 1e-3)))
    for _ in range(n_swaps):
        swap_pair()
    s1.record(side)
    b0, b1 = decode_ms(k_dec)
    torch.cuda.synchronize(dev)
    with_swaps = b0.elapsed_time(b1) / k_dec
    swap_overlap_ms = s0.elapsed_time(s1) / n_swaps
    if pa.pa_get_device_error() != 0:
        raise RuntimeError("device error bits set by the swap measurement")
    vals = max_over_ranks([swap_ms, memcpy_ms, alone, with_swaps, swap_overlap_ms], world, dev)
    swap_ms, memcpy_ms, alone, with_swaps, swap_overlap_ms = vals
    if rank != 0:
        return None
    gbs = lambda ms: round(2 * moved / (ms * 1e-3) / 1e9, 2)
    return {"workload": f"beam_cow_fp8 pool: {n} blocks x (K + V) of {block_bytes} B, out to "
                        "page-locked host memory and back",
            "bytes_per_direction": moved, "unit": "GB/s (host link, both directions)",
            "swap_blocks_ms": round(swap_ms, 5), "swap_blocks_gbs": gbs(swap_ms),
            "per_block_memcpy_ms": round(memcpy_ms, 5), "per_block_memcpy_gbs": gbs(memcpy_ms),
            "per_block_memcpy_calls": 4 * n,
            "overlap": {"decode_ms_alone": round(alone, 5),
                        "decode_ms_with_swaps": round(with_swaps, 5),
                        "decode_slowdown": round(with_swaps / alone, 4),
                        "swap_blocks_gbs_during_decode": gbs(swap_overlap_ms),
                        "swaps_on": "a second stream, launched together with the decodes"},
            "gpu_launches": 2 * (reps + 4) + 2 * n_swaps + 2 * k_dec + 6}


def prefill_flops(wl: W.Workload) -> int:
    """Causal attention FLOPs: 4 * D per (query head, visible key) pair (QK and PV)."""
    cfg = wl.cfg
    L = wl.seq_lens.numpy().astype(np.int64)
    qs = wl.query_start.numpy().astype(np.int64)
    pairs = 0
    for i in range(len(L)):
        n = qs[i + 1] - qs[i]
        pos = L[i] - n + np.arange(n)
        pairs += int((pos + 1).sum())
    return pairs * cfg.num_heads * cfg.head_dim * 4


# A timed region at least this long is a sustained run: its tensor-core kernel is
# held against the sustained peak (cuBLAS back to back for seconds, under the power
# cap), a shorter one against the burst peak.
SUSTAINED_REGION_S = 1.0


def tensor_peaks():
    """(burst, sustained) dense bf16 TFLOP/s and their description."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            m = json.load(fh)
        return (float(m["bf16_tflops"]), float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "measured")
    except Exception:
        return 1590.0, 1400.0, "fallback"


def prefill_case(name, dev, args, world, rank, with_e2e=True, with_cpu=False):
    """The multi-query (chunked prefill) step: cache write of the chunks + attention."""
    import paged_kv_cache_413_b200 as pa

    spec = dict(PREFILL[name])
    spec["seed"] += 1000 * rank
    wl = W.make_prefill_workload(spec.pop("num_seqs"), spec.pop("context"), spec.pop("chunk"),
                                 **spec)
    f = lambda t: t.to(dev)
    kc, vc, q, bt, sl = f(wl.key_cache), f(wl.value_cache), f(wl.query), f(wl.block_tables), \
        f(wl.seq_lens)
    nk, nv, sm, qs = f(wl.new_key), f(wl.new_value), f(wl.slot_mapping), f(wl.query_start)
    out = torch.empty_like(q)
    max_q = int((wl.query_start[1:] - wl.query_start[:-1]).max())
    max_len = int(wl.seq_lens.max())
    stream = torch.cuda.current_stream(dev)
    ev = []
    inputs = {"q": q, "nk": nk, "nv": nv, "sm": sm, "bt": bt, "sl": sl, "qs": qs}

    def writes(t):
        pa.pa_reshape_and_cache(t["nk"], t["nv"], kc, vc, t["sm"])

    def attend(t, out_t):
        pa.pa_paged_attention_prefill(out_t, t["q"], kc, vc, t["bt"], t["sl"], t["qs"],
                                      max_query_len=max_q, max_seq_len=max_len, scale=wl.scale)

    def run_step(t, out_t, timed=False):
        writes(t)
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        attend(t, out_t)
        if timed:
            e1.record(stream)
            ev.append((e0, e1))

    step, writes_step = graph_step(lambda: writes(inputs), lambda: attend(inputs, out),
                                   run_step, inputs, out, ev, dev, stream, args)
    elapsed_ms, kern_ms, clocks = timed_loop(step, ev, args.steps, args.warmup, dev, stream,
                                             world, rank, writes_step)
    cfg = wl.cfg
    L = wl.seq_lens.numpy().astype(np.int64)
    res = {"wl": wl, "elapsed_ms": elapsed_ms, "kern_ms": kern_ms, "clocks": clocks,
           "flops": prefill_flops(wl), "max_q": max_q,
           "kv_bytes": int(L.sum()) * cfg.num_kv_heads * cfg.head_dim * 2 * 2,
           "qo_bytes": 2 * q.numel() * 2, "query_tokens": int(wl.query_start[-1])}
    if with_e2e:
        host_src = {"q": wl.query, "nk": wl.new_key, "nv": wl.new_value, "sm": wl.slot_mapping,
                    "bt": wl.block_tables, "sl": wl.seq_lens, "qs": wl.query_start}
        e2e_steps = max(10, args.steps // 4)
        e2e_ms, h2d, d2h = pipelined_e2e(dev, stream, inputs, host_src, out, run_step,
                                         e2e_steps, world)
        res["e2e"] = (max_over_ranks([e2e_ms], world, dev)[0], e2e_steps, h2d, d2h)
    if with_cpu and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = prefill_cpu_baseline(wl)
    return res


def prefill_roofline(name, p):
    cfg = p["wl"].cfg
    burst, sustained, src = tensor_peaks()
    region_s = p["elapsed_ms"] * 1e-3
    if region_s >= SUSTAINED_REGION_S:
        peak = sustained
        kind = (f"{src} (bf16_tflops_sustained, cuBLAS back to back under the power cap: the "
                f"timed region ran {region_s:.1f} s of back-to-back steps)")
    else:
        peak = burst
        kind = f"{src} (bf16_tflops, cuBLAS burst: the timed region ran {region_s:.2f} s)"
    # the launcher's rule: 128-row tcgen05 tiles once a chunk fills one, two of them
    # in ping-pong once a (sequence, kv head) has two
    rows = p["max_q"] * (cfg.num_heads // cfg.num_kv_heads)
    kernel = ("prefill_pp_kernel (tcgen05.mma, two tiles in ping-pong, TMEM accumulators)"
              if rows > 128 else
              "prefill_tc_kernel (tcgen05.mma, TMEM accumulators)" if rows == 128 else
              "prefill_kernel (mma.sync m16n8k16)")
    achieved = p["flops"] / (p["kern_ms"] * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 2), "peak": peak,
            "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "frac_of_burst": round(achieved / burst, 4),
            "traffic": recorded_traffic(name), "launch_ms": round(p["kern_ms"], 5),
            "flops_per_launch": p["flops"],
            "hbm_gbs": round((p["kv_bytes"] + p["qo_bytes"]) / (p["kern_ms"] * 1e-3) / 1e9, 1)}


def prefill_entry(name, p, steps, world):
    roof = prefill_roofline(name, p)
    return {"workload": f"{name}: {DESCR[name]}", "launch_ms": roof["launch_ms"],
            "flops_per_launch": p["flops"], "achieved_tflops": roof["achieved"],
            "frac": roof["frac"], "frac_of_burst": roof["frac_of_burst"], "peak": roof["peak"],
            "peak_kind": roof["peak_kind"], "traffic": roof["traffic"], "kernel": roof["kernel"],
            "step_value": round(p["flops"] * world * steps / (p["elapsed_ms"] * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "ms_per_step": round(p["elapsed_ms"] / steps, 5), "steps": steps,
            "gpu_launches": 2 * steps, "clocks": p["clocks"]}


def run_prefill(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    p = prefill_case(args.config, dev, args, world, rank, with_e2e=True, with_cpu=(rank == 0))
    if rank != 0:
        return None
    flops = p["flops"]
    e2e_ms, e2e_steps, h2d, d2h = p["e2e"]
    tflops = flops * world * args.steps / (p["elapsed_ms"] * 1e-3) / 1e12
    return {"metric": "paged multi-query attention (chunked prefill): TFLOP/s", "value":
            round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(p["elapsed_ms"] / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"{args.config}: {DESCR[args.config]}",
                       "query_tokens": p["query_tokens"], "flops_per_step": flops,
                       "l2": f"KV read {p['kv_bytes'] / 1e6:.0f} MB per step, above the 126 MB L2",
                       "timing": timing_note(args)},
            "roofline": prefill_roofline(args.config, p),
            "e2e": {"value": round(flops * world * e2e_steps / (e2e_ms * 1e-3) / 1e12, 2),
                    "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": round(e2e_ms / e2e_steps, 5)},
            "cpu_baseline": p.get("cpu_baseline"),
            "gpu_launches": 2 * args.steps,
            "clocks": p["clocks"]}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step a bounded sample (one sequence)."""
    if rank != 0:
        return None
    import oracle

    cfg = W.CONFIGS[args.config]
    wl = W.make_workload(cfg)
    n = wl.seq_lens.numel()
    order = np.random.default_rng(0).permutation(n)
    for i in range(args.warmup):
        oracle_sample(wl, order[i % n:i % n + 1], cfg.out_dtype)
    total_t, total_b = 0.0, 0
    for i in range(args.steps):
        dt, b = oracle_sample(wl, order[i % n:i % n + 1], cfg.out_dtype)
        total_t += dt
        total_b += b
    v = total_b / total_t / 1e9
    return {"metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{args.config}: {DESCR[args.config]}",
                       "sample_per_step": "one sequence (its cache write + fp64 decode)"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"one of {n} sequences per step, {args.steps} steps"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(W.CONFIGS) + sorted(PREFILL))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=None)
    ap.add_argument("--block-size", type=int, default=0,
                    help="tokens per physical block (default: the workload's, 16)")
    ap.add_argument("--decode", default="auto", choices=["auto", "shared", "standard"],
                    help="copy-on-write workloads: shared-prefix decode (auto) or per sequence")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graphs", action="store_true",
                    help="timed steps call the library directly instead of replaying CUDA "
                         "graphs of the same calls")
    ap.add_argument("--no-configs", action="store_true",
                    help="default workload only: skip the `configs` map of the other workloads")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime

            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group(
                "nccl", timeout=datetime.timedelta(seconds=120),
                device_id=torch.device("cuda", local_rank))
        try:
            if args.config in PREFILL:
                line = run_prefill(args, rank, world, local_rank)
            else:
                line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
