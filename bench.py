#!/usr/bin/env python3
"""Paged decode attention benchmark (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config qwen]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]

A step is one decode step of the whole workload: for each of the 16 layers,
the cache write of every sequence's new token (pa_reshape_and_cache) then the
paged attention (pa_decode_attention), each layer with its own K/V pool, on
seeded synthetic data already resident in device memory.  Metric: attention
bytes (query read + KV read + output write) per step over the step time, in
GB/s, summed over ranks; also decode tokens/s per layer.

With N > 1 (one process per GPU under torch.distributed.run) each rank runs
its own batch of the same shape (a data-parallel shard drawn with its own
seed): the path has no exchange step, so there is no collective on the data
path; the step time is the maximum over ranks.

--impl reference times the CPU oracle (fp64, OpenMP) on a bounded sample of
the same workload on rank 0 and prints the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_455_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention achieved HBM GB/s (% of 8 TB/s); decode tokens/s/layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_kernel_qwen.md")
PREFILL_PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "prefill_tc_kernel_chunk512.md")
CSRC = os.path.join(ROOT, "paged_kv_cache_455_b200", "csrc")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def attention_bytes(layout: W.BatchLayout) -> int:
    """Bytes the method must move per layer: Q read + KV read + output write."""
    cfg = layout.config
    s = cfg.elem_size
    qo = 2 * cfg.num_seqs * cfg.num_q_heads * cfg.head_dim * s
    kv = int(layout.context_lens.astype(np.int64).sum()) * 2 * cfg.num_kv_heads * cfg.head_dim * s
    return qo + kv


# the sources each profiled kernel is built and launched from
DECODE_SOURCES = ("pa.cu", "pa_inst_bf16.cu", "pa_kernels.cuh", "pa_launch.cuh", "pa_ptx.cuh")
PREFILL_SOURCES = ("pa.cu", "pa_inst_prefill.cu", "pa_launch.cuh", "pa_prefill.cuh",
                   "pa_prefill_tc.cuh", "pa_ptx.cuh")


def kernel_source_hash(sources=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    for f in sorted(sources):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(summary=PROFILE_SUMMARY, sources=DECODE_SOURCES):
    """DRAM bytes per launch of a kernel from its committed ncu summary (the
    decode kernel's by default), or None if its sources changed since."""
    try:
        text = open(summary).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash(sources):
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self.period = period_s

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self._nvml is None or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the measured arm
# ---------------------------------------------------------------------------

class Workload:
    def __init__(self, cfg: W.DecodeConfig, device, shard: int, length_scale: float = 1.0,
                 layers=None):
        from paged_kv_cache_455_b200 import pa
        self.pa = pa
        self.cfg = cfg
        self.device = device
        self.layout = W.make_layout(cfg, length_scale=length_scale, shard=shard)
        self.layers = W.make_layers(self.layout, device, layers=layers)
        self.tables, self.lens, self.slots = W.device_metadata(self.layout, device)
        L = self.layout
        nbytes = pa.pa_decode_workspace_bytes(cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim,
                                              L.max_context_len)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.outs = [torch.empty_like(l.query) for l in self.layers]
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def attention(self, i, tables=None, lens=None):
        pa, l, L = self.pa, self.layers[i], self.layout
        pa.pa_decode_attention(self.outs[i], l.query, l.k_pool, l.v_pool,
                               self.tables if tables is None else tables,
                               self.lens if lens is None else lens, L.max_context_len,
                               self.cfg.scale, self.workspace, self.status)

    def layer_step(self, i, tables=None, lens=None, slots=None):
        l = self.layers[i]
        self.pa.pa_reshape_and_cache(l.key, l.value, l.k_pool, l.v_pool,
                                     self.slots if slots is None else slots, self.status)
        self.attention(i, tables, lens)

    def step(self):
        for i in range(len(self.layers)):
            self.layer_step(i)


def run_ours(args, rank, world, device, dist):
    from paged_kv_cache_455_b200 import pa
    cfg = W.CONFIGS[args.config]
    length_scale = 1.0
    if cfg.name == "pressure":
        free, _ = torch.cuda.mem_get_info(device)
        length_scale = W.fit_length_scale(cfg, free)
    wl = Workload(cfg, device, shard=rank, length_scale=length_scale, layers=args.layers)
    L = wl.layout
    nl = len(wl.layers)
    bytes_layer = attention_bytes(L)
    torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize(device)
    if int(wl.status.item()) != 0:
        raise RuntimeError(f"device status {int(wl.status.item())} during warm-up")

    # ---- one decode step (every layer: cache write then attention) and the
    # attention calls alone, each captured once as a CUDA graph and replayed;
    # the library launches on the current stream, which is the capture stream
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    step_graph, attn_graph = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        wl.step()
        torch.cuda.synchronize(device)
        l0 = pa.launch_count()
        with torch.cuda.graph(step_graph, stream=side):
            wl.step()
        launches_per_step = pa.launch_count() - l0
        with torch.cuda.graph(attn_graph, stream=side):
            for i in range(nl):
                wl.attention(i)
    torch.cuda.synchronize(device)
    for _ in range(2):
        step_graph.replay()
        attn_graph.replay()
    torch.cuda.synchronize(device)

    # ---- timed region: K replays of the step graph, device events, clocks
    # sampled meanwhile
    stream = torch.cuda.current_stream(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t0.record(stream)
        for _ in range(args.steps):
            step_graph.replay()
        t1.record(stream)
        torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    launches = launches_per_step * args.steps
    ms_total = t0.elapsed_time(t1)

    # ---- attention alone (the roofline's kernel): K replays of the
    # attention graph, events on the same stream
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        attn_graph.replay()
    a1.record(stream)
    torch.cuda.synchronize(device)
    attn_ms_mean = a0.elapsed_time(a1) / (args.steps * nl)

    # ---- the same step launched eagerly (host overhead included), for context
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(max(3, args.steps // 4)):
        wl.step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    eager_ms = e0.elapsed_time(e1) / max(3, args.steps // 4)
    del step_graph, attn_graph

    # max over ranks of the step time, sum over ranks of the work
    ms_per_step, attn_ms_worst, step_bytes_all, seqs_all = combine_ranks(
        dist, device, ms_total / args.steps, attn_ms_mean, bytes_layer * nl, cfg.num_seqs)
    if int(wl.status.item()) != 0:
        raise RuntimeError(f"device status {int(wl.status.item())} in the timed region")

    value = step_bytes_all / (ms_per_step * 1e-3) / 1e9
    t_layer_s = ms_per_step * 1e-3 / nl
    tokens_per_s_layer = seqs_all / t_layer_s

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, args, device, dist, world, bytes_layer)

    peak, peak_kind = measured_peak()
    achieved = bytes_layer / (attn_ms_mean * 1e-3) / 1e9
    traffic = profiled_traffic()

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) Q/K/V, seeded lengths and block tables)",
        "config": {
            "workload": f"{cfg.name}: {cfg.description}",
            "layers": nl, "num_seqs_per_gpu": cfg.num_seqs, "num_q_heads": cfg.num_q_heads,
            "num_kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
            "block_size": cfg.block_size, "sum_context_lens_per_gpu": int(L.context_lens.sum()),
            "max_context_len": L.max_context_len, "length_scale": length_scale,
            "parallelism": f"dp{world} (independent shards, no collective)",
            "l2": "no flush: every step streams each layer's own pool (far above the 126 MB L2)",
        },
        "pct_of_8tbs_per_gpu": round(100 * value / (NOMINAL_HBM_GBS * world), 2),
        "tokens_per_s_per_layer": round(tokens_per_s_layer, 1),
        "attention_only_gbs_per_gpu": round(achieved, 1),
        "timing": "each step replays one CUDA graph of all layers (cache write + attention); "
                  "eager launches of the same step take %.4f ms" % eager_ms,
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "peak_source": f"{peak_kind} HBM copy bandwidth",
            "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": "pa_decode_attention (decode_kernel, one launch per layer), replayed in a graph",
            "algorithmic_bytes_per_launch": bytes_layer,
            "launch_ms_mean": round(attn_ms_mean, 5), "launch_ms_worst_rank": round(attn_ms_worst, 5),
        },
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, L, wl.layers[0], budget_s=args.cpu_seconds)
    return out


def combine_ranks(dist, device, ms_per_step, attn_ms, step_bytes, seqs):
    """Maximum of the times and sum of the work over the ranks of `dist`
    (no process group: the values as they are).  Every rank calls it."""
    if dist is None:
        return ms_per_step, attn_ms, float(step_bytes), float(seqs)
    t = torch.tensor([ms_per_step, attn_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([float(step_bytes), float(seqs)], dtype=torch.float64, device=device)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t[0]), float(t[1]), float(w[0]), float(w[1])


def run_e2e(wl: Workload, args, device, dist, world, bytes_layer):
    """Same metric through the public API with host (pinned) buffers: each
    step copies every layer's query / new key / new value and the batch
    metadata host->device, runs the 16 layers, and copies every output back."""
    L, cfg = wl.layout, wl.cfg
    host_q = [l.query.cpu().pin_memory() for l in wl.layers]
    host_k = [l.key.cpu().pin_memory() for l in wl.layers]
    host_v = [l.value.cpu().pin_memory() for l in wl.layers]
    host_tab = torch.from_numpy(L.block_tables).pin_memory()
    host_len = torch.from_numpy(L.context_lens).pin_memory()
    host_slot = torch.from_numpy(L.slot_mapping).pin_memory()
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in wl.outs]
    dev_tab, dev_len, dev_slot = (torch.empty_like(wl.tables), torch.empty_like(wl.lens),
                                  torch.empty_like(wl.slots))
    h2d = sum(t.numel() * t.element_size() for t in host_q + host_k + host_v) + \
        sum(t.numel() * t.element_size() for t in (host_tab, host_len, host_slot))
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def step():
        dev_tab.copy_(host_tab, non_blocking=True)
        dev_len.copy_(host_len, non_blocking=True)
        dev_slot.copy_(host_slot, non_blocking=True)
        for i, l in enumerate(wl.layers):
            l.query.copy_(host_q[i], non_blocking=True)
            l.key.copy_(host_k[i], non_blocking=True)
            l.value.copy_(host_v[i], non_blocking=True)
            wl.layer_step(i, dev_tab, dev_len, dev_slot)
            host_out[i].copy_(wl.outs[i], non_blocking=True)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    steps = max(3, args.steps // 2)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / steps
    if dist is not None:
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t[0])
    value = world * bytes_layer * len(wl.layers) / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline arm)
# ---------------------------------------------------------------------------

def _oracle_sample(cfg, layout, layer, seqs):
    from oracle import oracle as O
    s = W.compact_sample(layout, layer, seqs)
    k, v = O.reshape_and_cache(s["key"], s["value"], s["k_pool"], s["v_pool"], s["slot_mapping"],
                               cfg.dtype)
    return s, k, v


def _time_oracle(cfg, s, k, v, threads):
    from oracle import oracle as O
    t = time.perf_counter()
    O.paged_attention(s["query"], k, v, s["block_tables"], s["context_lens"], cfg.scale,
                      cfg.dtype, num_threads=threads)
    return time.perf_counter() - t


def cpu_baseline(cfg, layout, layer, budget_s=10.0, threads=0):
    """Times the oracle (as it stands) on host cores on a bounded sample of one
    layer's sequences: the first n sequences, n grown until the run takes
    about budget_s / 4, then that sample is repeated to ~budget_s."""
    from oracle import oracle as O
    nthreads = O.threads(threads)
    n = min(cfg.num_seqs, max(1, nthreads))
    while True:
        seqs = np.arange(n)
        s, k, v = _oracle_sample(cfg, layout, layer, seqs)
        dt = _time_oracle(cfg, s, k, v, threads)
        if dt >= budget_s / 4 or n == cfg.num_seqs:
            break
        n = min(cfg.num_seqs, max(n + 1, int(n * min(8.0, (budget_s / 4) / max(dt, 1e-3)))))
    reps = min(100, max(1, int(round(budget_s / max(dt, 1e-3)))))
    total = dt
    for _ in range(reps - 1):
        total += _time_oracle(cfg, s, k, v, threads)
    runs = reps
    sample_layout = W.BatchLayout(cfg, s["context_lens"], s["block_tables"], s["slot_mapping"],
                                  int(k.shape[0]))
    nbytes = attention_bytes(sample_layout)
    secs = total / runs
    return {
        "value": round(nbytes / secs / 1e9, 3), "unit": "GB/s",
        "cores": int(min(nthreads, n)), "threads_requested": int(nthreads),
        "kind": "oracle",
        "sample": f"layer 0, first {n} of {cfg.num_seqs} sequences "
                  f"({int(s['context_lens'].sum())} tokens), fp64 C oracle with OpenMP over "
                  f"sequences, {runs} run(s) of {secs:.2f} s",
        "tokens_per_s_per_layer": round(n / secs, 2),
    }


def run_reference(args, rank, world, device):
    cfg = W.CONFIGS[args.config]
    layout = W.make_layout(cfg)
    (layer,) = W.make_layers(layout, device, layers=1)
    from oracle import oracle as O
    nthreads = O.threads(0)
    # each step: the oracle over a bounded sample of the workload's sequences
    n = min(cfg.num_seqs, max(1, nthreads))
    seqs = np.arange(n)
    s, k, v = _oracle_sample(cfg, layout, layer, seqs)
    while n < cfg.num_seqs and _time_oracle(cfg, s, k, v, 0) < args.cpu_seconds / 10:
        n = min(cfg.num_seqs, 2 * n)
        s, k, v = _oracle_sample(cfg, layout, layer, np.arange(n))
    for _ in range(args.warmup):
        _time_oracle(cfg, s, k, v, 0)
    times = [_time_oracle(cfg, s, k, v, 0) for _ in range(args.steps)]
    secs = float(np.mean(times))
    sample_layout = W.BatchLayout(cfg, s["context_lens"], s["block_tables"], s["slot_mapping"],
                                  int(k.shape[0]))
    nbytes = attention_bytes(sample_layout)
    value = nbytes / secs / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{cfg.name}: {cfg.description}",
                   "sample": f"layer 0, first {n} of {cfg.num_seqs} sequences per step"},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "kind": "oracle",
                         "cores": int(min(nthreads, n)),
                         "sample": f"layer 0, first {n} of {cfg.num_seqs} sequences "
                                   f"({int(s['context_lens'].sum())} tokens) per step"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "tokens_per_s_per_layer": round(n / secs, 2),
    }
    return line


# ---------------------------------------------------------------------------
# chunked prefill (--path prefill)
# ---------------------------------------------------------------------------

PREFILL_METRIC = "chunked-prefill paged attention TFLOP/s (causal flops)"


def prefill_workload(device, layers: int, seed: int = 455 + 6):
    """Qwen-shaped heads (Hq=16, Hkv=4, d=256, bs=16, bf16): B=16 sequences whose
    contexts are uniform in [1024, 4096] tokens, each ending with a 512-token
    chunk (the pages' example chunk size), one pool per layer."""
    rng = np.random.default_rng(seed)
    B, hq, hkv, d, bs, chunk = 16, 16, 4, 256, 16, 512
    lens = rng.integers(1024, 4097, size=B).astype(np.int32)
    need = -(-lens // bs)
    nb = int(need.sum()) + 64
    perm = rng.permutation(nb)
    tables = np.full((B, int(need.max())), -1, np.int32)
    pos = 0
    for b in range(B):
        tables[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    slots = np.concatenate([tables[b][np.arange(lens[b] - chunk, lens[b]) // bs] * bs +
                            np.arange(lens[b] - chunk, lens[b]) % bs for b in range(B)])
    cu = np.arange(B + 1, dtype=np.int32) * chunk
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    L = []
    for _ in range(layers):
        kp = torch.randn(nb, bs, hkv, d, generator=g, device=device).to(torch.bfloat16)
        vp = torch.randn(nb, bs, hkv, d, generator=g, device=device).to(torch.bfloat16)
        q = torch.randn(B * chunk, hq, d, generator=g, device=device).to(torch.bfloat16)
        key = torch.randn(B * chunk, hkv, d, generator=g, device=device).to(torch.bfloat16)
        val = torch.randn(B * chunk, hkv, d, generator=g, device=device).to(torch.bfloat16)
        L.append((q, key, val, kp, vp, torch.empty_like(q)))
    dev = dict(tables=torch.from_numpy(tables).to(device), lens=torch.from_numpy(lens).to(device),
               slots=torch.from_numpy(slots.astype(np.int64)).to(device),
               cu=torch.from_numpy(cu).to(device))
    flops = 0
    for b in range(B):
        keys = np.arange(lens[b] - chunk, lens[b], dtype=np.int64) + 1   # keys per row (causal)
        flops += 4 * d * hq * int(keys.sum())
    nbytes = 2 * B * chunk * hq * d * 2 + int(lens.astype(np.int64).sum()) * 2 * hkv * d * 2
    meta = dict(B=B, hq=hq, hkv=hkv, d=d, bs=bs, chunk=chunk, lens=lens, tables=tables, cu=cu,
                flops=flops, bytes=nbytes, scale=1.0 / 16.0)
    return L, dev, meta


def run_prefill(args, device):
    from paged_kv_cache_455_b200 import pa
    layers = args.layers or 4
    L, dev, meta = prefill_workload(device, layers)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    maxctx = int(meta["lens"].max())

    def attend(i):
        q, _, _, kp, vp, out = L[i]
        pa.pa_prefill_attention(out, q, dev["cu"], meta["chunk"], kp, vp, dev["tables"],
                                dev["lens"], maxctx, meta["scale"], status)

    def step():
        for i in range(layers):
            q, key, val, kp, vp, _ = L[i]
            pa.pa_reshape_and_cache(key, val, kp, vp, dev["slots"], status)
            attend(i)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")
    stream = torch.cuda.current_stream(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = pa.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(device)
    launches = pa.launch_count() - l0
    ms_step = t0.elapsed_time(t1) / args.steps
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        for i in range(layers):
            attend(i)
    a1.record(stream)
    torch.cuda.synchronize(device)
    attn_ms = a0.elapsed_time(a1) / (args.steps * layers)
    tflops = meta["flops"] / (attn_ms * 1e-3) / 1e12
    step_tflops = meta["flops"] * layers / (ms_step * 1e-3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 burst"
    except Exception:
        peak, src = 1590.0, "fallback"
    line = {
        "metric": PREFILL_METRIC, "value": round(step_tflops, 2), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V, seeded lengths and block tables)",
        "config": {"workload": "prefill: B=16 sequences, contexts U[1024,4096], each ending "
                               "with a 512-token chunk, Hq=16, Hkv=4, d=256, block 16, bf16",
                   "layers": layers, "l2": "no flush: each layer has its own pool"},
        "attention_tflops": round(tflops, 2),
        "attention_gbs": round(meta["bytes"] / (attn_ms * 1e-3) / 1e9, 1),
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "peak_source": src, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "traffic": profiled_traffic(PREFILL_PROFILE_SUMMARY, PREFILL_SOURCES),
                     "kernel": "pa_prefill_attention (prefill_tc_kernel<256, 4>: tcgen05.mma, "
                               "TMEM accumulators)",
                     "algorithmic_bytes_per_launch": meta["bytes"],
                     "algorithmic_flops_per_launch": meta["flops"],
                     "launch_ms_mean": round(attn_ms, 5)},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        q, _, _, kp, vp, _ = L[0]
        b = 0
        cu1 = np.array([0, meta["chunk"]])
        qs = W.to_numpy_elems(q[:meta["chunk"]])
        kp_h, vp_h = W.to_numpy_elems(kp), W.to_numpy_elems(vp)
        tt = time.perf_counter()
        O.prefill_attention_np(qs, kp_h, vp_h, meta["tables"][b:b + 1], meta["lens"][b:b + 1],
                               cu1, meta["scale"], "bf16")
        secs = time.perf_counter() - tt
        keys = np.arange(meta["lens"][b] - meta["chunk"], meta["lens"][b], dtype=np.int64) + 1
        f1 = 4 * meta["d"] * meta["hq"] * int(keys.sum())
        line["cpu_baseline"] = {"value": round(f1 / secs / 1e12, 6), "unit": "TFLOP/s",
                                "cores": os.cpu_count(), "kind": "oracle",
                                "sample": f"layer 0, sequence 0 (one 512-token chunk over "
                                          f"{int(meta['lens'][0])} tokens), numpy fp64 oracle, "
                                          f"{secs:.2f} s"}
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="qwen", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: the workload's 16); fewer only for profiling")
    ap.add_argument("--path", default="decode", choices=["decode", "prefill"],
                    help="decode (the default measurement) or the chunked-prefill path")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only
        if rank != 0:
            return 0
        device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
        print(json.dumps(run_reference(args, rank, world, device)), flush=True)
        return 0

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl ours needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=device)
        dist = tdist
    if args.path == "prefill":
        if world != 1:
            raise SystemExit("--path prefill runs on one GPU")
        print(json.dumps(run_prefill(args, device)), flush=True)
        return 0
    try:
        line = run_ours(args, rank, world, device, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
