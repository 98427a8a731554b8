#!/usr/bin/env python3
"""Paged decode attention benchmark (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]

A step is one decode step of the whole workload: for each of the 16 layers,
the cache write of every sequence's new token (pa_reshape_and_cache) then the
paged attention (pa_decode_attention), each layer with its own K/V pool, on
seeded synthetic data already resident in device memory.  Metric: attention
bytes (query read + KV read + output write) per step over the step time, in
GB/s, summed over ranks; also decode tokens/s per layer.

Without --config the line's headline is the memory-pressure workload (B=512,
~120 GB of pools, the largest that fits one GPU), with its end-to-end
number and the CPU oracle beside it; `per_config` holds the same
measurement for the Qwen-shaped, long-context and continuous-batch
workloads (and their FP8-cache variants), and `prefill` the chunked-prefill
path.  --config NAME measures that one workload as the headline.

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
# the default run: the largest single-GPU workload as the headline, the others
# (the long-context and mixed-batch ones among them) as per-config records
HEADLINE = "pressure"
PER_CONFIG = ("qwen", "long", "mix")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def attention_bytes(layout: W.BatchLayout, kv_elem: int = 0) -> int:
    """Bytes the method must move per layer: Q read + KV read + output write
    (KV elements of kv_elem bytes; 0: the config's element size)."""
    cfg = layout.config
    s = cfg.elem_size
    kv_elem = kv_elem or s
    qo = 2 * cfg.num_seqs * cfg.num_q_heads * cfg.head_dim * s
    kv = int(layout.context_lens.astype(np.int64).sum()) * 2 * cfg.num_kv_heads * cfg.head_dim * kv_elem
    return qo + kv


# the sources each profiled kernel is built and launched from
DECODE_SOURCES = ("pa.cu", "pa_inst_bf16.cu", "pa_kernels.cuh", "pa_launch.cuh", "pa_ptx.cuh")
DECODE8_SOURCES = DECODE_SOURCES + ("pa_inst_fp8.cu",)
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
                 layers=None, fp8: bool = False):
        from paged_kv_cache_455_b200 import pa
        self.pa = pa
        self.cfg = cfg
        self.device = device
        self.fp8 = fp8
        self.layout = W.make_layout(cfg, length_scale=length_scale, shard=shard)
        self.layers = (W.make_layers_fp8 if fp8 else W.make_layers)(self.layout, device,
                                                                    layers=layers)
        self.tables, self.lens, self.slots = W.device_metadata(self.layout, device)
        L = self.layout
        nbytes = pa.pa_decode_workspace_bytes(cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim,
                                              L.max_context_len)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.outs = [torch.empty_like(l.query) for l in self.layers]
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def attention(self, i, tables=None, lens=None):
        pa, l, L = self.pa, self.layers[i], self.layout
        tables = self.tables if tables is None else tables
        lens = self.lens if lens is None else lens
        if self.fp8:
            pa.pa_decode_attention_fp8(self.outs[i], l.query, l.k_pool, l.v_pool, tables, lens,
                                       L.max_context_len, self.cfg.scale, W.FP8_SCALE,
                                       W.FP8_SCALE, self.workspace, self.status)
        else:
            pa.pa_decode_attention(self.outs[i], l.query, l.k_pool, l.v_pool, tables, lens,
                                   L.max_context_len, self.cfg.scale, self.workspace, self.status)

    def cache_write(self, i, key, value, slots):
        l = self.layers[i]
        if self.fp8:
            self.pa.pa_reshape_and_cache_fp8(key, value, l.k_pool, l.v_pool, slots, W.FP8_SCALE,
                                             W.FP8_SCALE, self.status)
        else:
            self.pa.pa_reshape_and_cache(key, value, l.k_pool, l.v_pool, slots, self.status)

    def layer_step(self, i, tables=None, lens=None, slots=None):
        l = self.layers[i]
        self.cache_write(i, l.key, l.value, self.slots if slots is None else slots)
        self.attention(i, tables, lens)

    def step(self):
        for i in range(len(self.layers)):
            self.layer_step(i)


def profile_summary(name: str) -> str:
    return os.path.join(ROOT, "profiles", f"decode_kernel_{name}.md")


def measure_decode(cfg: W.DecodeConfig, args, rank, world, device, dist, headline: bool,
                   fp8: bool = False):
    """Times one workload: K replays of a CUDA graph of the 16-layer step
    (cache write + attention per layer) and K replays of a graph of the
    attention calls alone, on device events, with clocks sampled meanwhile.
    Returns the headline record (with end-to-end and CPU-baseline legs) or a
    per-config record."""
    from paged_kv_cache_455_b200 import pa
    length_scale = args.length_scale
    if cfg.name == "pressure" and length_scale == 1.0:
        free, _ = torch.cuda.mem_get_info(device)
        length_scale = W.fit_length_scale(cfg, free)
    wl = Workload(cfg, device, shard=rank, length_scale=length_scale, layers=args.layers, fp8=fp8)
    L = wl.layout
    nl = len(wl.layers)
    bytes_layer = attention_bytes(L, 1 if fp8 else 0)
    torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize(device)
    if int(wl.status.item()) != 0:
        raise RuntimeError(f"device status {int(wl.status.item())} during warm-up ({cfg.name})")

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

    eager_ms = None
    if headline:
        # ---- the same step launched eagerly (host overhead included)
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
    peak, peak_kind = measured_peak()
    achieved = bytes_layer / (attn_ms_mean * 1e-3) / 1e9
    traffic = profiled_traffic(profile_summary(cfg.name + ("_fp8" if fp8 else "")),
                               DECODE8_SOURCES if fp8 else DECODE_SOURCES)
    if traffic is not None and length_scale != 1.0:
        traffic = None   # the committed capture is of the unscaled workload

    if not headline:
        rec = {
            "workload": f"{cfg.name}: {cfg.description}" + (
                f"; FP8 (E4M3) cache, per-tensor scales {W.FP8_SCALE:.6g}, bf16 query and "
                "output" if fp8 else ""),
            "layers": nl, "num_seqs_per_gpu": cfg.num_seqs,
            "sum_context_lens_per_gpu": int(L.context_lens.sum()),
            "max_context_len": L.max_context_len,
            "step_ms": round(ms_per_step, 4),
            "step_gbs": round(value, 1),
            "step_pct_of_8tbs_per_gpu": round(100 * value / (NOMINAL_HBM_GBS * world), 2),
            "attention_us_per_launch": round(attn_ms_mean * 1e3, 2),
            "attention_us_worst_rank": round(attn_ms_worst * 1e3, 2),
            "attention_gbs_per_gpu": round(achieved, 1),
            "attention_pct_of_8tbs": round(100 * achieved / NOMINAL_HBM_GBS, 2),
            "frac": round(achieved / peak, 4),
            "peak": peak, "peak_source": f"{peak_kind} HBM copy bandwidth",
            "algorithmic_bytes_per_launch": bytes_layer,
            "traffic": traffic,
            "tokens_per_s_per_layer": round(tokens_per_s_layer, 1),
            "gpu_launches": int(launches),
            "clocks": clocks.summary(),
        }
        del wl
        torch.cuda.empty_cache()
        return rec

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, args, device, dist, world, bytes_layer)

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
        "dtype": "e4m3 KV, bf16 query/output" if fp8 else cfg.dtype,
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
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        out["cpu_baseline"] = cpu_baseline(cfg, L, wl.layers[0], budget_s=args.cpu_seconds)
    del wl
    torch.cuda.empty_cache()
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
    """Same metric through the public API with host (pinned) buffers.  Every
    step copies each layer's query, new key and new value (one pinned block
    per layer) and the batch metadata host->device, runs the layers, and
    copies every layer's output back.  The host->device copies run on one
    side stream and the device->host copies on another, ordered by events,
    so that they overlap the layers' kernels; the timed region starts before
    the first step's first copy and ends after its last one."""
    L, cfg = wl.layout, wl.cfg
    nl = len(wl.layers)
    l0 = wl.layers[0]
    parts = (l0.query, l0.key, l0.value)
    sizes = [t.numel() * t.element_size() for t in parts]
    per_layer = sum(sizes)
    host_in = torch.empty((nl, per_layer), dtype=torch.uint8).pin_memory()
    dev_in = torch.empty((nl, per_layer), dtype=torch.uint8, device=device)
    for i, l in enumerate(wl.layers):
        off = 0
        for t, n in zip((l.query, l.key, l.value), sizes):
            host_in[i, off:off + n].copy_(t.contiguous().view(-1).view(torch.uint8).cpu())
            off += n
    views = []
    for i in range(nl):
        off, vs = 0, []
        for t, n in zip(parts, sizes):
            vs.append(dev_in[i, off:off + n].view(t.dtype).view(t.shape))
            off += n
        views.append(vs)
    # metadata: slots (int64) first, then tables and lengths (int32)
    tab, lens, slots = L.block_tables, L.context_lens, L.slot_mapping
    mbytes = [slots.nbytes, tab.nbytes, lens.nbytes]
    host_meta = torch.empty(sum(mbytes), dtype=torch.uint8).pin_memory()
    off = 0
    for a, n in zip((slots, tab, lens), mbytes):
        host_meta[off:off + n].copy_(torch.from_numpy(np.ascontiguousarray(a)).view(-1).view(torch.uint8))
        off += n
    dev_meta = torch.empty_like(host_meta, device=device)
    d_slots = dev_meta[:mbytes[0]].view(torch.int64)
    d_tab = dev_meta[mbytes[0]:mbytes[0] + mbytes[1]].view(torch.int32).view(tab.shape)
    d_lens = dev_meta[mbytes[0] + mbytes[1]:].view(torch.int32)
    host_out = torch.empty((nl,) + tuple(l0.query.shape), dtype=l0.query.dtype).pin_memory()
    h2d_bytes = host_in.numel() + host_meta.numel()
    d2h_bytes = host_out.numel() * host_out.element_size()

    compute = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_used, ev_done, ev_back = ([ev() for _ in range(nl)] for _ in range(4))
    ev_meta, ev_meta_used = ev(), ev()

    def layer(i):
        q, k, v = views[i]
        l = wl.layers[i]
        wl.cache_write(i, k, v, d_slots)
        if wl.fp8:
            wl.pa.pa_decode_attention_fp8(wl.outs[i], q, l.k_pool, l.v_pool, d_tab, d_lens,
                                          L.max_context_len, cfg.scale, W.FP8_SCALE, W.FP8_SCALE,
                                          wl.workspace, wl.status)
        else:
            wl.pa.pa_decode_attention(wl.outs[i], q, l.k_pool, l.v_pool, d_tab, d_lens,
                                      L.max_context_len, cfg.scale, wl.workspace, wl.status)

    def step():
        with torch.cuda.stream(up):
            up.wait_event(ev_meta_used)
            dev_meta.copy_(host_meta, non_blocking=True)
            ev_meta.record(up)
            for i in range(nl):
                up.wait_event(ev_used[i])        # the previous step has read layer i's inputs
                dev_in[i].copy_(host_in[i], non_blocking=True)
                ev_in[i].record(up)
        compute.wait_event(ev_meta)
        for i in range(nl):
            compute.wait_event(ev_in[i])
            compute.wait_event(ev_back[i])       # the previous step's output i is on the host
            layer(i)
            ev_used[i].record(compute)
            ev_done[i].record(compute)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[i])
                host_out[i].copy_(wl.outs[i], non_blocking=True)
                ev_back[i].record(down)
        ev_meta_used.record(compute)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    steps = max(3, args.steps // 2)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    s.record(compute)
    up.wait_event(s)
    for _ in range(steps):
        step()
    for i in range(nl):
        compute.wait_event(ev_back[i])
    e.record(compute)
    torch.cuda.synchronize(device)
    if int(wl.status.item()) != 0:
        raise RuntimeError(f"device status {int(wl.status.item())} in the end-to-end leg")
    ms = s.elapsed_time(e) / steps
    if dist is not None:
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t[0])
    value = world * bytes_layer * nl / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
            "copies": "one pinned block per layer (query, new key, new value) and one of "
                      "metadata host->device on a side stream, every layer's output "
                      "device->host on another, overlapping the kernels"}


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
    cfg = W.CONFIGS[args.config or HEADLINE]
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


def run_prefill(args, device, record: bool = False):
    """Times the chunked-prefill step (--path prefill), or, with record=True,
    the same measurement as a sub-record of the default decode line."""
    from paged_kv_cache_455_b200 import pa
    layers = 4 if record else (args.layers or 4)
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=None, choices=sorted(W.CONFIGS),
                    help="measure only this workload (default: the memory-pressure headline "
                         "plus the per-config records)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: the workload's 16); fewer only for profiling")
    ap.add_argument("--path", default="decode", choices=["decode", "prefill"],
                    help="decode (the default measurement) or the chunked-prefill path")
    ap.add_argument("--length-scale", type=float, default=1.0,
                    help="shrink every context length (profiling captures of the large "
                         "workloads only)")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="with --config: measure the workload over an FP8 (E4M3) cache")
    ap.add_argument("--no-prefill", action="store_true")
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
        if args.config is not None:
            line = measure_decode(W.CONFIGS[args.config], args, rank, world, device, dist,
                                  headline=True, fp8=args.fp8)
        else:
            per = {}
            if not args.no_per_config:
                for name in PER_CONFIG:
                    per[name] = measure_decode(W.CONFIGS[name], args, rank, world, device, dist,
                                               headline=False)
                for name in PER_CONFIG:
                    per[name + "_fp8"] = measure_decode(W.CONFIGS[name], args, rank, world, device,
                                                        dist, headline=False, fp8=True)
            prefill = None
            if world == 1 and not args.no_prefill:
                prefill = run_prefill(args, device, record=True)
                torch.cuda.empty_cache()
            line = measure_decode(W.CONFIGS[HEADLINE], args, rank, world, device, dist,
                                  headline=True)
            line["per_config"] = per
            line["prefill"] = prefill
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
