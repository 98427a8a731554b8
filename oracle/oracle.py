"""CPU oracle for paged KV-cache decode attention (TEST INFRASTRUCTURE ONLY).

This module is the yardstick the CUDA library is measured against.  It shares
no code with the CUDA path and never imports it; only ``tests/``, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may use
it.  The product path must never call into here.

Two independent fp64 implementations live here:

* ``pa_oracle.c`` (loaded through ctypes): gathers each sequence's blocks
  through its block table into contiguous K/V, then runs exact softmax
  attention; OpenMP over sequences.  Used for the big cases and for timing.
* ``paged_attention_np`` / ``partition_attention_np``: the same definition in
  numpy (fancy-index gather, ``einsum``, ``exp``), used on small cases and to
  cross-check the C code.

Sources on the pages (cited by page title and section):

* KV-size formula ``2 * L * H_KV * d_head * T * b``: "Optimizing LLM Inference:
  A Deep Dive into vLLM's PagedAttention and Continuous Batching", section
  "Understanding the KV Cache Bottleneck".
* Contiguous-vs-paged reservation of 3, 5 and 2 tokens: "High-Throughput LLM
  Inference & Training: A Deep Dive into vLLM", Figure 1 and Figure 2.
* Block table mapping logical to physical blocks, paged cache that appears
  contiguous to attention: "Optimizing LLM Inference ...", section
  "PagedAttention: Borrowing a 50-Year-Old OS Masterpiece"; "vLLM
  Architecture, Memory and Benchmarks Deep Dive", section 2.
* New tokens stored in blocks handed out on demand, only the last block of a
  sequence partly filled: "vLLM Architecture, Memory and Benchmarks Deep
  Dive", section 2 ("On-Demand Allocation").
* Grouped-query attention (16 layers, 4 KV heads, head dim 256): same page,
  section 1.

Readings where the pages are silent: query head ``hq`` uses KV head
``hq // (Hq // Hkv)``; ``context_lens`` counts the token being decoded, whose
K/V the cache write stores at ``slot_mapping``; a length-0 sequence yields a
zero output; a negative slot means "no token" and is skipped.

Element types: ``"f32"`` arrays are ``numpy.float32``; ``"bf16"`` arrays are
``numpy.uint16`` holding raw bfloat16 bits (the upper half of a binary32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_DTYPE_CODE = {"f32": 0, "bf16": 1}
_ELEM_SIZE = {"f32": 4, "bf16": 2}

_lib = None


def build(force: bool = False) -> str:
    """Compiles pa_oracle.c into liboracle.so with gcc (plain -O2, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_kv_bytes.restype = i64
    lib.oracle_kv_bytes.argtypes = [i64, i64, i64, i64, i64]
    lib.oracle_reshape_and_cache.restype = i64
    lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32]
    lib.oracle_threads.restype = i32
    lib.oracle_threads.argtypes = [i32]
    lib.oracle_paged_attention.restype = i32
    lib.oracle_paged_attention.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32,
                                           i64, dbl, i32, i32]
    lib.oracle_partition_attention.restype = i32
    lib.oracle_partition_attention.argtypes = [P, P, P, P, P, P, P, i32, P, i32, i32, i32,
                                               i32, i32, i64, dbl, i32, i32, i32, i32]
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check_elem(a: np.ndarray, dtype: str) -> np.ndarray:
    want = np.float32 if dtype == "f32" else np.uint16
    if a.dtype != want:
        raise TypeError(f"{dtype} data must be numpy {want.__name__}, got {a.dtype}")
    return np.ascontiguousarray(a)


# --------------------------------------------------------------------------
# Size helpers (closed forms printed on the pages)
# --------------------------------------------------------------------------

def kv_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, bytes_per_elem: int) -> int:
    """M_KV = 2 * L * H_KV * d_head * T * b (the factor 2 is K and V)."""
    return int(_load().oracle_kv_bytes(layers, kv_heads, head_dim, tokens, bytes_per_elem))


def reservation_counts(lengths, max_len: int, block_size: int) -> dict:
    """Slots reserved, used and left unused by two allocation policies.

    Contiguous: every request reserves ``max_len`` slots.  Paged: every request
    holds ceil(len / block_size) blocks of ``block_size`` slots; the slots the
    paged policy does not take, out of what the contiguous one reserves, are
    "freed" for other requests.
    """
    used = sum(int(n) for n in lengths)
    contig_reserved = max_len * len(lengths)
    paged_reserved = sum(-(-int(n) // block_size) * block_size for n in lengths)
    return {
        "contiguous": {"reserved": contig_reserved, "used": used,
                       "unused": contig_reserved - used,
                       "unused_frac": (contig_reserved - used) / contig_reserved},
        "paged": {"reserved": paged_reserved, "used": used,
                  "unused": paged_reserved - used,
                  "freed": contig_reserved - paged_reserved},
    }


# --------------------------------------------------------------------------
# Cache write
# --------------------------------------------------------------------------

def reshape_and_cache(key, value, k_pool, v_pool, slot_mapping, dtype: str):
    """Returns new (k_pool, v_pool) with each token's K/V rows stored at its slot.

    key/value are [T, Hkv, d]; pools are [nb, bs, Hkv, d]; slot_mapping is [T]
    int64.  Negative slots are skipped.  Raises ValueError for a slot past the
    pool (the pool is left as it was, since copies are returned).
    """
    key = _check_elem(key, dtype)
    value = _check_elem(value, dtype)
    k_out = np.array(_check_elem(k_pool, dtype), copy=True)
    v_out = np.array(_check_elem(v_pool, dtype), copy=True)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    nb, bs, hkv, d = k_out.shape
    bad = _load().oracle_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_out), _ptr(v_out),
                                           _ptr(slots), slots.shape[0], hkv, d, bs, nb,
                                           _ELEM_SIZE[dtype])
    if bad:
        raise ValueError(f"{bad} slot(s) outside the pool of {nb * bs} slots")
    return k_out, v_out


def reshape_and_cache_np(key, value, k_pool, v_pool, slot_mapping):
    """numpy restatement of the cache write (independent of the C code)."""
    k_out = np.array(k_pool, copy=True)
    v_out = np.array(v_pool, copy=True)
    nb, bs = k_out.shape[:2]
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        if slot >= nb * bs:
            raise ValueError("slot outside the pool")
        k_out[slot // bs, slot % bs] = key[t]
        v_out[slot // bs, slot % bs] = value[t]
    return k_out, v_out


def copy_blocks_np(k_pool, v_pool, block_mapping):
    """Returns new (k_pool, v_pool) in which block dst of each (src, dst) pair
    of block_mapping [P, 2] holds block src of the input pools, read before
    any copy (the copy copy-on-write sharing needs: "vLLM Architecture, Memory
    and Benchmarks Deep Dive", section 2, "Copy-on-Write (CoW) Branching").
    Raises ValueError for a block id outside the pool."""
    k_in, v_in = np.asarray(k_pool), np.asarray(v_pool)
    k_out, v_out = np.array(k_in, copy=True), np.array(v_in, copy=True)
    nb = k_in.shape[0]
    for src, dst in np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2):
        if not (0 <= src < nb and 0 <= dst < nb):
            raise ValueError("block id outside the pool")
        k_out[dst] = k_in[src]
        v_out[dst] = v_in[src]
    return k_out, v_out


def swap_blocks_np(dst_k, dst_v, src_k, src_v, block_mapping):
    """Returns new (dst_k, dst_v) in which block dst of each (src, dst) pair
    holds block src of the source pools (paging blocks between GPU and host
    memory: "Inside vLLM: Anatomy of a High-Throughput LLM Inference System",
    section "Memory-Efficient KV Cache Storage").  Raises ValueError for a
    block id outside its pool."""
    k_out, v_out = np.array(dst_k, copy=True), np.array(dst_v, copy=True)
    src_k, src_v = np.asarray(src_k), np.asarray(src_v)
    for src, dst in np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2):
        if not (0 <= src < src_k.shape[0] and 0 <= dst < k_out.shape[0]):
            raise ValueError("block id outside the pool")
        k_out[dst] = src_k[src]
        v_out[dst] = src_v[src]
    return k_out, v_out


# --------------------------------------------------------------------------
# Attention (C, fp64)
# --------------------------------------------------------------------------

def paged_attention(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                    dtype: str, num_threads: int = 0) -> np.ndarray:
    """Exact fp64 paged decode attention; returns [B, Hq, d] float64."""
    q = _check_elem(q, dtype)
    k_pool = _check_elem(k_pool, dtype)
    v_pool = _check_elem(v_pool, dtype)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, hq, d = q.shape
    nb, bs, hkv, d2 = k_pool.shape
    if d2 != d or bt.shape[0] != B or cl.shape[0] != B:
        raise ValueError("shape mismatch")
    out = np.zeros((B, hq, d), dtype=np.float64)
    rc = _load().oracle_paged_attention(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                        _ptr(bt), bt.shape[1], _ptr(cl), B, hq, hkv, d, bs, nb,
                                        float(scale), _DTYPE_CODE[dtype], int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_paged_attention rejected its inputs (code {rc})")
    return out


def partition_attention(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                        dtype: str, partition_size: int, max_parts: int,
                        num_threads: int = 0):
    """Per-partition (out, max, sum) in fp64, shapes [B,Hq,P,d], [B,Hq,P], [B,Hq,P]."""
    q = _check_elem(q, dtype)
    k_pool = _check_elem(k_pool, dtype)
    v_pool = _check_elem(v_pool, dtype)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, hq, d = q.shape
    nb, bs, hkv, _ = k_pool.shape
    po = np.zeros((B, hq, max_parts, d), dtype=np.float64)
    pm = np.zeros((B, hq, max_parts), dtype=np.float64)
    ps = np.zeros((B, hq, max_parts), dtype=np.float64)
    rc = _load().oracle_partition_attention(_ptr(po), _ptr(pm), _ptr(ps), _ptr(q),
                                            _ptr(k_pool), _ptr(v_pool), _ptr(bt), bt.shape[1],
                                            _ptr(cl), B, hq, hkv, d, bs, nb, float(scale),
                                            _DTYPE_CODE[dtype], int(partition_size),
                                            int(max_parts), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_partition_attention rejected its inputs (code {rc})")
    return po, pm, ps


def merge_partitions(part_out, part_max, part_sum) -> np.ndarray:
    """Log-sum-exp merge of partition results along axis -2 / -1.

    With M = max_p m_p and w_p = l_p * exp(m_p - M):
    out = sum_p w_p * o_p / sum_p w_p.  All-empty rows give zeros.
    """
    pm = np.asarray(part_max, dtype=np.float64)
    ps = np.asarray(part_sum, dtype=np.float64)
    po = np.asarray(part_out, dtype=np.float64)
    M = pm.max(axis=-1, keepdims=True)
    Msafe = np.where(np.isfinite(M), M, 0.0)
    w = np.where(ps > 0, ps * np.exp(pm - Msafe), 0.0)
    den = w.sum(axis=-1)
    num = (w[..., None] * po).sum(axis=-2)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def threads(num_threads: int = 0) -> int:
    """Threads the C oracle uses for a request of ``num_threads`` (0 = all)."""
    return int(_load().oracle_threads(int(num_threads)))


# --------------------------------------------------------------------------
# numpy twin (independent second fp64 path)
# --------------------------------------------------------------------------

def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact conversion of f32 / raw-bf16 data to float64 ("f64" data is
    returned as it is)."""
    if dtype == "f64":
        return np.asarray(a, dtype=np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    bits = np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def gather_np(pool: np.ndarray, table_row: np.ndarray, ctx: int) -> np.ndarray:
    """Contiguous [ctx, Hkv, d] view of one sequence through its block table."""
    bs = pool.shape[1]
    t = np.arange(ctx)
    return pool[np.asarray(table_row)[t // bs], t % bs]


def paged_attention_np(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                       dtype: str) -> np.ndarray:
    """numpy fp64 paged decode attention, same contract as ``paged_attention``."""
    qf = to_f64(q, dtype)
    kf = to_f64(k_pool, dtype)
    vf = to_f64(v_pool, dtype)
    B, hq, d = qf.shape
    hkv = kf.shape[2]
    group = hq // hkv
    out = np.zeros((B, hq, d), dtype=np.float64)
    for b in range(B):
        ctx = int(context_lens[b])
        if ctx == 0:
            continue
        kc = gather_np(kf, block_tables[b], ctx)            # [ctx, Hkv, d]
        vc = gather_np(vf, block_tables[b], ctx)
        kq = np.repeat(kc, group, axis=1)                    # [ctx, Hq, d]
        vq = np.repeat(vc, group, axis=1)
        s = scale * np.einsum("hd,thd->ht", qf[b], kq)       # [Hq, ctx]
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[b] = np.einsum("ht,thd->hd", p, vq) / p.sum(axis=1, keepdims=True)
    return out


def partition_attention_np(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                           dtype: str, partition_size: int, max_parts: int):
    """numpy twin of ``partition_attention``."""
    qf = to_f64(q, dtype)
    kf = to_f64(k_pool, dtype)
    vf = to_f64(v_pool, dtype)
    B, hq, d = qf.shape
    group = hq // kf.shape[2]
    po = np.zeros((B, hq, max_parts, d))
    pm = np.full((B, hq, max_parts), -np.inf)
    ps = np.zeros((B, hq, max_parts))
    for b in range(B):
        ctx = int(context_lens[b])
        kc = np.repeat(gather_np(kf, block_tables[b], ctx), group, axis=1)
        vc = np.repeat(gather_np(vf, block_tables[b], ctx), group, axis=1)
        s = scale * np.einsum("hd,thd->ht", qf[b], kc)
        for p in range(max_parts):
            t0, t1 = p * partition_size, min((p + 1) * partition_size, ctx)
            if t1 <= t0:
                continue
            sp = s[:, t0:t1]
            m = sp.max(axis=1)
            e = np.exp(sp - m[:, None])
            pm[b, :, p] = m
            ps[b, :, p] = e.sum(axis=1)
            po[b, :, p] = np.einsum("ht,thd->hd", e, vc[t0:t1]) / ps[b, :, p][:, None]
    return po, pm, ps


__all__ = [
    "build", "kv_bytes", "reservation_counts", "reshape_and_cache", "reshape_and_cache_np",
    "paged_attention", "partition_attention", "merge_partitions", "threads", "to_f64",
    "gather_np", "paged_attention_np", "partition_attention_np",
]


# --------------------------------------------------------------------------
# Chunked prefill (numpy, fp64)
# --------------------------------------------------------------------------

def prefill_attention_np(q, k_pool, v_pool, block_tables, context_lens, cu_q_lens, scale: float,
                         dtype: str) -> np.ndarray:
    """Exact fp64 attention of a chunk of query tokens per sequence over its
    paged cache, causal within the chunk; returns [total_q, Hq, d] float64.

    Sequence b's chunk is query rows cu_q_lens[b] .. cu_q_lens[b + 1] - 1
    (n_b rows); context_lens[b] counts every cached token including the
    chunk, so chunk row j sits at position p = ctx_b - n_b + j and attends to
    the keys at positions 0 .. p, reached through the block table ("vLLM
    Architecture, Memory and Benchmarks Deep Dive", section 4, chunked
    prefill; section 2, block table).  Query head hq uses KV head
    hq // (Hq // Hkv).  A chunk longer than its context raises ValueError.
    """
    qf = to_f64(q, dtype)
    kf = to_f64(k_pool, dtype)
    vf = to_f64(v_pool, dtype)
    hq, d = qf.shape[1], qf.shape[2]
    hkv = kf.shape[2]
    group = hq // hkv
    out = np.zeros(qf.shape, dtype=np.float64)
    cu = np.asarray(cu_q_lens, dtype=np.int64)
    for b in range(len(context_lens)):
        ctx, q0, n = int(context_lens[b]), int(cu[b]), int(cu[b + 1] - cu[b])
        if n == 0:
            continue
        if n > ctx:
            raise ValueError("chunk longer than its context")
        kc = gather_np(kf, block_tables[b], ctx)          # [ctx, Hkv, d]
        vc = gather_np(vf, block_tables[b], ctx)
        pos = ctx - n + np.arange(n)                       # positions of the chunk rows
        allowed = np.arange(ctx)[None, :] <= pos[:, None]  # [n, ctx] causal
        for h in range(hq):
            kh, vh = kc[:, h // group], vc[:, h // group]
            s = scale * (qf[q0:q0 + n, h] @ kh.T)          # [n, ctx]
            s = np.where(allowed, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            out[q0:q0 + n, h] = (p @ vh) / p.sum(axis=1, keepdims=True)
    return out



# --------------------------------------------------------------------------
# FP8 (E4M3) KV cache (numpy, fp64)
#
# A quantised cache halves the bytes a bandwidth-bound decode step reads
# ("vLLM Architecture, Memory and Benchmarks Deep Dive", section 4, FP8:
# fewer bytes per value double the effective memory bandwidth; "Inside vLLM:
# Anatomy of a High-Throughput LLM Inference System", FAQ: quantized KV
# caches).  Reading taken where the pages give no format: each pool element
# is one E4M3 byte with a per-tensor scale, K = code value * k_scale and
# V = code value * v_scale; the cache write stores the E4M3 code of
# x / scale, the division taken in binary32, rounded to nearest (ties to the
# even code) and saturated to +-448.
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_to_f64(codes) -> np.ndarray:
    """Value of each E4M3 byte: bit 7 is the sign, bits 6..3 the exponent
    (bias 7), bits 2..0 the mantissa; exponent field 0 holds the subnormals
    m * 2^-9; 0x7f and 0xff are NaN; there are no infinities."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where((c & 0x80) != 0, -mag, mag)


def f32_to_e4m3(x) -> np.ndarray:
    """E4M3 code (uint8) of each binary32 value: the nearest of the 127
    non-negative finite magnitudes (ties to the even code), magnitudes above
    448 (infinities included) saturating to 448, the sign kept (also for
    zero); NaN gives 0x7f."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    grid = e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))      # codes 0..126, increasing
    nan = np.isnan(x)
    a = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    tie_pick = np.where(lo % 2 == 0, lo, hi)
    code = np.where(d_hi < d_lo, hi, np.where(d_lo < d_hi, lo, tie_pick))
    code = np.where(np.signbit(x), code | 0x80, code)
    return np.where(nan, 0x7F, code).astype(np.uint8)


def quantize_e4m3(x, scale: float) -> np.ndarray:
    """E4M3 codes of x / scale, the division taken in binary32."""
    y = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return f32_to_e4m3(y)


def dequantize_e4m3(codes, scale: float) -> np.ndarray:
    """fp64 values code * scale (exact: a code has at most 4 significant bits,
    a binary32 scale 24)."""
    return e4m3_to_f64(codes) * float(np.float32(scale))


def reshape_and_cache_fp8_np(key, value, k_pool, v_pool, slot_mapping, k_scale: float,
                             v_scale: float):
    """Cache write into E4M3 pools: key/value are raw bf16 [T, Hkv, d], pools
    uint8 codes [nb, bs, Hkv, d]; each token's rows become the codes of
    key / k_scale and value / v_scale (``quantize_e4m3``) at its slot.
    Negative slots are skipped; a slot past the pool raises ValueError."""
    kq = quantize_e4m3(to_f64(key, "bf16").astype(np.float32), k_scale)
    vq = quantize_e4m3(to_f64(value, "bf16").astype(np.float32), v_scale)
    return reshape_and_cache_np(kq, vq, np.asarray(k_pool, dtype=np.uint8),
                                np.asarray(v_pool, dtype=np.uint8), slot_mapping)


def paged_attention_fp8_np(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                           k_scale: float, v_scale: float) -> np.ndarray:
    """Exact fp64 decode attention over an E4M3 cache: the query is raw bf16,
    the pools' codes are dequantised exactly (``dequantize_e4m3``) and the
    result is the definition of ``paged_attention_np`` on those values."""
    return paged_attention_np(to_f64(q, "bf16"), dequantize_e4m3(k_pool, k_scale),
                              dequantize_e4m3(v_pool, v_scale), block_tables, context_lens,
                              scale, "f64")


__all__ += ["E4M3_MAX", "e4m3_to_f64", "f32_to_e4m3", "quantize_e4m3", "dequantize_e4m3",
            "reshape_and_cache_fp8_np", "paged_attention_fp8_np"]
