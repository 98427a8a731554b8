"""Seeded synthetic decode workloads (input generation only).

This module builds the inputs that both the CUDA library and the CPU oracle
consume: context lengths, block tables drawn from a simulated free list, the
slot of each sequence's new token, and N(0, 1) query / key / value / pool
contents.  It contains none of the attention arithmetic.

Workload shapes follow the pages' GQA example (16 full-attention layers, 4 KV
heads, head dim 256, BF16 -- "vLLM Architecture, Memory and Benchmarks Deep
Dive", section 1) and their 16- or 32-token blocks (same page, section 2).
The block allocator is a FIFO free list: ``get_blocks`` pops from the front,
``release_blocks`` appends a sequence's blocks at the back, and running out of
blocks is an error, not a crash ("Inside vLLM: Anatomy of a High-Throughput
LLM Inference System", sections "Memory-Efficient KV Cache Storage" and
"Garbage Collection & Reuse").

Conventions (readings of the pages, which do not fix them):

* ``context_lens[b]`` counts the token being decoded; its K/V are written by
  the cache write to ``slot_mapping[b]``, the slot of logical position
  ``context_lens[b] - 1``.
* Before the step, that slot, the unused tail of each sequence's last block
  and every block no sequence owns hold NaN, so that a masking or placement
  error shows up as a non-finite output.
* Unused block-table entries hold -1.
"""
from __future__ import annotations

import math
from collections import deque
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch


# --------------------------------------------------------------------------
# Block allocator (harness)
# --------------------------------------------------------------------------

class FifoBlockAllocator:
    """FIFO free-list allocator of physical KV blocks.

    ``get_blocks`` takes blocks from the front of the free list, and
    ``release_blocks`` returns a sequence's blocks to the back, in the order
    the sequence held them.  Asking for more blocks than are free raises
    ``MemoryError`` and leaves the allocator unchanged.
    """

    def __init__(self, free_list):
        self.free_blocks = deque(int(b) for b in free_list)
        self.block_table: Dict[int, List[int]] = {}

    @property
    def num_free(self) -> int:
        return len(self.free_blocks)

    def get_blocks(self, seq_id: int, num_blocks: int) -> List[int]:
        if seq_id in self.block_table:
            raise KeyError(f"sequence {seq_id} already holds blocks")
        if num_blocks > len(self.free_blocks):
            raise MemoryError(f"need {num_blocks} blocks, {len(self.free_blocks)} free")
        blocks = [self.free_blocks.popleft() for _ in range(num_blocks)]
        self.block_table[seq_id] = blocks
        return blocks

    def release_blocks(self, seq_id: int) -> None:
        if seq_id in self.block_table:
            self.free_blocks.extend(self.block_table.pop(seq_id))


# --------------------------------------------------------------------------
# Workload configurations
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class DecodeConfig:
    name: str
    index: int            # 1-based; the seed is 455 + index
    layers: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str            # "f32" or "bf16"
    scale: float
    description: str

    @property
    def seed(self) -> int:
        return 455 + self.index

    @property
    def elem_size(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


CONFIGS: Dict[str, DecodeConfig] = {
    "tiny": DecodeConfig(
        "tiny", 1, 1, 3, 8, 2, 64, 4, "f32", 1.0 / 8.0,
        "tiny paged decode: 1 layer, B=3, lengths {3,5,2}, Hq=8, Hkv=2, d=64, "
        "block 4, fp32, 16-block pool from a seeded permutation"),
    "qwen": DecodeConfig(
        "qwen", 2, 16, 64, 16, 4, 256, 16, "bf16", 1.0 / 16.0,
        "16 layers, B=64, lengths U[128,4096], Hq=16, Hkv=4, d=256, block 16, bf16, "
        "tables from a seeded shuffled free list with 10% spare blocks"),
    "long": DecodeConfig(
        "long", 3, 16, 8, 16, 4, 256, 16, "bf16", 1.0 / 16.0,
        "16 layers, B=8, every length 8192, Hq=16, Hkv=4, d=256, block 16, bf16, "
        "4096 used blocks scattered over an 8192-block pool"),
    "mix": DecodeConfig(
        "mix", 4, 16, 256, 16, 4, 256, 32, "bf16", 1.0 / 16.0,
        "16 layers, B=256, lengths lognormal(median 512, sigma 1) clipped to [1,32768], "
        "Hq=16, Hkv=4, d=256, block 32, bf16, pool fragmented by 10k allocate/free events"),
    "pressure": DecodeConfig(
        "pressure", 5, 16, 512, 16, 4, 256, 16, "bf16", 1.0 / 16.0,
        "16 layers, B=512, lengths U[1024,6144], Hq=16, Hkv=4, d=256, block 16, bf16, "
        "pool of every needed block of all 16 layers (~120 GB), seeded random free list"),
}


@dataclass
class BatchLayout:
    """Host-side (numpy) description of one decode step's batch."""
    config: DecodeConfig
    context_lens: np.ndarray          # [B] int32
    block_tables: np.ndarray          # [B, max_blocks] int32, -1 past each sequence
    slot_mapping: np.ndarray          # [B] int64, -1 for an empty sequence
    num_blocks: int                   # physical blocks per layer pool
    length_scale: float = 1.0         # < 1 when lengths were shrunk to fit memory
    notes: Dict[str, object] = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if len(self.context_lens) else 0


def _lognormal_lengths(rng: np.random.Generator, n: int) -> np.ndarray:
    x = rng.lognormal(mean=math.log(512.0), sigma=1.0, size=n)
    return np.clip(np.rint(x), 1, 32768).astype(np.int64)


def draw_context_lens(cfg: DecodeConfig, rng: np.random.Generator) -> np.ndarray:
    if cfg.name == "tiny":
        return np.array([3, 5, 2], dtype=np.int64)
    if cfg.name == "qwen":
        return rng.integers(128, 4096, size=cfg.num_seqs, endpoint=True)
    if cfg.name == "long":
        return np.full(cfg.num_seqs, 8192, dtype=np.int64)
    if cfg.name == "mix":
        return _lognormal_lengths(rng, cfg.num_seqs)
    if cfg.name == "pressure":
        return rng.integers(1024, 6144, size=cfg.num_seqs, endpoint=True)
    raise KeyError(cfg.name)


def _blocks_needed(lens, bs: int) -> np.ndarray:
    return -(-np.asarray(lens, dtype=np.int64) // bs)


def _fragment_history(rng: np.random.Generator, alloc: FifoBlockAllocator, bs: int,
                      events: int) -> Dict[str, int]:
    """Runs ``events`` random allocate/free events, then releases every live
    sequence in the order it was allocated."""
    live: List[int] = []
    next_id = 1 << 30
    done = {"alloc": 0, "alloc_failed": 0, "free": 0, "free_empty": 0}
    for _ in range(events):
        if rng.random() < 0.5:
            n = int(_blocks_needed(_lognormal_lengths(rng, 1), bs)[0])
            try:
                alloc.get_blocks(next_id, n)
                live.append(next_id)
                done["alloc"] += 1
            except MemoryError:
                done["alloc_failed"] += 1
            next_id += 1
        else:
            if not live:
                done["free_empty"] += 1
                continue
            victim = live.pop(int(rng.integers(0, len(live))))
            alloc.release_blocks(victim)
            done["free"] += 1
    for sid in live:
        alloc.release_blocks(sid)
    return done


def shard_seed(cfg: DecodeConfig, shard: int) -> int:
    """Seed of data-parallel shard ``shard`` (shard 0 is the config's seed)."""
    return cfg.seed + 7919 * shard


def make_layout(cfg: DecodeConfig, length_scale: float = 1.0, shard: int = 0) -> BatchLayout:
    """Draws lengths and block tables for ``cfg`` from numpy's generator seeded
    with ``shard_seed(cfg, shard)``.  ``length_scale`` < 1 shrinks every length
    (used only to fit the memory-pressure pool into free device memory)."""
    rng = np.random.default_rng(shard_seed(cfg, shard))
    lens = draw_context_lens(cfg, rng)
    if length_scale != 1.0:
        lens = np.maximum(1, np.rint(lens * length_scale)).astype(np.int64)
    bs = cfg.block_size
    need = _blocks_needed(lens, bs)
    total = int(need.sum())
    notes: Dict[str, object] = {}
    if cfg.name == "tiny":
        nb = 16
        free = rng.permutation(nb)
    elif cfg.name == "qwen":
        nb = int(math.ceil(total * 1.10))
        free = rng.permutation(nb)
    elif cfg.name == "long":
        nb = 2 * total
        free = rng.permutation(nb)
    elif cfg.name == "mix":
        nb = int(math.ceil(total * 1.25))
        free = np.arange(nb)
    elif cfg.name == "pressure":
        nb = total
        free = rng.permutation(nb)
    else:
        raise KeyError(cfg.name)
    alloc = FifoBlockAllocator(free)
    if cfg.name == "mix":
        notes["history"] = _fragment_history(rng, alloc, bs, 10_000)
    max_blocks = max(1, int(need.max()) if len(need) else 1)
    tables = np.full((cfg.num_seqs, max_blocks), -1, dtype=np.int32)
    slots = np.full(cfg.num_seqs, -1, dtype=np.int64)
    for b in range(cfg.num_seqs):
        blocks = alloc.get_blocks(b, int(need[b]))
        tables[b, :len(blocks)] = blocks
        ctx = int(lens[b])
        if ctx > 0:
            last = ctx - 1
            slots[b] = int(tables[b, last // bs]) * bs + last % bs
    notes["shard"] = shard
    return BatchLayout(cfg, lens.astype(np.int32), tables, slots, nb, length_scale, notes)


def fit_length_scale(cfg: DecodeConfig, free_bytes: int, reserve_bytes: int = 8 << 30) -> float:
    """Largest length scale (<= 1) whose pools for all layers fit ``free_bytes``
    minus ``reserve_bytes``."""
    base = make_layout(cfg)
    per_block = 2 * cfg.layers * cfg.block_size * cfg.num_kv_heads * cfg.head_dim * cfg.elem_size
    need = base.num_blocks * per_block
    budget = max(0, free_bytes - reserve_bytes)
    if need <= budget:
        return 1.0
    scale = math.floor(1000.0 * budget / need) / 1000.0
    # lengths round per sequence, so step down until the pools really fit
    while scale > 0 and make_layout(cfg, scale).num_blocks * per_block > budget:
        scale = round(scale - 0.001, 3)
    return scale


# --------------------------------------------------------------------------
# Tensor contents
# --------------------------------------------------------------------------

def valid_slots(layout: BatchLayout) -> np.ndarray:
    """Slots holding a cached token before the step (positions < ctx - 1)."""
    bs = layout.config.block_size
    parts = []
    for b, ctx in enumerate(layout.context_lens):
        t = np.arange(max(0, int(ctx) - 1), dtype=np.int64)
        parts.append(layout.block_tables[b, t // bs].astype(np.int64) * bs + t % bs)
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


@dataclass
class LayerTensors:
    query: torch.Tensor       # [B, Hq, d]
    key: torch.Tensor         # [B, Hkv, d]   new token
    value: torch.Tensor       # [B, Hkv, d]   new token
    k_pool: torch.Tensor      # [nb, bs, Hkv, d]
    v_pool: torch.Tensor      # [nb, bs, Hkv, d]


def _randn(shape, gen: torch.Generator, device, dtype) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def _fill_pool(pool_rows: torch.Tensor, slots: torch.Tensor, gen: torch.Generator,
               chunk_rows: int) -> None:
    """Writes N(0,1) rows into pool_rows[slots] in chunks (bounded temporaries)."""
    row_shape = pool_rows.shape[1:]
    for s in range(0, slots.numel(), chunk_rows):
        idx = slots[s:s + chunk_rows]
        pool_rows[idx] = _randn((idx.numel(),) + tuple(row_shape), gen, pool_rows.device,
                                pool_rows.dtype)


def make_layers(layout: BatchLayout, device, layers: Optional[int] = None,
                chunk_rows: int = 1 << 16) -> List[LayerTensors]:
    """Draws every layer's tensors with a torch generator on ``device`` seeded
    with the layout's shard seed.  Values are N(0,1) drawn in fp32 and cast to the
    config's dtype; pool slots outside ``valid_slots`` are NaN."""
    cfg = layout.config
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(shard_seed(cfg, int(layout.notes.get("shard", 0))))
    nl = cfg.layers if layers is None else layers
    slots = torch.from_numpy(valid_slots(layout)).to(device)
    B, hq, hkv, d = cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    nb, bs = layout.num_blocks, cfg.block_size
    dt = cfg.torch_dtype
    out = []
    for _ in range(nl):
        q = _randn((B, hq, d), gen, device, dt)
        k = _randn((B, hkv, d), gen, device, dt)
        v = _randn((B, hkv, d), gen, device, dt)
        pools = []
        for _kv in range(2):
            pool = torch.full((nb, bs, hkv, d), float("nan"), device=device, dtype=dt)
            _fill_pool(pool.view(nb * bs, hkv, d), slots, gen, chunk_rows)
            pools.append(pool)
        out.append(LayerTensors(q, k, v, pools[0], pools[1]))
    return out


# FP8 (E4M3) cache contents: the per-tensor scales of the synthetic
# workloads put 8 standard deviations at the format's largest value, 448.
FP8_SCALE = 8.0 / 448.0
FP8_NAN = 0x7F


def fp8_codes(x: torch.Tensor, scale: float) -> torch.Tensor:
    """E4M3 codes (uint8) of the draws x / scale, clamped to +-448, through
    torch's own float8_e4m3fn conversion (input generation only)."""
    y = (x.float() / scale).clamp_(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


def make_layers_fp8(layout: BatchLayout, device, layers: Optional[int] = None,
                    scale: float = FP8_SCALE, chunk_rows: int = 1 << 16) -> List[LayerTensors]:
    """Like ``make_layers`` but with E4M3 pools (uint8 codes): pool rows in
    ``valid_slots`` are codes of N(0,1) draws / ``scale``, every other row is
    the NaN code; query and the new token's key / value are bf16 N(0,1)."""
    cfg = layout.config
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(shard_seed(cfg, int(layout.notes.get("shard", 0))) + 104729)
    nl = cfg.layers if layers is None else layers
    slots = torch.from_numpy(valid_slots(layout)).to(device)
    B, hq, hkv, d = cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    nb, bs = layout.num_blocks, cfg.block_size
    out = []
    for _ in range(nl):
        q = _randn((B, hq, d), gen, device, torch.bfloat16)
        k = _randn((B, hkv, d), gen, device, torch.bfloat16)
        v = _randn((B, hkv, d), gen, device, torch.bfloat16)
        pools = []
        for _kv in range(2):
            pool = torch.full((nb, bs, hkv, d), FP8_NAN, device=device, dtype=torch.uint8)
            rows = pool.view(nb * bs, hkv, d)
            for s0 in range(0, slots.numel(), chunk_rows):
                idx = slots[s0:s0 + chunk_rows]
                rows[idx] = fp8_codes(torch.randn((idx.numel(), hkv, d), generator=gen,
                                                  device=device), scale)
            pools.append(pool)
        out.append(LayerTensors(q, k, v, pools[0], pools[1]))
    return out


def device_metadata(layout: BatchLayout, device):
    """(block_tables, context_lens, slot_mapping) as tensors on ``device``."""
    return (torch.from_numpy(layout.block_tables).to(device),
            torch.from_numpy(layout.context_lens).to(device),
            torch.from_numpy(layout.slot_mapping).to(device))


# --------------------------------------------------------------------------
# Host copies for the oracle
# --------------------------------------------------------------------------

def to_numpy_elems(t: torch.Tensor) -> np.ndarray:
    """fp32 -> numpy float32; bf16 -> numpy uint16 holding the raw bits;
    E4M3 codes (uint8) -> numpy uint8."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.uint8:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def compact_sample(layout: BatchLayout, layer: LayerTensors, seqs) -> dict:
    """Host copy of the inputs of the sequences ``seqs`` only.

    The blocks these sequences own are copied into a compact host pool and
    their tables are relabelled to index it (a relabelling of physical blocks,
    under which the result of paged attention is unchanged).  Returns numpy
    arrays ready for the oracle plus ``block_map`` (new id -> old id).
    """
    seqs = np.asarray(seqs, dtype=np.int64)
    bs = layout.config.block_size
    need = _blocks_needed(layout.context_lens[seqs], bs)
    old_ids = np.concatenate([layout.block_tables[b, :n] for b, n in zip(seqs, need)]) \
        if len(seqs) else np.zeros(0, dtype=np.int32)
    new_tables = np.full((len(seqs), layout.max_blocks), -1, dtype=np.int32)
    pos = 0
    for i, n in enumerate(need):
        new_tables[i, :n] = np.arange(pos, pos + n, dtype=np.int32)
        pos += int(n)
    idx = torch.from_numpy(old_ids.astype(np.int64)).to(layer.k_pool.device)
    new_slots = np.full(len(seqs), -1, dtype=np.int64)
    for i, b in enumerate(seqs):
        s = int(layout.slot_mapping[b])
        if s >= 0:
            blk_old, off = s // bs, s % bs
            j = int(np.nonzero(layout.block_tables[b, :need[i]] == blk_old)[0][0])
            new_slots[i] = int(new_tables[i, j]) * bs + off
    sel = torch.from_numpy(seqs).to(layer.query.device)
    return {
        "query": to_numpy_elems(layer.query[sel]),
        "key": to_numpy_elems(layer.key[sel]),
        "value": to_numpy_elems(layer.value[sel]),
        "k_pool": to_numpy_elems(layer.k_pool[idx]),
        "v_pool": to_numpy_elems(layer.v_pool[idx]),
        "block_tables": new_tables,
        "context_lens": layout.context_lens[seqs].copy(),
        "slot_mapping": new_slots,
        "block_map": old_ids,
    }
