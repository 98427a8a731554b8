"""Host-side block manager with reference counts: copy-on-write sharing.

"vLLM Architecture, Memory and Benchmarks Deep Dive", section 2: a sequence's
KV cache lives in fixed-size physical blocks named by its block table, new
blocks are handed out on demand as the sequence grows, and under
"Copy-on-Write (CoW) Branching" the rollouts of one prompt share the
prompt's blocks, a block being cloned only when the sequences sharing it
diverge.

Readings taken where the page is silent:

* a fork shares every block of the parent (each block's reference count goes
  up by one); the child starts with the parent's length;
* a block is written only at the position after a sequence's last token, so
  only a sequence's last, partly filled block can ever need a copy: appending
  to a block whose count is above one first moves the sequence to a fresh
  block holding a copy of the shared one (a (source, destination) pair for
  ``pa_copy_blocks``), and the shared block loses one reference;
* full blocks are never written again and stay shared until freed;
* a block returns to the back of the free list when its count reaches zero.

The manager only does bookkeeping; the device work is ``pa_copy_blocks`` for
the returned pairs followed by ``pa_reshape_and_cache`` for the new tokens.

Swapping ("Inside vLLM: Anatomy of a High-Throughput LLM Inference System",
section "Memory-Efficient KV Cache Storage": blocks move between GPU and CPU
memory, the less used ones paged out to the host when the cache outgrows the
GPU): ``swap_out`` moves all of a sequence's (unshared) blocks to host
blocks and frees the device ones, ``swap_in`` brings them back into fresh
device blocks; each returns the (source, destination) pairs for
``pa_swap_blocks``.
"""
from __future__ import annotations

from collections import deque
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Iterable[int]] = None,
                 num_host_blocks: int = 0):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = range(num_blocks) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the block ids")
        self.free = deque(order)
        self.refs = np.zeros(num_blocks, dtype=np.int32)
        self.tables: Dict[int, List[int]] = {}
        self.lens: Dict[int, int] = {}
        self.host_free = deque(range(num_host_blocks))
        self.swapped: Dict[int, List[int]] = {}

    @property
    def num_free(self) -> int:
        return len(self.free)

    def _take(self) -> int:
        if not self.free:
            raise MemoryError("no free block")
        b = self.free.popleft()
        self.refs[b] = 1
        return b

    def _drop(self, b: int) -> None:
        self.refs[b] -= 1
        if self.refs[b] == 0:
            self.free.append(b)

    def allocate(self, seq: int, num_tokens: int) -> List[int]:
        """Blocks for a new sequence of num_tokens tokens (all or nothing)."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise MemoryError(f"need {need} blocks, {len(self.free)} free")
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = num_tokens
        return list(self.tables[seq])

    def fork(self, parent: int, child: int) -> None:
        """The child shares all of the parent's blocks and its length."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        blocks = list(self.tables[parent])
        for b in blocks:
            self.refs[b] += 1
        self.tables[child] = blocks
        self.lens[child] = self.lens[parent]

    def append_slot(self, seq: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Makes room for one more token of seq.

        Returns (slot, copy): the slot (block * block_size + offset) the new
        token's K/V goes to, and a (source, destination) block pair to copy
        first, or None.  On MemoryError nothing changes.
        """
        table, pos = self.tables[seq], self.lens[seq]
        off = pos % self.block_size
        copy = None
        if off == 0:
            table.append(self._take())
        elif self.refs[table[-1]] > 1:
            src = table[-1]
            dst = self._take()
            self.refs[src] -= 1          # still held by another sequence: never freed here
            table[-1] = dst
            copy = (src, dst)
        self.lens[seq] = pos + 1
        return table[pos // self.block_size] * self.block_size + off, copy

    def swap_out(self, seq: int) -> List[Tuple[int, int]]:
        """(device block, host block) pairs that move seq to host memory; its
        device blocks are freed.  Shared blocks cannot move (ValueError); too
        few host blocks raise MemoryError; either way nothing changes."""
        table = self.tables[seq]
        if any(self.refs[b] > 1 for b in table):
            raise ValueError(f"sequence {seq} shares blocks")
        if len(table) > len(self.host_free):
            raise MemoryError(f"need {len(table)} host blocks, {len(self.host_free)} free")
        pairs = [(b, self.host_free.popleft()) for b in table]
        for b in table:
            self._drop(b)
        self.swapped[seq] = [h for _, h in pairs]
        self.tables[seq] = []
        return pairs

    def swap_in(self, seq: int) -> List[Tuple[int, int]]:
        """(host block, device block) pairs that bring seq back into fresh
        device blocks; its host blocks are freed.  MemoryError (nothing
        changes) if the device has too few free blocks."""
        host = self.swapped[seq]
        if len(host) > len(self.free):
            raise MemoryError(f"need {len(host)} blocks, {len(self.free)} free")
        pairs = [(h, self._take()) for h in host]
        self.host_free.extend(host)
        self.tables[seq] = [d for _, d in pairs]
        del self.swapped[seq]
        return pairs

    def free_seq(self, seq: int) -> None:
        for b in self.tables.pop(seq):
            self._drop(b)
        self.host_free.extend(self.swapped.pop(seq, []))
        del self.lens[seq]

    def block_tables(self, seqs: List[int], max_blocks: Optional[int] = None):
        """(block_tables int32 [B, max_blocks] padded with -1, context_lens int32 [B])."""
        width = max([len(self.tables[s]) for s in seqs] + [1]) if max_blocks is None else max_blocks
        tab = np.full((len(seqs), width), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            tab[i, :len(self.tables[s])] = self.tables[s]
        lens = np.array([self.lens[s] for s in seqs], dtype=np.int32)
        return tab, lens
