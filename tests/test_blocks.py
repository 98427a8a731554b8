"""Copy-on-write block sharing on the host: the reference-counted block
manager, the oracle's block copy, and the invariance that makes sharing
sound ("vLLM Architecture, Memory and Benchmarks Deep Dive", section 2,
"Copy-on-Write (CoW) Branching": rollouts of one prompt share its blocks,
and a block is cloned only when the sequences sharing it diverge)."""
import numpy as np
import pytest

from oracle import oracle as O
from paged_kv_cache_455_b200.blocks import BlockManager


def test_fork_shares_every_block_and_counts_references():
    m = BlockManager(16, 4)
    m.allocate(0, 10)                      # 3 blocks, last one half full
    m.fork(0, 1)
    m.fork(0, 2)
    assert m.tables[1] == m.tables[0] == m.tables[2]
    assert all(m.refs[b] == 3 for b in m.tables[0])
    assert m.num_free == 13


def test_append_copies_only_a_shared_partial_block():
    m = BlockManager(16, 4)
    m.allocate(0, 10)
    m.fork(0, 1)
    full = m.tables[0][:2]
    last = m.tables[0][2]
    slot, copy = m.append_slot(1)
    assert copy is not None and copy[0] == last and copy[1] != last
    assert m.tables[1][:2] == full                 # full blocks stay shared
    assert slot == copy[1] * 4 + 2                  # position 10 = block 2, offset 2
    assert m.refs[last] == 1 and m.refs[copy[1]] == 1
    # the parent now owns its last block alone: no copy
    slot0, copy0 = m.append_slot(0)
    assert copy0 is None and slot0 == last * 4 + 2


def test_append_at_a_block_boundary_takes_a_fresh_block_without_copy():
    m = BlockManager(8, 4)
    m.allocate(0, 8)
    m.fork(0, 1)
    slot, copy = m.append_slot(1)
    assert copy is None
    assert len(m.tables[1]) == 3 and m.tables[1][:2] == m.tables[0]
    assert slot == m.tables[1][2] * 4


def test_free_returns_blocks_when_the_last_reference_goes():
    m = BlockManager(8, 4, free_order=[7, 6, 5, 4, 3, 2, 1, 0])
    m.allocate(0, 6)                       # blocks 7, 6
    m.fork(0, 1)
    m.free_seq(0)
    assert m.num_free == 6                 # still held by sequence 1
    m.free_seq(1)
    assert m.num_free == 8
    assert list(m.free)[-2:] == [7, 6]     # back of the queue, in table order


def test_out_of_blocks_is_an_error_and_changes_nothing():
    m = BlockManager(3, 4)
    m.allocate(0, 12)
    with pytest.raises(MemoryError):
        m.allocate(1, 1)
    assert 1 not in m.tables and m.num_free == 0
    m2 = BlockManager(3, 4)
    m2.allocate(0, 6)
    m2.fork(0, 1)
    m2.append_slot(1)                       # the copy takes the last free block
    m2.append_slot(0)                       # sequence 0 now owns its block alone
    m2.append_slot(0)
    assert m2.lens[0] == 8 and m2.num_free == 0
    with pytest.raises(MemoryError):
        m2.append_slot(0)                   # position 8 needs a new block
    assert m2.lens[0] == 8 and len(m2.tables[0]) == 2


def test_grpo_rollouts_need_one_copy_each():
    bs, prompt, rollouts, steps = 16, 100, 8, 20
    m = BlockManager(64, bs)
    m.allocate(0, prompt)
    for r in range(1, rollouts + 1):
        m.fork(0, r)
    m.free_seq(0)
    copies = 0
    for _ in range(steps):
        for r in range(1, rollouts + 1):
            _, c = m.append_slot(r)
            copies += c is not None
    # only the shared partial block is cloned, and the last rollout still
    # holding it keeps the original
    assert copies == rollouts - 1
    shared = m.tables[1][:prompt // bs]
    assert all(m.tables[r][:prompt // bs] == shared for r in range(1, rollouts + 1))
    assert all(m.refs[b] == rollouts for b in shared)
    # blocks in use: 6 shared + per rollout ceil(120 / 16) - 6 = 2
    assert 64 - m.num_free == prompt // bs + rollouts * (-(-(prompt + steps) // bs) - prompt // bs)


def test_oracle_copy_is_exact_and_touches_nothing_else():
    rng = np.random.default_rng(7)
    k = rng.standard_normal((10, 4, 2, 8)).astype(np.float32)
    v = rng.standard_normal((10, 4, 2, 8)).astype(np.float32)
    mapping = np.array([[3, 7], [1, 0], [3, 5]], dtype=np.int64)
    k2, v2 = O.copy_blocks_np(k, v, mapping)
    for src, dst in mapping:
        assert k2[dst].tobytes() == k[src].tobytes() and v2[dst].tobytes() == v[src].tobytes()
    untouched = [b for b in range(10) if b not in mapping[:, 1]]
    assert k2[untouched].tobytes() == k[untouched].tobytes()
    assert v2[untouched].tobytes() == v[untouched].tobytes()
    with pytest.raises(ValueError):
        O.copy_blocks_np(k, v, np.array([[0, 10]]))


def test_attention_over_shared_blocks_equals_attention_over_private_copies():
    """Sharing is only bookkeeping: attention through tables that alias the
    prompt's blocks equals attention through tables whose blocks are private
    copies (the oracle on both)."""
    rng = np.random.default_rng(11)
    bs, hq, hkv, d, prompt, extra, R = 4, 8, 2, 16, 10, 3, 3
    m = BlockManager(32, bs)
    m.allocate(0, prompt)
    for r in range(1, R + 1):
        m.fork(0, r)
    k = rng.standard_normal((32, bs, hkv, d)).astype(np.float32)
    v = rng.standard_normal((32, bs, hkv, d)).astype(np.float32)
    for r in range(1, R + 1):
        for _ in range(extra):
            slot, c = m.append_slot(r)
            if c is not None:
                k, v = O.copy_blocks_np(k, v, np.array([c]))
            k[slot // bs, slot % bs] = rng.standard_normal((hkv, d))
            v[slot // bs, slot % bs] = rng.standard_normal((hkv, d))
    seqs = list(range(1, R + 1))
    tab, lens = m.block_tables(seqs)
    q = rng.standard_normal((R, hq, d)).astype(np.float32)
    shared = O.paged_attention_np(q, k, v, tab, lens, 0.25, "f32")
    # materialise: every sequence gets its own copy of every block
    kp = np.zeros((R * tab.shape[1], bs, hkv, d), dtype=np.float32)
    vp = np.zeros_like(kp)
    priv = np.full_like(tab, -1)
    n = 0
    for i in range(R):
        for j in range(-(-lens[i] // bs)):
            kp[n], vp[n] = k[tab[i, j]], v[tab[i, j]]
            priv[i, j] = n
            n += 1
    private = O.paged_attention_np(q, kp, vp, priv, lens, 0.25, "f32")
    assert np.abs(shared - private).max() == 0.0
    assert len(set(tab[:, 0])) == 1        # the prompt's first block really is shared


def test_swap_out_and_in_moves_every_block_and_restores_the_table():
    m = BlockManager(8, 4, num_host_blocks=4)
    m.allocate(0, 10)                       # 3 blocks
    m.allocate(1, 4)
    before = list(m.tables[0])
    out = m.swap_out(0)
    assert [d for d, _ in out] == before and m.tables[0] == []
    assert m.num_free == 8 - 1 and len(m.host_free) == 1
    m.allocate(2, 8)                        # the freed device blocks are reused
    back = m.swap_in(0)
    assert [h for h, _ in back] == [h for _, h in out]
    assert len(m.tables[0]) == 3 and m.lens[0] == 10 and len(m.host_free) == 4
    slot, copy = m.append_slot(0)           # appends after the swap as before
    assert copy is None and slot == m.tables[0][2] * 4 + 2


def test_swap_refuses_shared_blocks_and_short_pools():
    m = BlockManager(8, 4, num_host_blocks=2)
    m.allocate(0, 6)
    m.fork(0, 1)
    with pytest.raises(ValueError):
        m.swap_out(0)
    m.allocate(2, 12)                       # 3 blocks > 2 host blocks
    with pytest.raises(MemoryError):
        m.swap_out(2)
    assert len(m.tables[2]) == 3 and len(m.host_free) == 2


def test_oracle_swap_copies_between_pools():
    rng = np.random.default_rng(3)
    dev_k = rng.standard_normal((6, 4, 2, 8)).astype(np.float32)
    dev_v = rng.standard_normal((6, 4, 2, 8)).astype(np.float32)
    host_k = np.zeros((3, 4, 2, 8), np.float32)
    host_v = np.zeros((3, 4, 2, 8), np.float32)
    hk, hv = O.swap_blocks_np(host_k, host_v, dev_k, dev_v, np.array([[5, 0], [2, 2]]))
    assert hk[0].tobytes() == dev_k[5].tobytes() and hv[2].tobytes() == dev_v[2].tobytes()
    assert not hk[1].any() and not hv[1].any()
    with pytest.raises(ValueError):
        O.swap_blocks_np(host_k, host_v, dev_k, dev_v, np.array([[6, 0]]))
