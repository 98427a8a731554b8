"""Seeded input generators and the FIFO block allocator (host logic)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_455_b200 import workloads as W


def test_fifo_allocator_reuses_released_blocks_in_order():
    a = W.FifoBlockAllocator(range(8))
    assert a.get_blocks(1, 3) == [0, 1, 2]
    assert a.get_blocks(2, 2) == [3, 4]
    a.release_blocks(1)
    # free list is now 5, 6, 7, 0, 1, 2
    assert a.get_blocks(3, 4) == [5, 6, 7, 0]
    a.release_blocks(2)
    assert a.get_blocks(4, 3) == [1, 2, 3]
    owned = [b for blocks in a.block_table.values() for b in blocks]
    assert len(owned) == len(set(owned))


def test_fifo_allocator_overflow_is_an_error_and_changes_nothing():
    a = W.FifoBlockAllocator(range(4))
    a.get_blocks(1, 3)
    with pytest.raises(MemoryError):
        a.get_blocks(2, 2)
    assert a.num_free == 1 and 2 not in a.block_table
    a.release_blocks(99)          # unknown sequence: nothing happens
    assert a.num_free == 1


def test_tiny_config_is_the_pages_3_5_2_example():
    L = W.make_layout(W.CONFIGS["tiny"])
    assert list(L.context_lens) == [3, 5, 2]
    need = [(L.block_tables[b] >= 0).sum() for b in range(3)]
    assert need == [1, 2, 1]
    assert L.num_blocks == 16


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_layout_invariants(name):
    cfg = W.CONFIGS[name]
    L = W.make_layout(cfg)
    bs = cfg.block_size
    assert L.context_lens.shape == (cfg.num_seqs,)
    used = L.block_tables[L.block_tables >= 0]
    assert len(np.unique(used)) == len(used), "a block is owned twice"
    assert used.min() >= 0 and used.max() < L.num_blocks
    for b, ctx in enumerate(L.context_lens):
        n = -(-int(ctx) // bs)
        assert (L.block_tables[b, :n] >= 0).all() and (L.block_tables[b, n:] == -1).all()
        last = int(ctx) - 1
        assert L.slot_mapping[b] == L.block_tables[b, last // bs] * bs + last % bs
    # same seed, same layout
    L2 = W.make_layout(cfg)
    assert np.array_equal(L.block_tables, L2.block_tables)
    assert np.array_equal(L.context_lens, L2.context_lens)


def test_length_distributions():
    q = W.make_layout(W.CONFIGS["qwen"]).context_lens
    assert q.min() >= 128 and q.max() <= 4096
    assert W.make_layout(W.CONFIGS["long"]).context_lens.tolist() == [8192] * 8
    m = W.make_layout(W.CONFIGS["mix"])
    assert m.context_lens.min() >= 1 and m.context_lens.max() <= 32768
    assert 300 < np.median(m.context_lens) < 800
    assert m.notes["history"]["alloc"] + m.notes["history"]["alloc_failed"] \
        + m.notes["history"]["free"] + m.notes["history"]["free_empty"] == 10_000
    p = W.make_layout(W.CONFIGS["pressure"]).context_lens
    assert p.min() >= 1024 and p.max() <= 6144


def test_mix_pool_is_fragmented():
    """After the allocate/free history the batch's blocks are not handed out
    in pool order."""
    m = W.make_layout(W.CONFIGS["mix"])
    first = m.block_tables[:, 0]
    assert not np.all(np.diff(first) > 0)


def test_memory_fit_scale():
    cfg = W.CONFIGS["pressure"]
    L = W.make_layout(cfg)
    per_block = 2 * 16 * 16 * 4 * 256 * 2
    need = L.num_blocks * per_block
    assert W.fit_length_scale(cfg, need + (8 << 30)) == 1.0
    s = W.fit_length_scale(cfg, need // 2 + (8 << 30))
    assert 0.45 < s <= 0.5
    L2 = W.make_layout(cfg, length_scale=s)
    assert L2.num_blocks * per_block <= need // 2 + 1


def test_tensor_contents_nan_outside_context():
    L = W.make_layout(W.CONFIGS["tiny"])
    (layer,) = W.make_layers(L, "cpu")
    nb, bs = L.num_blocks, 4
    flat = layer.k_pool.view(nb * bs, -1)
    valid = set(W.valid_slots(L).tolist())
    for s in range(nb * bs):
        assert bool(torch.isfinite(flat[s]).all()) == (s in valid)
    # the new token's slot is empty before the write
    for s in L.slot_mapping:
        assert torch.isnan(flat[s]).all()
    again = W.make_layers(L, "cpu")[0]
    assert torch.equal(layer.query, again.query)
    assert torch.equal(layer.k_pool.nan_to_num(0), again.k_pool.nan_to_num(0))


def test_compact_sample_relabels_blocks():
    L = W.make_layout(W.CONFIGS["tiny"])
    (layer,) = W.make_layers(L, "cpu")
    s = W.compact_sample(L, layer, [2, 1])
    assert s["block_tables"].tolist() == [[0, -1], [1, 2]]
    assert s["block_map"].tolist() == [L.block_tables[2, 0], L.block_tables[1, 0],
                                       L.block_tables[1, 1]]
    want = W.to_numpy_elems(layer.k_pool[list(L.block_tables[1])])
    assert s["k_pool"][1:3].tobytes() == want.tobytes()
    assert s["slot_mapping"].tolist() == [0 * 4 + 1, 2 * 4 + 0]
