"""Copy-on-write block sharing and host swap on the GPU, through the C ABI
("vLLM Architecture, Memory and Benchmarks Deep Dive", section 2,
"Copy-on-Write (CoW) Branching"; "Inside vLLM: Anatomy of a High-Throughput
LLM Inference System", section "Memory-Efficient KV Cache Storage").

pa_copy_blocks must be bit-exact against the oracle's copy over the whole
pools.  A GRPO-shaped run (one prompt, 8 rollouts sharing its blocks, each
appending its own tokens with the block manager's copies) must decode every
rollout within the attention tolerance of the oracle replaying the same
copies and writes, and must never change the shared prompt blocks.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_cache_455_b200 import workloads as W
from paged_kv_cache_455_b200.blocks import BlockManager

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_455_b200 import pa as mod
    return mod


def _pools(nb, bs, hkv, d, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    k = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(tdt)
    v = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(tdt)
    return k, v


@pytest.mark.parametrize("dtype,bs,hkv,d", [("bf16", 16, 4, 256), ("f32", 32, 2, 128),
                                            ("bf16", 4, 1, 64)])
def test_copy_blocks_is_bit_exact(pa, dtype, bs, hkv, d):
    nb = 64
    k, v = _pools(nb, bs, hkv, d, dtype, 3)
    rng = np.random.default_rng(5)
    ids = rng.permutation(nb)
    mapping = np.stack([ids[:20], ids[20:40]], axis=1).astype(np.int64)   # distinct dsts, no chains
    k_ref, v_ref = O.copy_blocks_np(W.to_numpy_elems(k), W.to_numpy_elems(v), mapping)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.pa_copy_blocks(k, v, torch.from_numpy(mapping).to(DEV), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert W.to_numpy_elems(k).tobytes() == k_ref.tobytes()
    assert W.to_numpy_elems(v).tobytes() == v_ref.tobytes()


def test_copy_blocks_skips_bad_pairs_and_reports(pa):
    nb, bs, hkv, d = 16, 16, 4, 256
    k, v = _pools(nb, bs, hkv, d, "bf16", 4)
    k0, v0 = W.to_numpy_elems(k), W.to_numpy_elems(v)
    mapping = np.array([[1, 2], [3, nb], [-1, 4], [5, 6]], dtype=np.int64)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.pa_copy_blocks(k, v, torch.from_numpy(mapping).to(DEV), status)
    torch.cuda.synchronize()
    assert int(status.item()) == pa.PA_DEV_BAD_BLOCK
    k_ref, v_ref = O.copy_blocks_np(k0, v0, mapping[[0, 3]])
    assert W.to_numpy_elems(k).tobytes() == k_ref.tobytes()
    assert W.to_numpy_elems(v).tobytes() == v_ref.tobytes()


def test_grpo_rollouts_share_the_prompt_and_decode_exactly(pa):
    bs, hq, hkv, d, dtype = 16, 16, 4, 256, "bf16"
    prompt, rollouts, steps, nb = 100, 8, 20, 64
    scale = d ** -0.5
    k, v = _pools(nb, bs, hkv, d, dtype, 9)
    k_host, v_host = W.to_numpy_elems(k), W.to_numpy_elems(v)   # the oracle's replay
    m = BlockManager(nb, bs, free_order=np.random.default_rng(1).permutation(nb))
    m.allocate(0, prompt)                   # the prompt's K/V: whatever the pool holds there
    for r in range(1, rollouts + 1):
        m.fork(0, r)
    m.free_seq(0)
    prompt_blocks = list(m.tables[1][:prompt // bs])
    prompt_bytes = k_host[prompt_blocks].tobytes()
    seqs = list(range(1, rollouts + 1))
    g = torch.Generator(device=DEV)
    g.manual_seed(10)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    copies = 0
    for _ in range(steps):
        slots, pairs = [], []
        for r in seqs:
            slot, c = m.append_slot(r)
            slots.append(slot)
            if c is not None:
                pairs.append(c)
        if pairs:
            mapping = np.array(pairs, dtype=np.int64)
            pa.pa_copy_blocks(k, v, torch.from_numpy(mapping).to(DEV), status)
            k_host, v_host = O.copy_blocks_np(k_host, v_host, mapping)
            copies += len(pairs)
        key = torch.randn(rollouts, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
        value = torch.randn(rollouts, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
        slot_t = torch.tensor(slots, dtype=torch.int64, device=DEV)
        pa.pa_reshape_and_cache(key, value, k, v, slot_t, status)
        k_host, v_host = O.reshape_and_cache(W.to_numpy_elems(key), W.to_numpy_elems(value),
                                             k_host, v_host, np.array(slots), dtype)
    torch.cuda.synchronize()
    assert copies == rollouts - 1           # the last holder keeps the shared block
    assert W.to_numpy_elems(k).tobytes() == k_host.tobytes()
    assert W.to_numpy_elems(v).tobytes() == v_host.tobytes()
    assert k_host[prompt_blocks].tobytes() == prompt_bytes   # shared blocks untouched

    tab, lens = m.block_tables(seqs)
    assert (tab[:, :prompt // bs] == np.array(prompt_blocks)).all()
    q = torch.randn(rollouts, hq, d, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(pa.pa_decode_workspace_bytes(rollouts, hq, hkv, d, int(lens.max())),
                     dtype=torch.uint8, device=DEV)
    pa.pa_decode_attention(out, q, k, v, torch.from_numpy(tab).to(DEV),
                           torch.from_numpy(lens).to(DEV), int(lens.max()), scale, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.paged_attention(W.to_numpy_elems(q), k_host, v_host, tab, lens, scale, dtype)
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL[dtype]


def test_swap_out_and_back_in_is_exact_and_decodes_identically(pa):
    bs, hq, hkv, d, nb, host_nb = 16, 16, 4, 256, 48, 24
    k, v = _pools(nb, bs, hkv, d, "bf16", 12)
    m = BlockManager(nb, bs, free_order=np.random.default_rng(2).permutation(nb),
                     num_host_blocks=host_nb)
    m.allocate(0, 200)
    m.allocate(1, 150)
    g = torch.Generator(device=DEV)
    g.manual_seed(13)
    q = torch.randn(2, hq, d, generator=g, device=DEV).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def decode():
        tab, lens = m.block_tables([0, 1])
        out = torch.empty_like(q)
        ws = torch.empty(pa.pa_decode_workspace_bytes(2, hq, hkv, d, int(lens.max())),
                         dtype=torch.uint8, device=DEV)
        pa.pa_decode_attention(out, q, k, v, torch.from_numpy(tab).to(DEV),
                               torch.from_numpy(lens).to(DEV), int(lens.max()), 1 / 16, ws, status)
        torch.cuda.synchronize()
        return out

    before = decode()
    host_k = torch.zeros(host_nb, bs, hkv, d, dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros(host_nb, bs, hkv, d, dtype=torch.bfloat16).pin_memory()
    out_pairs = np.array(m.swap_out(0), dtype=np.int64)
    pa.pa_swap_blocks(host_k, host_v, k, v, torch.from_numpy(out_pairs).to(DEV), status)
    torch.cuda.synchronize()
    zeros = np.zeros_like(W.to_numpy_elems(host_k))
    ref_k, ref_v = O.swap_blocks_np(zeros, zeros, W.to_numpy_elems(k), W.to_numpy_elems(v),
                                    out_pairs)
    assert W.to_numpy_elems(host_k).tobytes() == ref_k.tobytes()
    assert W.to_numpy_elems(host_v).tobytes() == ref_v.tobytes()
    k[torch.from_numpy(out_pairs[:, 0]).to(DEV)] = 0          # the freed blocks get reused
    v[torch.from_numpy(out_pairs[:, 0]).to(DEV)] = 0
    m.allocate(2, 40)
    in_pairs = np.array(m.swap_in(0), dtype=np.int64)
    assert set(in_pairs[:, 1]).isdisjoint(m.tables[2])
    pa.pa_swap_blocks(k, v, host_k, host_v, torch.from_numpy(in_pairs).to(DEV), status)
    after = decode()
    assert int(status.item()) == 0
    assert torch.equal(before, after)       # same data, same tiles: bit-identical
