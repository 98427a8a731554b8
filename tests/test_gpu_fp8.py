"""FP8 (E4M3) cache on the GPU, through the C ABI, against the fp64 oracle.

The oracle reads the same E4M3 pool, dequantises every code exactly and
computes exact softmax attention ("vLLM Architecture, Memory and Benchmarks
Deep Dive", section 4, FP8; "Inside vLLM: Anatomy of a High-Throughput LLM
Inference System", FAQ, quantized KV caches).  Bars: the cache write is
bit-exact over the whole pool (both sides take the rounding decision in
binary32, then to nearest E4M3); attention is within 2e-2 (bf16 outputs of
order 1; the kernel rounds the query and the softmax weights to f16 and
accumulates in fp32).
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_cache_455_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = 2e-2
SC = W.FP8_SCALE


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_455_b200 import pa as mod
    return mod


def _step(pa, layout, layer, workspace=True, scale=None):
    cfg = layout.config
    tables, lens, slots = W.device_metadata(layout, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.pa_reshape_and_cache_fp8(layer.key, layer.value, layer.k_pool, layer.v_pool, slots, SC, SC,
                                status)
    out = torch.full_like(layer.query, float("nan"))
    ws = None
    if workspace:
        ws = torch.empty(pa.pa_decode_workspace_bytes(cfg.num_seqs, cfg.num_q_heads,
                                                      cfg.num_kv_heads, cfg.head_dim,
                                                      layout.max_context_len),
                         dtype=torch.uint8, device=DEV)
    pa.pa_decode_attention_fp8(out, layer.query, layer.k_pool, layer.v_pool, tables, lens,
                               layout.max_context_len, cfg.scale if scale is None else scale,
                               SC, SC, ws, status)
    torch.cuda.synchronize()
    return out, int(status.item())


def _check(pa, cfg, sample=None, workspace=True):
    layout = W.make_layout(cfg)
    (layer,) = W.make_layers_fp8(layout, DEV, layers=1)
    seqs = np.arange(cfg.num_seqs) if sample is None else np.sort(
        np.random.default_rng(cfg.seed + 2000).choice(cfg.num_seqs, sample, replace=False))
    s = W.compact_sample(layout, layer, seqs)                # before the write
    full_k = W.to_numpy_elems(layer.k_pool) if sample is None else None
    full_v = W.to_numpy_elems(layer.v_pool) if sample is None else None
    out, status = _step(pa, layout, layer, workspace)
    assert status == 0
    # cache write: bit-exact
    if sample is None:
        k_ref, v_ref = O.reshape_and_cache_fp8_np(W.to_numpy_elems(layer.key),
                                                  W.to_numpy_elems(layer.value), full_k, full_v,
                                                  layout.slot_mapping, SC, SC)
        assert W.to_numpy_elems(layer.k_pool).tobytes() == k_ref.tobytes()
        assert W.to_numpy_elems(layer.v_pool).tobytes() == v_ref.tobytes()
    k_ref, v_ref = O.reshape_and_cache_fp8_np(s["key"], s["value"], s["k_pool"], s["v_pool"],
                                              s["slot_mapping"], SC, SC)
    after = W.compact_sample(layout, layer, seqs)
    assert after["k_pool"].tobytes() == k_ref.tobytes()
    assert after["v_pool"].tobytes() == v_ref.tobytes()
    ref = O.paged_attention_fp8_np(s["query"], k_ref, v_ref, s["block_tables"],
                                   s["context_lens"], cfg.scale, SC, SC)
    got = out[torch.from_numpy(seqs).to(DEV)].double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL, f"{cfg.name}: max abs error {err}"
    return err


def test_fp8_tiny_shape(pa):
    # the tiny workload's lengths {3, 5, 2} and heads (group 4), at the
    # smallest head dimension and block size an FP8 cache supports
    cfg = dataclasses.replace(W.CONFIGS["tiny"], head_dim=128, block_size=16, dtype="bf16",
                              scale=128 ** -0.5)
    _check(pa, cfg)


def test_fp8_qwen_shaped_full_layer(pa):
    cfg = W.CONFIGS["qwen"]
    _check(pa, cfg, sample=24)


def test_fp8_qwen_shaped_without_workspace(pa):
    _check(pa, W.CONFIGS["qwen"], sample=12, workspace=False)


def test_fp8_long_contexts(pa):
    _check(pa, W.CONFIGS["long"], sample=3)


def test_fp8_mix(pa):
    _check(pa, W.CONFIGS["mix"], sample=24)


@pytest.mark.parametrize("d,hq,hkv,bs", [(256, 16, 4, 16), (128, 8, 8, 32), (128, 16, 2, 16),
                                         (256, 8, 1, 32), (128, 32, 4, 16), (256, 8, 4, 16)])
def test_fp8_every_tail_length(pa, d, hq, hkv, bs):
    """Lengths 1 .. 40 (every position of the last tile), groups 1 to 8."""
    base = W.CONFIGS["qwen"]
    cfg = dataclasses.replace(base, num_seqs=40, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                              block_size=bs, scale=d ** -0.5)
    rng = np.random.default_rng(d + hq + bs)
    lens = np.arange(1, 41)
    need = -(-lens // bs)
    nb = int(need.sum()) + 7
    perm = rng.permutation(nb)
    tables = np.full((40, int(need.max())), -1, np.int32)
    pos = 0
    for b in range(40):
        tables[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    slots = np.array([tables[b, (n - 1) // bs] * bs + (n - 1) % bs for b, n in enumerate(lens)],
                     np.int64)
    layout = W.BatchLayout(cfg, lens.astype(np.int32), tables, slots, nb)
    (layer,) = W.make_layers_fp8(layout, DEV, layers=1)
    s = W.compact_sample(layout, layer, np.arange(40))
    out, status = _step(pa, layout, layer)
    assert status == 0
    k_ref, v_ref = O.reshape_and_cache_fp8_np(s["key"], s["value"], s["k_pool"], s["v_pool"],
                                              s["slot_mapping"], SC, SC)
    ref = O.paged_attention_fp8_np(s["query"], k_ref, v_ref, s["block_tables"],
                                   s["context_lens"], cfg.scale, SC, SC)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL


def test_fp8_block_relabelling_is_bit_identical(pa):
    cfg = dataclasses.replace(W.CONFIGS["qwen"], num_seqs=16)
    layout = W.make_layout(cfg)
    (layer,) = W.make_layers_fp8(layout, DEV, layers=1)
    out1, st1 = _step(pa, layout, layer)
    # move every block to a new place and relabel the tables to match
    perm = torch.randperm(layout.num_blocks, generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(layout.num_blocks)
    k2 = torch.empty_like(layer.k_pool)
    v2 = torch.empty_like(layer.v_pool)
    k2[perm.to(DEV)] = layer.k_pool
    v2[perm.to(DEV)] = layer.v_pool
    tables = layout.block_tables.copy()
    valid = tables >= 0
    tables[valid] = perm.numpy()[tables[valid]]
    slots = layout.slot_mapping.copy()
    bs = cfg.block_size
    slots = perm.numpy()[slots // bs] * bs + slots % bs
    layout2 = W.BatchLayout(cfg, layout.context_lens, tables, slots, layout.num_blocks)
    layer2 = W.LayerTensors(layer.query, layer.key, layer.value, k2, v2)
    out2, st2 = _step(pa, layout2, layer2)
    assert st1 == 0 and st2 == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_fp8_copy_and_swap_are_bit_exact(pa):
    cfg = dataclasses.replace(W.CONFIGS["qwen"], num_seqs=4)
    layout = W.make_layout(cfg)
    (layer,) = W.make_layers_fp8(layout, DEV, layers=1)
    kp0, vp0 = W.to_numpy_elems(layer.k_pool), W.to_numpy_elems(layer.v_pool)
    mapping = np.array([[0, 5], [7, 2], [3, 11]], np.int64)
    pa.pa_copy_blocks(layer.k_pool, layer.v_pool, torch.from_numpy(mapping).to(DEV))
    torch.cuda.synchronize()
    k_ref, v_ref = O.copy_blocks_np(kp0, vp0, mapping)
    assert W.to_numpy_elems(layer.k_pool).tobytes() == k_ref.tobytes()
    assert W.to_numpy_elems(layer.v_pool).tobytes() == v_ref.tobytes()
    host_k = torch.zeros((6,) + tuple(layer.k_pool.shape[1:]), dtype=torch.uint8).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    out_map = np.array([[5, 0], [2, 4]], np.int64)
    pa.pa_swap_blocks(host_k, host_v, layer.k_pool, layer.v_pool,
                      torch.from_numpy(out_map).to(DEV))
    torch.cuda.synchronize()
    hk_ref, hv_ref = O.swap_blocks_np(np.zeros_like(host_k.numpy()), np.zeros_like(host_v.numpy()),
                                      k_ref, v_ref, out_map)
    assert host_k.numpy().tobytes() == hk_ref.tobytes()
    assert host_v.numpy().tobytes() == hv_ref.tobytes()
