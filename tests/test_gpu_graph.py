"""A decode step captured once as a CUDA graph and replayed ("vLLM
Architecture, Memory and Benchmarks Deep Dive", section 4: CUDA Graphs record
the whole step once and replay it, removing per-kernel launch overhead).

Four layers, each with its own pools: per layer the cache write of every
sequence's new token, then decode attention with the caller's workspace.
After each of two replays every layer's pools must equal the oracle's cache
write byte for byte, and every layer's output must match the fp64 oracle
within the bf16 tolerance.
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


def test_captured_four_layer_step_matches_the_oracle_on_every_replay():
    from paged_kv_cache_455_b200 import pa
    # qwen-shaped layers (Hq 16, Hkv 4, d 256, blocks of 16, U[128, 4096]
    # lengths) with 16 sequences, so that the host copies stay small
    cfg = dataclasses.replace(W.CONFIGS["qwen"], num_seqs=16, layers=4)
    layout = W.make_layout(cfg)
    layers = W.make_layers(layout, DEV)
    tables, lens, slots = W.device_metadata(layout, DEV)

    # the oracle's step, from the inputs before any write
    want_pools, want_out = [], []
    for l in layers:
        k_ref, v_ref = O.reshape_and_cache(W.to_numpy_elems(l.key), W.to_numpy_elems(l.value),
                                           W.to_numpy_elems(l.k_pool), W.to_numpy_elems(l.v_pool),
                                           layout.slot_mapping, cfg.dtype)
        want_pools.append((k_ref, v_ref))
        want_out.append(O.paged_attention(W.to_numpy_elems(l.query), k_ref, v_ref,
                                          layout.block_tables, layout.context_lens, cfg.scale,
                                          cfg.dtype))

    ws = torch.empty(pa.pa_decode_workspace_bytes(cfg.num_seqs, cfg.num_q_heads,
                                                  cfg.num_kv_heads, cfg.head_dim,
                                                  layout.max_context_len),
                     dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    outs = [torch.full_like(l.query, float("nan")) for l in layers]

    def step():
        for l, o in zip(layers, outs):
            pa.pa_reshape_and_cache(l.key, l.value, l.k_pool, l.v_pool, slots, status)
            pa.pa_decode_attention(o, l.query, l.k_pool, l.v_pool, tables, lens,
                                   layout.max_context_len, cfg.scale, ws, status)

    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    launches = pa.launch_count()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    assert pa.launch_count() - launches == 2 * len(layers)
    torch.cuda.synchronize()
    # capturing ran nothing: the pools still hold NaN at the new tokens' slots
    for l in layers:
        assert torch.isnan(l.k_pool.float().view(-1, cfg.num_kv_heads, cfg.head_dim)[slots]).all()

    for replay in range(2):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"device status after replay {replay}"
        for i, l in enumerate(layers):
            k_ref, v_ref = want_pools[i]
            assert W.to_numpy_elems(l.k_pool).tobytes() == k_ref.tobytes(), f"layer {i} K pool"
            assert W.to_numpy_elems(l.v_pool).tobytes() == v_ref.tobytes(), f"layer {i} V pool"
            got = outs[i].double().cpu().numpy()
            assert np.isfinite(got).all()
            assert np.abs(got - want_out[i]).max() <= TOL, f"layer {i} output, replay {replay}"
    del graph
