"""The decode kernel's bounded waits, made to run out on purpose.

Every wait inside the decode kernel is bounded; one that runs out sets
PA_DEV_WAIT_TIMEOUT and the kernel returns normally, so the CUDA context stays
usable.  The test hooks of include/pa_testing.h shorten the limit to 2 ms and
make one CTA's producer leave one tile's copies unissued: the stage they would
fill never completes, the CTA's consumer warps give up waiting for it, zero
the outputs of the sequence whose work they held, and count nothing in.  No
fault, trap or hang is involved.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_cache_455_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = 2e-2


def _case(seed, lens, hq=16, hkv=4, d=256, bs=16):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    need = -(-lens // bs)
    nb = int(need.sum()) + 8
    perm = rng.permutation(nb)
    tables = np.full((len(lens), int(need.max())), -1, np.int32)
    pos = 0
    for b in range(len(lens)):
        tables[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = torch.randn(len(lens), hq, d, generator=g, device=DEV).to(torch.bfloat16)
    kp = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    vp = torch.randn(nb, bs, hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    return q, kp, vp, tables, lens


def test_a_wait_that_runs_out_sets_the_status_zeroes_its_outputs_and_leaves_the_context_usable():
    from paged_kv_cache_455_b200 import pa
    # sequence 0 is split over (nearly) every CTA, CTA 1 among them; sequence
    # 1 is short and held by the last CTAs only
    q, kp, vp, tables, lens = _case(21, [8192, 100])
    tab, cl = torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV)
    ws = torch.empty(pa.pa_decode_workspace_bytes(2, 16, 4, 256, 8192), dtype=torch.uint8,
                     device=DEV)
    ref = O.paged_attention(W.to_numpy_elems(q), W.to_numpy_elems(kp), W.to_numpy_elems(vp),
                            tables, lens, 1.0 / 16.0, "bf16")

    def run():
        out = torch.full_like(q, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        pa.pa_decode_attention(out, q, kp, vp, tab, cl, 8192, 1.0 / 16.0, ws, status)
        torch.cuda.synchronize()
        return out, int(status.item())

    pa.testing_set_wait_limit_ns(2_000_000)
    pa.testing_withhold_copy(1)
    try:
        out, status = run()
    finally:
        pa.testing_withhold_copy(-1)
        pa.testing_set_wait_limit_ns(0)
    assert status & pa.PA_DEV_WAIT_TIMEOUT
    assert status & ~pa.PA_DEV_WAIT_TIMEOUT == 0
    assert (out[0].float() == 0).all(), "a sequence whose work was lost must be zeros"
    got1 = out[1].double().cpu().numpy()
    assert np.isfinite(got1).all()
    assert np.abs(got1 - ref[1]).max() <= TOL

    # the context is still usable, and the next call is exact again
    out, status = run()
    assert status == 0
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL


def test_a_wait_that_runs_out_with_merges_inside_the_decode_kernel():
    """Many sequences per CTA: cut segments are merged by their last arriving
    piece inside the decode kernel (no merge pass).  CTA 1's range is lost
    from its second tile on; every output is then exactly zero or matches
    the oracle, some are zero, and the next call is exact."""
    from paged_kv_cache_455_b200 import pa
    lens = [3000 + 37 * i for i in range(48)]
    q, kp, vp, tables, lens = _case(22, lens)
    tab, cl = torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV)
    ws = torch.empty(pa.pa_decode_workspace_bytes(len(lens), 16, 4, 256, int(lens.max())),
                     dtype=torch.uint8, device=DEV)
    ref = O.paged_attention(W.to_numpy_elems(q), W.to_numpy_elems(kp), W.to_numpy_elems(vp),
                            tables, lens, 1.0 / 16.0, "bf16")

    def run():
        out = torch.full_like(q, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        launches = pa.launch_count()
        pa.pa_decode_attention(out, q, kp, vp, tab, cl, int(lens.max()), 1.0 / 16.0, ws, status)
        torch.cuda.synchronize()
        assert pa.launch_count() - launches == 1, "expected no merge pass"
        return out, int(status.item())

    pa.testing_set_wait_limit_ns(2_000_000)
    pa.testing_withhold_copy(1)
    try:
        out, status = run()
    finally:
        pa.testing_withhold_copy(-1)
        pa.testing_set_wait_limit_ns(0)
    assert status & pa.PA_DEV_WAIT_TIMEOUT
    assert status & ~pa.PA_DEV_WAIT_TIMEOUT == 0
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    heads = got.reshape(len(lens), 4, -1)          # per (sequence, KV head group of 4 heads)
    want = ref.reshape(len(lens), 4, -1)
    zero = (heads == 0).all(axis=2)
    exact = np.abs(heads - want).max(axis=2) <= TOL
    assert (zero | exact).all(), "an output is neither zeros nor the oracle's"
    assert zero.any(), "the lost range zeroed nothing"

    out, status = run()
    assert status == 0
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL


def test_a_wait_that_runs_out_over_an_fp8_cache():
    """Two consumer warps per KV head (E4M3 cache): the withheld tile is the
    second warp's first; its partner's hand-off waits run out as well.  The
    long sequence is zeros, the short one exact, the next call exact."""
    import dataclasses
    from paged_kv_cache_455_b200 import pa
    base = W.CONFIGS["qwen"]
    lens = np.array([8192, 100], np.int32)
    bs = 16
    cfg = dataclasses.replace(base, num_seqs=2)
    rng = np.random.default_rng(23)
    need = -(-lens // bs)
    nb = int(need.sum()) + 8
    perm = rng.permutation(nb)
    tables = np.full((2, int(need.max())), -1, np.int32)
    pos = 0
    for b in range(2):
        tables[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    slots = np.array([tables[b, (n - 1) // bs] * bs + (n - 1) % bs for b, n in enumerate(lens)],
                     np.int64)
    layout = W.BatchLayout(cfg, lens, tables, slots, nb)
    (layer,) = W.make_layers_fp8(layout, DEV, layers=1)
    s = W.compact_sample(layout, layer, np.arange(2))
    tab, cl, sl = W.device_metadata(layout, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.pa_reshape_and_cache_fp8(layer.key, layer.value, layer.k_pool, layer.v_pool, sl,
                                W.FP8_SCALE, W.FP8_SCALE, status)
    k_ref, v_ref = O.reshape_and_cache_fp8_np(s["key"], s["value"], s["k_pool"], s["v_pool"],
                                              s["slot_mapping"], W.FP8_SCALE, W.FP8_SCALE)
    ref = O.paged_attention_fp8_np(s["query"], k_ref, v_ref, s["block_tables"],
                                   s["context_lens"], cfg.scale, W.FP8_SCALE, W.FP8_SCALE)
    ws = torch.empty(pa.pa_decode_workspace_bytes(2, 16, 4, 256, 8192), dtype=torch.uint8,
                     device=DEV)

    def run():
        out = torch.full_like(layer.query, float("nan"))
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        pa.pa_decode_attention_fp8(out, layer.query, layer.k_pool, layer.v_pool, tab, cl, 8192,
                                   cfg.scale, W.FP8_SCALE, W.FP8_SCALE, ws, st)
        torch.cuda.synchronize()
        return out, int(st.item())

    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pa.testing_set_wait_limit_ns(2_000_000)
    pa.testing_withhold_copy(1)
    try:
        out, st = run()
    finally:
        pa.testing_withhold_copy(-1)
        pa.testing_set_wait_limit_ns(0)
    assert st & pa.PA_DEV_WAIT_TIMEOUT
    assert st & ~pa.PA_DEV_WAIT_TIMEOUT == 0
    assert (out[0].float() == 0).all(), "a sequence whose work was lost must be zeros"
    got1 = out[1].double().cpu().numpy()
    assert np.isfinite(got1).all()
    assert np.abs(got1 - ref[1]).max() <= TOL

    out, st = run()
    assert st == 0
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL
