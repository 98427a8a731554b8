"""CUDA path vs the fp64 oracle, through the C ABI, on the GPU.

Tolerances: cache writes bit-exact; attention max |gpu - oracle| <= 1e-5 for
fp32 data and <= 2e-2 for bf16 data (fp32 accumulation on the GPU, outputs of
order 1).  Every workload configuration runs one full-size layer in the same
launch configuration the benchmark times (the library's preferred split);
the oracle checks every sequence where it finishes in seconds and a seeded
sample of sequences otherwise.
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_cache_455_b200 import workloads as W
import pins

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_455_b200 import pa as mod
    return mod


def _elems(t):
    return W.to_numpy_elems(t)


def _to_dev(a: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16" and a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(DEV)


def gpu_step(pa, q, key, value, k_pool, v_pool, tables, lens, slots, max_ctx, scale,
             workspace="preferred", status=None):
    """One decode step on the GPU: cache write, then attention."""
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.pa_reshape_and_cache(key, value, k_pool, v_pool, slots, status)
    out = torch.full_like(q, float("nan"))
    B, hq, d = q.shape
    ws = None
    if workspace == "preferred":
        nbytes = pa.pa_decode_workspace_bytes(B, hq, k_pool.shape[2], d, max_ctx)
        if nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    elif workspace is not None:
        ws = workspace
    pa.pa_decode_attention(out, q, k_pool, v_pool, tables, lens, max_ctx, scale, ws, status)
    torch.cuda.synchronize()
    return out, int(status.item())


def max_err(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu.detach().float().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite GPU output"
    return float(np.abs(g - ref).max()) if g.size else 0.0


# ---------------------------------------------------------------------------
# The five workload configurations
# ---------------------------------------------------------------------------

def _check_config(pa, name, sample=None, whole_pool_check=True):
    cfg = W.CONFIGS[name]
    layout = W.make_layout(cfg)
    (layer,) = W.make_layers(layout, DEV, layers=1)
    tables, lens, slots = W.device_metadata(layout, DEV)
    seqs = np.arange(cfg.num_seqs) if sample is None else np.sort(
        np.random.default_rng(cfg.seed + 1000).choice(cfg.num_seqs, sample, replace=False))
    s = W.compact_sample(layout, layer, seqs)                    # inputs before the write
    pool_before = None
    if whole_pool_check:
        kp0, vp0 = _elems(layer.k_pool), _elems(layer.v_pool)
    else:
        pool_before = (layer.k_pool.clone(), layer.v_pool.clone())

    out, status = gpu_step(pa, layer.query, layer.key, layer.value, layer.k_pool, layer.v_pool,
                           tables, lens, slots, layout.max_context_len, cfg.scale)
    assert status == 0

    # cache write: bit-exact
    if whole_pool_check:
        k_ref, v_ref = O.reshape_and_cache(_elems(layer.key), _elems(layer.value), kp0, vp0,
                                           layout.slot_mapping, cfg.dtype)
        assert _elems(layer.k_pool).tobytes() == k_ref.tobytes()
        assert _elems(layer.v_pool).tobytes() == v_ref.tobytes()
    else:
        # every slot but the written ones is unchanged (bitwise) ...
        written = torch.from_numpy(layout.slot_mapping[layout.slot_mapping >= 0]).to(DEV)
        for after, before in zip((layer.k_pool, layer.v_pool), pool_before):
            a = after.view(-1, cfg.num_kv_heads * cfg.head_dim).view(torch.int16)
            b = before.view(-1, cfg.num_kv_heads * cfg.head_dim).view(torch.int16)
            keep = torch.ones(a.shape[0], dtype=torch.bool, device=DEV)
            keep[written] = False
            assert torch.equal(a[keep], b[keep])
        del pool_before
    # ... and the sampled sequences' blocks equal the oracle's write
    k_ref, v_ref = O.reshape_and_cache(s["key"], s["value"], s["k_pool"], s["v_pool"],
                                       s["slot_mapping"], cfg.dtype)
    idx = torch.from_numpy(s["block_map"].astype(np.int64)).to(DEV)
    assert _elems(layer.k_pool[idx]).tobytes() == k_ref.tobytes()
    assert _elems(layer.v_pool[idx]).tobytes() == v_ref.tobytes()

    # attention on the sampled sequences
    ref = O.paged_attention(s["query"], k_ref, v_ref, s["block_tables"], s["context_lens"],
                            cfg.scale, cfg.dtype)
    err = max_err(out[torch.from_numpy(seqs).to(DEV)], ref)
    assert err <= TOL[cfg.dtype], f"{name}: max abs error {err}"
    return err


def test_tiny_config(pa):
    _check_config(pa, "tiny")


def test_qwen_config_full_layer(pa):
    _check_config(pa, "qwen")


def test_long_config_full_layer(pa):
    _check_config(pa, "long")


def test_mix_config_full_layer(pa):
    _check_config(pa, "mix")


def test_pressure_config_full_layer_sampled(pa):
    _check_config(pa, "pressure", sample=48, whole_pool_check=False)


# ---------------------------------------------------------------------------
# Random small cases (shapes, tails, groups, block sizes)
# ---------------------------------------------------------------------------

def _case(rng, dtype, **shape):
    """A pins.random_case whose last token of each sequence is the new token:
    its pool slot is emptied (NaN) and its K/V passed to the cache write."""
    c = pins.random_case(rng, dtype=dtype, **shape)
    bs = c["k_pool"].shape[1]
    hkv, d = c["k_pool"].shape[2:]
    B = len(c["context_lens"])
    kp, vp = c["k_pool"].copy(), c["v_pool"].copy()
    key = np.zeros((B, hkv, d), kp.dtype)
    value = np.zeros((B, hkv, d), kp.dtype)
    slots = np.full(B, -1, np.int64)
    nan = pins._to_elems(np.full((hkv, d), np.nan), dtype)
    for b, ctx in enumerate(c["context_lens"]):
        if ctx == 0:
            continue
        t = int(ctx) - 1
        blk, off = int(c["block_tables"][b, t // bs]), t % bs
        key[b], value[b] = kp[blk, off], vp[blk, off]
        kp[blk, off] = nan
        vp[blk, off] = nan
        slots[b] = blk * bs + off
    c.update(k_pool_empty=kp, v_pool_empty=vp, key=key, value=value, slots=slots)
    return c


def _run_case(pa, c, scale, workspace="preferred", max_ctx=None):
    dt = c["dtype"]
    q = _to_dev(c["q"], dt)
    kp, vp = _to_dev(c["k_pool_empty"], dt), _to_dev(c["v_pool_empty"], dt)
    key, value = _to_dev(c["key"], dt), _to_dev(c["value"], dt)
    tables = torch.from_numpy(c["block_tables"]).to(DEV)
    lens = torch.from_numpy(c["context_lens"]).to(DEV)
    slots = torch.from_numpy(c["slots"]).to(DEV)
    mc = int(c["context_lens"].max()) if max_ctx is None else max_ctx
    out, status = gpu_step(pa, q, key, value, kp, vp, tables, lens, slots, mc, scale, workspace)
    return out, status, kp, vp


def _oracle_case(c, scale):
    k_ref, v_ref = O.reshape_and_cache(c["key"], c["value"], c["k_pool_empty"],
                                       c["v_pool_empty"], c["slots"], c["dtype"])
    return O.paged_attention(c["q"], k_ref, v_ref, c["block_tables"], c["context_lens"], scale,
                             c["dtype"]), k_ref, v_ref


SHAPES = [
    dict(B=3, hq=8, hkv=2, d=64, bs=4, lens=(3, 5, 2)),
    dict(B=5, hq=16, hkv=4, d=256, bs=16, lens=(1, 15, 16, 17, 700)),
    dict(B=4, hq=16, hkv=4, d=256, bs=32, lens=(31, 32, 33, 1000)),
    dict(B=3, hq=8, hkv=8, d=128, bs=8, lens=(9, 300, 77)),            # MHA
    dict(B=3, hq=16, hkv=2, d=128, bs=16, lens=(1, 513, 260)),         # group 8
    dict(B=2, hq=4, hkv=2, d=64, bs=8, lens=(1000, 3)),                # group 2
    dict(B=6, hq=8, hkv=1, d=64, bs=4, lens=(1, 2, 3, 4, 5, 600)),      # MQA-like group 8
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{B}_hq{hq}_hkv{hkv}_d{d}_bs{bs}".format(**s))
def test_random_shapes_match_oracle(pa, dtype, shape):
    rng = np.random.default_rng(zlib.crc32(repr((dtype, sorted(shape.items()))).encode()))
    c = _case(rng, dtype, **shape)
    scale = 1.0 / np.sqrt(shape["d"])
    ref, k_ref, v_ref = _oracle_case(c, scale)
    for ws in ("preferred", None):
        out, status, kp, vp = _run_case(pa, c, scale, ws)
        assert status == 0
        assert _elems(kp).tobytes() == k_ref.tobytes()
        assert _elems(vp).tobytes() == v_ref.tobytes()
        assert max_err(out, ref) <= TOL[dtype]


def test_every_tail_length(pa):
    """Lengths 1..80 cover every ragged tail of a 16-token tile and of 4- to
    32-token blocks, at several partition counts."""
    rng = np.random.default_rng(31)
    for bs in (4, 8, 16, 32):
        c = _case(rng, "bf16", B=80, hq=16, hkv=4, d=64, bs=bs, lens=tuple(range(1, 81)))
        ref, _, _ = _oracle_case(c, 0.125)
        out, status, _, _ = _run_case(pa, c, 0.125)
        assert status == 0 and max_err(out, ref) <= TOL["bf16"]


def test_ctx1_returns_v_exactly(pa):
    rng = np.random.default_rng(32)
    for dtype in ("f32", "bf16"):
        c = _case(rng, dtype, B=4, hq=16, hkv=4, d=256, bs=16, lens=(1, 1, 1, 1))
        out, status, _, _ = _run_case(pa, c, 0.0625)
        want = pins._from_elems(c["value"], dtype).repeat(4, axis=1)
        got = out.float().cpu().double().numpy()
        assert status == 0 and np.array_equal(got, want)


def test_zero_length_gives_zeros(pa):
    rng = np.random.default_rng(33)
    c = _case(rng, "bf16", B=3, hq=16, hkv=4, d=128, bs=16, lens=(40, 1, 300))
    c["context_lens"] = np.asarray([40, 0, 300], np.int32)
    c["slots"][1] = -1
    ref, _, _ = _oracle_case(c, 0.1)
    out, status, _, _ = _run_case(pa, c, 0.1)
    assert status == 0
    assert torch.count_nonzero(out[1]) == 0
    assert max_err(out, ref) <= TOL["bf16"]


def test_context_at_table_capacity(pa):
    rng = np.random.default_rng(34)
    c = _case(rng, "bf16", B=2, hq=16, hkv=4, d=256, bs=16, lens=(640, 5))
    assert c["block_tables"].shape[1] * 16 == 640
    ref, _, _ = _oracle_case(c, 0.0625)
    out, status, _, _ = _run_case(pa, c, 0.0625, max_ctx=640)
    assert status == 0 and max_err(out, ref) <= TOL["bf16"]


def test_split_and_unsplit_agree(pa):
    rng = np.random.default_rng(35)
    c = _case(rng, "bf16", B=4, hq=16, hkv=4, d=256, bs=16, lens=(2000, 1, 257, 4096))
    a, _, _, _ = _run_case(pa, c, 0.0625, "preferred")
    b, _, _, _ = _run_case(pa, c, 0.0625, None)
    small = torch.empty(pa.pa_splitk_workspace_bytes(4, 16, 256, 3), dtype=torch.uint8,
                        device=DEV)
    d, _, _, _ = _run_case(pa, c, 0.0625, small)       # fits only 3 partitions
    ref, _, _ = _oracle_case(c, 0.0625)
    for x in (a, b, d):
        assert max_err(x, ref) <= TOL["bf16"]
    assert (a.float() - b.float()).abs().max().item() <= 2e-2


def test_block_relabelling_is_bit_identical(pa):
    rng = np.random.default_rng(36)
    c = _case(rng, "bf16", B=4, hq=16, hkv=4, d=256, bs=16, lens=(100, 1500, 33, 700),
              spare_blocks=30)
    base, _, _, _ = _run_case(pa, c, 0.0625)
    nb = c["k_pool"].shape[0]
    for _ in range(2):
        pi = rng.permutation(nb)
        c2 = dict(c)
        for k in ("k_pool_empty", "v_pool_empty"):
            x = np.empty_like(c[k])
            x[pi] = c[k]
            c2[k] = x
        t = c["block_tables"]
        c2["block_tables"] = np.where(t >= 0, pi[np.maximum(t, 0)], -1).astype(np.int32)
        bs = 16
        c2["slots"] = np.array([pi[s // bs] * bs + s % bs if s >= 0 else -1 for s in c["slots"]],
                               np.int64)
        out, _, _, _ = _run_case(pa, c2, 0.0625)
        assert torch.equal(out.view(torch.int16), base.view(torch.int16))


def test_simt_and_mma_bf16_paths_both_match(pa, monkeypatch):
    rng = np.random.default_rng(37)
    c = _case(rng, "bf16", B=5, hq=16, hkv=4, d=256, bs=16, lens=(1, 16, 17, 900, 2500))
    ref, _, _ = _oracle_case(c, 0.0625)
    mma, _, _, _ = _run_case(pa, c, 0.0625)
    monkeypatch.setenv("PA_DECODE_MATH", "simt")
    simt, _, _, _ = _run_case(pa, c, 0.0625)
    monkeypatch.delenv("PA_DECODE_MATH")
    assert max_err(mma, ref) <= TOL["bf16"]
    assert max_err(simt, ref) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# Explicit split-K API
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_explicit_splitk_partials_and_reduce(pa, dtype):
    rng = np.random.default_rng(38)
    c = _case(rng, dtype, B=4, hq=16, hkv=4, d=128, bs=16, lens=(1, 100, 512, 1111))
    P, maxp = 256, 5
    k_ref, v_ref = O.reshape_and_cache(c["key"], c["value"], c["k_pool_empty"],
                                       c["v_pool_empty"], c["slots"], dtype)
    po, pm, ps = O.partition_attention(c["q"], k_ref, v_ref, c["block_tables"],
                                       c["context_lens"], 0.09, dtype, P, maxp)
    full = O.paged_attention(c["q"], k_ref, v_ref, c["block_tables"], c["context_lens"], 0.09,
                             dtype)
    q = _to_dev(c["q"], dtype)
    kp, vp = _to_dev(k_ref, dtype), _to_dev(v_ref, dtype)
    tables = torch.from_numpy(c["block_tables"]).to(DEV)
    lens = torch.from_numpy(c["context_lens"]).to(DEV)
    B, hq, d = q.shape
    tmp = torch.full((B, hq, maxp, d), float("nan"), device=DEV)
    ml = torch.full((B, hq, maxp), float("nan"), device=DEV)
    es = torch.full((B, hq, maxp), float("nan"), device=DEV)
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_splitk(out, q, kp, vp, tables, lens, 1111, 0.09, P, tmp, ml, es)
    pa.pa_splitk_reduce(out, tmp, ml, es, lens, P)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    for b, ctx in enumerate(c["context_lens"]):
        n = max(1, -(-int(ctx) // P))
        g_ml = ml[b, :, :n].double().cpu().numpy()
        g_es = es[b, :, :n].double().cpu().numpy()
        g_tmp = tmp[b, :, :n].double().cpu().numpy()
        # partition maxima are logits: compared against fp64 with the
        # output tolerance scaled by the logit magnitude
        assert np.abs(g_ml - pm[b, :, :n]).max() <= tol * max(1.0, np.abs(pm[b, :, :n]).max())
        assert np.abs(g_es / ps[b, :, :n] - 1).max() <= 5 * tol
        assert np.abs(g_tmp - po[b, :, :n]).max() <= tol
        assert torch.isnan(tmp[b, :, n:]).all()          # untouched past n_b
    assert max_err(out, full) <= tol


# ---------------------------------------------------------------------------
# Device-side error reporting (no trap, finite output)
# ---------------------------------------------------------------------------

def test_bad_block_id_sets_status_and_zeroes_that_head(pa):
    rng = np.random.default_rng(39)
    c = _case(rng, "bf16", B=3, hq=16, hkv=4, d=64, bs=16, lens=(50, 60, 70))
    c["block_tables"] = c["block_tables"].copy()
    c["block_tables"][1, 2] = 1 << 20                   # past the pool
    c["slots"][1] = -1                                  # keep the write valid
    out, status, _, _ = _run_case(pa, c, 0.125, None)
    assert status & 2
    assert torch.isfinite(out.float()).all()
    assert torch.count_nonzero(out[1]) == 0
    good = [0, 2]
    k_ref, v_ref = O.reshape_and_cache(c["key"], c["value"], c["k_pool_empty"],
                                       c["v_pool_empty"], c["slots"], "bf16")
    ref = O.paged_attention(c["q"][good], k_ref, v_ref, c["block_tables"][good],
                            c["context_lens"][good], 0.125, "bf16")
    assert max_err(out[good], ref) <= TOL["bf16"]


def test_bad_slot_and_bad_context_set_status(pa):
    rng = np.random.default_rng(40)
    c = _case(rng, "f32", B=2, hq=8, hkv=2, d=64, bs=4, lens=(5, 6))
    c["slots"] = np.asarray([c["slots"][0], 10**9], np.int64)
    out, status, kp, _ = _run_case(pa, c, 0.125)
    assert status & 1
    c2 = _case(rng, "f32", B=2, hq=8, hkv=2, d=64, bs=4, lens=(5, 6))
    c2["context_lens"] = np.asarray([5, -3], np.int32)
    c2["slots"][1] = -1
    out, status, _, _ = _run_case(pa, c2, 0.125, max_ctx=6)
    assert status & 4
    assert torch.count_nonzero(out[1]) == 0 and torch.isfinite(out).all()
