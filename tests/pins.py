"""Pins that tie the oracle to facts outside itself.

Each ``check_*`` function takes an attention implementation with the oracle's
signature ``attn(q, k_pool, v_pool, block_tables, context_lens, scale, dtype)``
and raises AssertionError when the implementation breaks the fact it checks.
``test_oracle_pins`` runs them on both oracle implementations;
``test_oracle_mutants`` runs them on deliberately broken copies of the numpy
oracle to show that each plausible mistake fails at least one of them.

The facts:

* ctx = 1: softmax over one token is 1, so the output is that token's V row.
* all keys of a (sequence, KV head) equal: all weights are equal, so the
  output is the plain mean of the V rows.
* adding one vector u to every key of a KV head adds the constant scale*q.u to
  every logit of each query head, which softmax ignores.
* a key with a logit ~1000 above every other takes all the weight (the others
  underflow to exactly 0 in fp64), so the output is its V row.
* relabelling physical blocks by any permutation (moving the pool rows to
  match) leaves every result bit-identical: the block table only says where
  a logical block lives.  ("High-Throughput LLM Inference & Training: A Deep
  Dive into vLLM", Figure 2: blocks live anywhere in physical memory.)
* a paged cache must look contiguous to attention ("Optimizing LLM Inference:
  A Deep Dive into vLLM's PagedAttention and Continuous Batching", section
  "PagedAttention: Borrowing a 50-Year-Old OS Masterpiece"): attention over a
  paged pool equals torch's scaled_dot_product_attention (fp64, GQA) over the
  same K/V laid out contiguously.
* NaN in slots past each sequence's length and in blocks nobody owns does not
  reach the output.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F


def _to_elems(x: np.ndarray, dtype: str) -> np.ndarray:
    """float values -> the oracle's element encoding (f32 or raw bf16 bits)."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x32
    t = torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _from_elems(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64)
    bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def scatter_to_pool(kc_list, bs: int, num_blocks: int, rng: np.random.Generator,
                    fill=np.nan, dtype="f32"):
    """Places contiguous per-sequence K (or V) [ctx, Hkv, d] arrays into a paged
    pool through a random block table; returns (pool, tables)."""
    hkv, d = kc_list[0].shape[1:]
    need = [-(-k.shape[0] // bs) for k in kc_list]
    if sum(need) > num_blocks:
        raise ValueError("pool too small")
    perm = rng.permutation(num_blocks)
    pool = np.full((num_blocks, bs, hkv, d), fill, dtype=np.float64)
    maxb = max(1, max(need))
    tables = np.full((len(kc_list), maxb), -1, dtype=np.int32)
    pos = 0
    for b, kc in enumerate(kc_list):
        for j in range(need[b]):
            phys = int(perm[pos])
            pos += 1
            tables[b, j] = phys
            rows = kc[j * bs:(j + 1) * bs]
            pool[phys, :rows.shape[0]] = rows
    return _to_elems(pool, dtype), tables


def random_case(rng, B=3, hq=8, hkv=2, d=64, bs=4, lens=(3, 5, 2), dtype="f32",
                spare_blocks=5):
    """Random contiguous K/V per sequence, paged into a NaN-filled pool."""
    kc = [rng.standard_normal((n, hkv, d)) for n in lens]
    vc = [rng.standard_normal((n, hkv, d)) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + spare_blocks
    seed = int(rng.integers(1 << 30))
    kp, tables = scatter_to_pool(kc, bs, nb, np.random.default_rng(seed), dtype=dtype)
    vp, tables2 = scatter_to_pool(vc, bs, nb, np.random.default_rng(seed), dtype=dtype)
    assert np.array_equal(tables, tables2)
    q = _to_elems(rng.standard_normal((B, hq, d)), dtype)
    return {
        "q": q, "k_pool": kp, "v_pool": vp, "block_tables": tables,
        "context_lens": np.asarray(lens, dtype=np.int32),
        # contiguous copies at the element precision, for the library routine
        "kc": [_from_elems(_to_elems(k, dtype), dtype) for k in kc],
        "vc": [_from_elems(_to_elems(v, dtype), dtype) for v in vc],
        "dtype": dtype,
    }


def _run(attn, case, scale):
    return attn(case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                case["context_lens"], scale, case["dtype"])


# --------------------------------------------------------------------------

def check_ctx1_returns_v(attn):
    rng = np.random.default_rng(11)
    for dtype in ("f32", "bf16"):
        case = random_case(rng, B=4, hq=8, hkv=2, d=32, bs=4, lens=(1, 1, 1, 1), dtype=dtype)
        out = _run(attn, case, 0.3)
        for b in range(4):
            for hq in range(8):
                want = case["vc"][b][0, hq // 4]
                assert np.array_equal(out[b, hq], want), "ctx=1 must return the V row"


def check_equal_keys_give_mean(attn):
    rng = np.random.default_rng(12)
    lens = (7, 13, 4)
    hkv, d, bs = 2, 16, 4
    kc = []
    for n in lens:
        k1 = rng.standard_normal((1, hkv, d))
        kc.append(np.repeat(k1, n, axis=0))
    vc = [rng.standard_normal((n, hkv, d)) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + 3
    kp, tab = scatter_to_pool(kc, bs, nb, np.random.default_rng(5))
    vp, _ = scatter_to_pool(vc, bs, nb, np.random.default_rng(5))
    q = _to_elems(rng.standard_normal((3, 4, d)), "f32")
    out = attn(q, kp, vp, tab, np.asarray(lens, np.int32), 0.7, "f32")
    for b, n in enumerate(lens):
        v32 = _from_elems(_to_elems(vc[b], "f32"), "f32")
        for hq in range(4):
            want = v32[:, hq // 2].mean(axis=0)
            np.testing.assert_allclose(out[b, hq], want, rtol=0, atol=1e-12)


def check_key_shift_invariance(attn):
    rng = np.random.default_rng(13)
    case = random_case(rng, B=3, hq=4, hkv=2, d=16, bs=4, lens=(9, 6, 11), dtype="f32")
    # keys on a 1/8 grid and integer shifts keep every shifted key exact in f32
    kq = np.round(case["k_pool"].astype(np.float64) * 8.0) / 8.0
    case = dict(case, k_pool=kq.astype(np.float32))
    base = _run(attn, case, 0.25)
    # shift every key of KV head h by the same vector u_h
    u = rng.integers(-3, 4, size=(2, 16)).astype(np.float64)
    kp = kq + u[None, None, :, :]
    shifted = dict(case, k_pool=kp.astype(np.float32))
    out = _run(attn, shifted, 0.25)
    np.testing.assert_allclose(out, base, rtol=0, atol=1e-12)


def check_dominant_key_takes_all(attn):
    rng = np.random.default_rng(14)
    d, scale = 16, 0.5
    lens = (5, 8)
    q = rng.standard_normal((2, 1, d))
    kc, vc, winners = [], [], []
    for b, n in enumerate(lens):
        k = np.zeros((n, 1, d))
        j = int(rng.integers(n))
        k[j, 0] = q[b, 0] * (1000.0 / (scale * float(q[b, 0] @ q[b, 0])))
        kc.append(k)
        vc.append(rng.standard_normal((n, 1, d)))
        winners.append(j)
    kp, tab = scatter_to_pool(kc, 4, 8, np.random.default_rng(3))
    vp, _ = scatter_to_pool(vc, 4, 8, np.random.default_rng(3))
    out = attn(_to_elems(q, "f32"), kp, vp, tab, np.asarray(lens, np.int32), scale, "f32")
    for b, j in enumerate(winners):
        want = _from_elems(_to_elems(vc[b][j, 0], "f32"), "f32")
        assert np.array_equal(out[b, 0], want), "the dominant key must take all the weight"


def check_block_permutation_invariance(attn):
    rng = np.random.default_rng(15)
    for dtype in ("f32", "bf16"):
        case = random_case(rng, B=4, hq=8, hkv=4, d=32, bs=4, lens=(1, 9, 16, 23),
                           dtype=dtype, spare_blocks=7)
        base = _run(attn, case, 0.2)
        nb = case["k_pool"].shape[0]
        for _ in range(3):
            pi = rng.permutation(nb)
            kp = np.empty_like(case["k_pool"])
            vp = np.empty_like(case["v_pool"])
            kp[pi] = case["k_pool"]
            vp[pi] = case["v_pool"]
            tab = np.where(case["block_tables"] >= 0, pi[np.maximum(case["block_tables"], 0)], -1)
            out = _run(attn, dict(case, k_pool=kp, v_pool=vp, block_tables=tab.astype(np.int32)),
                       0.2)
            assert np.array_equal(out, base), "relabelling physical blocks changed the result"


def _sdpa(q64, kc, vc, scale):
    """torch scaled_dot_product_attention (fp64, GQA) of one sequence."""
    qt = torch.from_numpy(q64)[None, :, None, :]                  # [1, Hq, 1, d]
    kt = torch.from_numpy(np.ascontiguousarray(kc.transpose(1, 0, 2)))[None]   # [1,Hkv,ctx,d]
    vt = torch.from_numpy(np.ascontiguousarray(vc.transpose(1, 0, 2)))[None]
    o = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)
    return o[0, :, 0, :].numpy()


def check_matches_unpaged_sdpa(attn):
    rng = np.random.default_rng(16)
    shapes = [
        dict(B=3, hq=8, hkv=2, d=64, bs=4, lens=(3, 5, 2)),
        dict(B=4, hq=16, hkv=4, d=32, bs=16, lens=(1, 17, 40, 16)),
        dict(B=2, hq=6, hkv=3, d=16, bs=8, lens=(8, 29)),
        dict(B=3, hq=4, hkv=4, d=16, bs=32, lens=(30, 2, 32)),    # MHA; one block each
        dict(B=2, hq=8, hkv=1, d=16, bs=4, lens=(12, 7)),         # MQA
    ]
    for dtype in ("f32", "bf16"):
        for sh in shapes:
            case = random_case(rng, dtype=dtype, **sh)
            scale = float(rng.uniform(0.05, 0.6))
            out = _run(attn, case, scale)
            q64 = _from_elems(case["q"], dtype)
            for b in range(sh["B"]):
                want = _sdpa(q64[b], case["kc"][b], case["vc"][b], scale)
                np.testing.assert_allclose(out[b], want, rtol=0, atol=1e-12)


def check_nan_outside_context_is_ignored(attn):
    rng = np.random.default_rng(17)
    case = random_case(rng, B=3, hq=4, hkv=2, d=16, bs=8, lens=(3, 9, 14), spare_blocks=4)
    assert np.isnan(case["k_pool"]).any()
    out = _run(attn, case, 0.3)
    assert np.isfinite(out).all(), "NaN outside the contexts reached the output"
    clean = dict(case, k_pool=np.nan_to_num(case["k_pool"], nan=7.0),
                 v_pool=np.nan_to_num(case["v_pool"], nan=-7.0))
    assert np.array_equal(_run(attn, clean, 0.3), out)


ALL_CHECKS = [
    check_ctx1_returns_v,
    check_equal_keys_give_mean,
    check_key_shift_invariance,
    check_dominant_key_takes_all,
    check_block_permutation_invariance,
    check_matches_unpaged_sdpa,
    check_nan_outside_context_is_ignored,
]
