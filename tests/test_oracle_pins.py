"""The oracle pinned to the pages' printed values and to mathematical facts.

Every check in ``pins.py`` runs against both oracle implementations (the C
fp64 code and its numpy twin); the two are also compared with each other.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O
import pins

IMPLS = {"c": O.paged_attention, "numpy": O.paged_attention_np}


def test_kv_bytes_matches_the_pages_worked_example(golden_dir):
    with open(os.path.join(golden_dir, "kv_bytes.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        got = O.kv_bytes(c["layers"], c["kv_heads"], c["head_dim"], c["tokens"],
                         c["bytes_per_elem"])
        assert got == c["expected_bytes"]
        assert got / 2**30 == c["expected_gib"]
        assert round(got / 1e9, 2) == c["expected_gb_decimal_2dp"]


def test_kv_bytes_is_linear_in_each_factor():
    base = O.kv_bytes(16, 4, 256, 8192, 2)
    assert O.kv_bytes(32, 4, 256, 8192, 2) == 2 * base
    assert O.kv_bytes(16, 8, 256, 8192, 2) == 2 * base
    assert O.kv_bytes(16, 4, 128, 8192, 2) == base // 2
    assert O.kv_bytes(16, 4, 256, 1, 2) * 8192 == base
    assert O.kv_bytes(16, 4, 256, 8192, 4) == 2 * base


def test_reservation_counts_match_figures_1_and_2(golden_dir):
    with open(os.path.join(golden_dir, "reservation_3_5_2.json")) as f:
        g = json.load(f)
    r = O.reservation_counts(g["lengths"], g["max_len"], g["block_size"])
    c, p = r["contiguous"], r["paged"]
    assert (c["reserved"], c["used"], c["unused"]) == (
        g["contiguous"]["reserved"], g["contiguous"]["used"], g["contiguous"]["unused"])
    assert round(100 * c["unused_frac"]) == g["contiguous"]["unused_pct_rounded"]
    assert (p["reserved"], p["used"], p["unused"], p["freed"]) == (
        g["paged"]["reserved"], g["paged"]["used"], g["paged"]["unused"], g["paged"]["freed"])
    blocks = [-(-n // g["block_size"]) for n in g["lengths"]]
    assert blocks == g["paged"]["blocks"]


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(impl, check):
    check(IMPLS[impl])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_c_and_numpy_oracles_agree(dtype):
    rng = np.random.default_rng(21)
    for sh in [dict(B=3, hq=8, hkv=2, d=64, bs=4, lens=(3, 5, 2)),
               dict(B=5, hq=16, hkv=4, d=256, bs=16, lens=(1, 15, 16, 17, 300)),
               dict(B=2, hq=16, hkv=4, d=128, bs=32, lens=(33, 97))]:
        case = pins.random_case(rng, dtype=dtype, **sh)
        args = (case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                case["context_lens"], 0.0625, dtype)
        a = O.paged_attention(*args)
        b = O.paged_attention_np(*args)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
        # one thread and many threads give the same bits
        assert np.array_equal(O.paged_attention(*args, num_threads=1), a)


def test_zero_length_sequence_gives_zeros():
    rng = np.random.default_rng(22)
    case = pins.random_case(rng, B=3, hq=4, hkv=2, d=16, bs=4, lens=(3, 1, 2))
    case["context_lens"] = np.asarray([3, 0, 2], np.int32)
    for impl in IMPLS.values():
        out = impl(case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                   case["context_lens"], 0.5, "f32")
        assert np.array_equal(out[1], np.zeros_like(out[1]))
        assert np.isfinite(out).all()


def test_c_oracle_rejects_bad_block_ids_and_lengths():
    rng = np.random.default_rng(23)
    case = pins.random_case(rng, B=3, hq=4, hkv=2, d=16, bs=4, lens=(3, 5, 2))
    bad = case["block_tables"].copy()
    bad[1, 1] = case["k_pool"].shape[0]
    with pytest.raises(ValueError):
        O.paged_attention(case["q"], case["k_pool"], case["v_pool"], bad,
                          case["context_lens"], 0.5, "f32")
    too_long = np.asarray([3, 5, 4 * case["block_tables"].shape[1] + 1], np.int32)
    with pytest.raises(ValueError):
        O.paged_attention(case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                          too_long, 0.5, "f32")


# -- split over context partitions ------------------------------------------

@pytest.mark.parametrize("impl", ["c", "numpy"])
def test_partition_merge_reproduces_unsplit_attention(impl):
    part = O.partition_attention if impl == "c" else O.partition_attention_np
    rng = np.random.default_rng(24)
    for dtype in ("f32", "bf16"):
        case = pins.random_case(rng, B=4, hq=8, hkv=2, d=32, bs=4, lens=(1, 7, 33, 64),
                                dtype=dtype)
        args = (case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
                case["context_lens"], 0.3, dtype)
        full = O.paged_attention(*args)
        for P in (4, 8, 12, 64, 100):
            maxp = -(-64 // P)
            po, pm, ps = part(*args, P, maxp)
            np.testing.assert_allclose(O.merge_partitions(po, pm, ps), full, rtol=0, atol=1e-12)


def test_each_partition_is_attention_over_its_own_tokens():
    """Partition p (P a multiple of the block size) equals plain attention over
    a sequence made of that partition's blocks only."""
    rng = np.random.default_rng(25)
    case = pins.random_case(rng, B=2, hq=4, hkv=2, d=16, bs=4, lens=(21, 30))
    P = 8
    args = (case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
            case["context_lens"], 0.4, "f32")
    po, pm, ps = O.partition_attention(*args, P, 4)
    for b, ctx in enumerate(case["context_lens"]):
        for p in range(4):
            t0, t1 = p * P, min((p + 1) * P, int(ctx))
            if t1 <= t0:
                assert pm[b, 0, p] == -np.inf and ps[b, 0, p] == 0
                continue
            sub = case["block_tables"][b, t0 // 4:].copy()[None]
            want = O.paged_attention(case["q"][b:b + 1], case["k_pool"], case["v_pool"], sub,
                                     np.asarray([t1 - t0], np.int32), 0.4, "f32")
            np.testing.assert_allclose(po[b, :, p], want[0], rtol=0, atol=1e-12)
            # the max logit is attained by a token of the partition and the
            # sum counts that token with weight exp(0) = 1
            assert np.all(ps[b, :, p] >= 1.0) and np.all(ps[b, :, p] <= t1 - t0)


def test_c_and_numpy_partitions_agree():
    rng = np.random.default_rng(26)
    case = pins.random_case(rng, B=3, hq=16, hkv=4, d=64, bs=16, lens=(5, 100, 257),
                            dtype="bf16")
    args = (case["q"], case["k_pool"], case["v_pool"], case["block_tables"],
            case["context_lens"], 0.125, "bf16", 64, 5)
    a = O.partition_attention(*args)
    b = O.partition_attention_np(*args)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)


# -- cache write --------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_cache_write_places_rows_and_touches_nothing_else(dtype):
    rng = np.random.default_rng(27)
    nb, bs, hkv, d, T = 6, 4, 2, 8, 5
    pool = pins._to_elems(np.full((nb, bs, hkv, d), np.nan), dtype)
    key = pins._to_elems(rng.standard_normal((T, hkv, d)), dtype)
    value = pins._to_elems(rng.standard_normal((T, hkv, d)), dtype)
    slots = np.array([0, 23, -1, 9, 14], dtype=np.int64)
    k2, v2 = O.reshape_and_cache(key, value, pool, pool, slots, dtype)
    k3, v3 = O.reshape_and_cache_np(key, value, pool, pool, slots)
    assert k2.tobytes() == k3.tobytes() and v2.tobytes() == v3.tobytes()
    flat_k = k2.reshape(nb * bs, hkv, d)
    flat_v = v2.reshape(nb * bs, hkv, d)
    written = set()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        assert flat_k[s].tobytes() == key[t].tobytes()
        assert flat_v[s].tobytes() == value[t].tobytes()
        written.add(int(s))
    untouched = [i for i in range(nb * bs) if i not in written]
    assert flat_k[untouched].tobytes() == pool.reshape(nb * bs, hkv, d)[untouched].tobytes()


def test_cache_write_rejects_slots_past_the_pool():
    pool = np.zeros((2, 4, 1, 8), np.float32)
    kv = np.ones((1, 1, 8), np.float32)
    with pytest.raises(ValueError):
        O.reshape_and_cache(kv, kv, pool, pool, np.array([8], np.int64), "f32")
