"""Pins of the chunked-prefill oracle ("vLLM Architecture, Memory and
Benchmarks Deep Dive", section 4, chunked prefill: a long prompt is cut into
chunks that attend, causally, to everything cached before them and to
themselves).  Each pin ties the oracle to something outside it."""
import inspect

import numpy as np
import pytest
import torch

from oracle import oracle as O
import pins


def _case(rng, lens, chunk, hq=8, hkv=2, d=16, bs=4):
    """Pools with the given contexts; sequence b's chunk is its last chunk[b] tokens."""
    kc = [rng.standard_normal((n, hkv, d)).astype(np.float32) for n in lens]
    vc = [rng.standard_normal((n, hkv, d)).astype(np.float32) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + 3
    k_pool, tables = pins.scatter_to_pool(kc, bs, nb, rng)
    v_pool = np.full_like(k_pool, np.nan)        # V through the same tables
    for b, n in enumerate(lens):
        t = np.arange(n)
        v_pool[tables[b][t // bs], t % bs] = vc[b]
    cu = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int64)
    q = rng.standard_normal((int(cu[-1]), hq, d)).astype(np.float32)
    return q, k_pool, v_pool, tables, np.array(lens, np.int32), cu, kc, vc


def test_one_token_chunks_are_decode():
    rng = np.random.default_rng(1)
    q, kp, vp, tab, lens, cu, _, _ = _case(rng, [5, 9, 1, 13], [1, 1, 1, 1])
    pre = O.prefill_attention_np(q, kp, vp, tab, lens, cu, 0.3, "f32")
    dec = O.paged_attention_np(q, kp, vp, tab, lens, 0.3, "f32")
    assert np.abs(pre - dec).max() <= 1e-12


def test_whole_prompt_chunk_is_causal_sdpa():
    rng = np.random.default_rng(2)
    lens = [7, 12]
    q, kp, vp, tab, lens_a, cu, kc, vc = _case(rng, lens, lens)
    pre = O.prefill_attention_np(q, kp, vp, tab, lens_a, cu, 0.25, "f32")
    for b, n in enumerate(lens):
        qt = torch.from_numpy(q[cu[b]:cu[b + 1]]).double().transpose(0, 1)      # [Hq, n, d]
        kt = torch.from_numpy(kc[b]).double().transpose(0, 1).repeat_interleave(4, dim=0)
        vt = torch.from_numpy(vc[b]).double().transpose(0, 1).repeat_interleave(4, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                               scale=0.25)
        assert np.abs(pre[cu[b]:cu[b + 1]] - ref.transpose(0, 1).numpy()).max() <= 1e-12


def test_rows_ignore_keys_after_their_position():
    rng = np.random.default_rng(3)
    q, kp, vp, tab, lens, cu, _, _ = _case(rng, [11], [6])
    base = O.prefill_attention_np(q, kp, vp, tab, lens, cu, 0.3, "f32")
    bs = kp.shape[1]
    for p in range(11 - 6, 11):
        k2, v2 = kp.copy(), vp.copy()
        for t in range(p + 1, 11):                 # every key after position p
            k2[tab[0][t // bs], t % bs] += 5.0
            v2[tab[0][t // bs], t % bs] -= 3.0
        out = O.prefill_attention_np(q, k2, v2, tab, lens, cu, 0.3, "f32")
        row = p - (11 - 6)
        assert np.array_equal(out[row], base[row])
        if row + 1 < 6:
            assert not np.array_equal(out[row + 1:], base[row + 1:])


def test_splitting_a_chunk_changes_nothing():
    rng = np.random.default_rng(4)
    q, kp, vp, tab, lens, cu, _, _ = _case(rng, [20], [9])
    whole = O.prefill_attention_np(q, kp, vp, tab, lens, cu, 0.3, "f32")
    first = O.prefill_attention_np(q[:4], kp, vp, tab, np.array([20 - 5], np.int32),
                                   np.array([0, 4]), 0.3, "f32")
    second = O.prefill_attention_np(q[4:], kp, vp, tab, lens, np.array([0, 5]), 0.3, "f32")
    assert np.abs(np.concatenate([first, second]) - whole).max() <= 1e-12


def test_chunk_longer_than_context_is_an_error():
    rng = np.random.default_rng(5)
    q, kp, vp, tab, lens, cu, _, _ = _case(rng, [3], [3])
    with pytest.raises(ValueError):
        O.prefill_attention_np(q, kp, vp, tab, np.array([2], np.int32), cu, 0.3, "f32")


MUTANTS = {
    "mask_off_by_one": ("<= pos[:, None]", "< pos[:, None] + 2"),
    "positions_from_zero": ("pos = ctx - n + np.arange(n)", "pos = np.arange(n)"),
    "no_mask": ("s = np.where(allowed, s, -np.inf)", "s = s"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_mutant_fails_a_pin(name):
    old, new = MUTANTS[name]
    src = inspect.getsource(O.prefill_attention_np)
    assert src.count(old) == 1
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    mutant = ns["prefill_attention_np"]
    orig = O.prefill_attention_np
    failed = 0
    try:
        O.prefill_attention_np = mutant
        for check in (test_one_token_chunks_are_decode, test_whole_prompt_chunk_is_causal_sdpa,
                      test_rows_ignore_keys_after_their_position,
                      test_splitting_a_chunk_changes_nothing):
            try:
                with np.errstate(all="ignore"):
                    check()
            except (AssertionError, ValueError, IndexError):
                failed += 1
    finally:
        O.prefill_attention_np = orig
    assert failed > 0
