"""Pins of the oracle's FP8 (E4M3) cache: the code format, the rounding of
the cache write, and attention over a dequantised cache.

The facts they rest on, none of them the oracle itself:

* torch's float8_e4m3fn type (a library implementation of the OCP E4M3
  format: 4 exponent bits of bias 7, 3 mantissa bits, subnormals, NaN at
  S.1111.111, no infinities) decodes every byte to the same value, and
  rounds every binary32 value inside the format's range to the same code;
* closed forms of the format: 448 is the largest finite value, 2^-9 the
  smallest subnormal, 2^-6 the smallest normal, 1.0 is 0x38;
* round to nearest puts a value halfway between two codes on the even one;
  saturation clamps finite overflow (and infinities) to +-448;
* a code has at most 4 significant bits, so with a power-of-two scale every
  dequantised value is exact in bf16, and attention over an E4M3 cache must
  then equal the (independent, C) bf16 oracle over those bf16 values;
* rounding to 3 mantissa bits is off by at most 2^-4 of the value in the
  normal range and by at most 2^-10 times the scale in the subnormal one.
"""
import inspect

import numpy as np
import pytest
import torch

from oracle import oracle as O
import pins


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_encode(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    assert np.array_equal(O.e4m3_to_f64(codes), _torch_decode(codes), equal_nan=True)


def test_decode_closed_forms():
    v = O.e4m3_to_f64(np.array([0x7E, 0x01, 0x08, 0x38, 0xC0, 0x00, 0x80, 0x7F, 0xFF, 0x07],
                               dtype=np.uint8))
    assert v[0] == 448.0 and v[1] == 2.0 ** -9 and v[2] == 2.0 ** -6 and v[3] == 1.0
    assert v[4] == -2.0 and v[5] == 0.0 and v[6] == 0.0 and np.signbit(v[6])
    assert np.isnan(v[7]) and np.isnan(v[8]) and v[9] == 7 * 2.0 ** -9


def test_encode_matches_torch_inside_the_range():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(200_000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) < 460].astype(np.float32)
    assert np.array_equal(O.f32_to_e4m3(x), _torch_encode(x))


def test_encode_ties_go_to_the_even_code():
    grid = O.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (grid[:-1] + grid[1:]) / 2)   # exact
    k = np.arange(0x7E)
    want = np.where(k % 2 == 0, k, k + 1).astype(np.uint8)
    assert np.array_equal(O.f32_to_e4m3(mids), want)
    assert np.array_equal(O.f32_to_e4m3(-mids), want | 0x80)


def test_encode_saturates_and_keeps_nan():
    x = np.array([448.0, 449.0, 470.0, 1e30, np.inf, -500.0, -np.inf, np.nan, -0.0],
                 dtype=np.float32)
    got = O.f32_to_e4m3(x)
    assert got.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80]


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_to_f64(codes).astype(np.float32)
    assert np.array_equal(O.f32_to_e4m3(vals), codes)


@pytest.mark.parametrize("scale", [1.0, 1.0 / 56.0, 0.37, 3.0])
def test_quantisation_error_bound(scale):
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(100_000) * 60 * scale).astype(np.float32)
    x = x[np.abs(x) <= 440 * scale]
    back = O.dequantize_e4m3(O.quantize_e4m3(x, scale), scale)
    err = np.abs(back - x.astype(np.float64))
    # half a unit in the last place of a 3-bit mantissa, plus the binary32
    # rounding of x / scale, in each range
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scale) * (1 + 2.0 ** -20)
    assert (err <= bound).all()


def _fp8_case(rng, lens, hq, hkv, d, bs, k_scale, v_scale):
    """Random finite codes, laid out in a paged pool with NaN codes in every
    slot no sequence owns; the same values as bf16 for the C oracle."""
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    kc = [rng.choice(finite, size=(n, hkv, d)) for n in lens]
    vc = [rng.choice(finite, size=(n, hkv, d)) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + 3
    perm = rng.permutation(nb)
    k_pool = np.full((nb, bs, hkv, d), 0x7F, np.uint8)
    v_pool = np.full((nb, bs, hkv, d), 0x7F, np.uint8)
    tables = np.full((len(lens), max(-(-n // bs) for n in lens)), -1, np.int32)
    pos = 0
    for b, n in enumerate(lens):
        for j in range(-(-n // bs)):
            tables[b, j] = perm[pos]
            rows = slice(j * bs, min((j + 1) * bs, n))
            k_pool[perm[pos], :rows.stop - rows.start] = kc[b][rows]
            v_pool[perm[pos], :rows.stop - rows.start] = vc[b][rows]
            pos += 1
    q = pins._to_elems(rng.standard_normal((len(lens), hq, d)), "bf16")

    def as_bf16(pool, s):
        vals = O.e4m3_to_f64(pool) * s
        return pins._to_elems(vals, "bf16")
    return q, k_pool, v_pool, tables, np.asarray(lens, np.int32), as_bf16(k_pool, k_scale), \
        as_bf16(v_pool, v_scale)


@pytest.mark.parametrize("shape", [(8, 2, 64, 4), (16, 4, 128, 16), (4, 4, 256, 32)])
def test_fp8_attention_equals_the_bf16_oracle_on_exactly_representable_values(shape):
    hq, hkv, d, bs = shape
    rng = np.random.default_rng(hq * 1000 + d)
    k_scale, v_scale = 2.0 ** -3, 2.0 ** 2      # different, so a swap shows
    lens = [1, 7, 33, 70]
    q, kp, vp, tables, cl, kp16, vp16 = _fp8_case(rng, lens, hq, hkv, d, bs, k_scale, v_scale)
    # the bf16 pools hold exactly the dequantised values (NaN where the code is NaN)
    assert np.array_equal(pins._from_elems(kp16, "bf16"), O.dequantize_e4m3(kp, k_scale),
                          equal_nan=True)
    scale = d ** -0.5
    ref = O.paged_attention(q, kp16, vp16, tables, cl, scale, "bf16")
    got = O.paged_attention_fp8_np(q, kp, vp, tables, cl, scale, k_scale, v_scale)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_fp8_attention_of_one_token_is_its_scaled_v_row():
    rng = np.random.default_rng(3)
    q, kp, vp, tables, cl, _, _ = _fp8_case(rng, [1, 1], 8, 2, 64, 4, 0.3, 0.07)
    got = O.paged_attention_fp8_np(q, kp, vp, tables, cl, 0.125, 0.3, 0.07)
    for b in range(2):
        v = O.dequantize_e4m3(vp[tables[b, 0], 0], 0.07)        # [Hkv, d]
        assert np.array_equal(got[b], np.repeat(v, 4, axis=0))


def test_fp8_cache_write_places_codes_and_leaves_the_rest():
    rng = np.random.default_rng(4)
    T, hkv, d, nb, bs = 5, 2, 64, 6, 4
    key = pins._to_elems(rng.standard_normal((T, hkv, d)) * 3, "bf16")
    val = pins._to_elems(rng.standard_normal((T, hkv, d)) * 3, "bf16")
    k_pool = rng.integers(0, 256, size=(nb, bs, hkv, d), dtype=np.uint8)
    v_pool = rng.integers(0, 256, size=(nb, bs, hkv, d), dtype=np.uint8)
    slots = np.array([3, -1, 22, 0, 9], np.int64)
    k_scale, v_scale = 1.0 / 56.0, 0.02
    ko, vo = O.reshape_and_cache_fp8_np(key, val, k_pool, v_pool, slots, k_scale, v_scale)
    touched = np.zeros((nb, bs), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        touched[s // bs, s % bs] = True
        for src, out, sc in ((key, ko, k_scale), (val, vo, v_scale)):
            x = pins._from_elems(src[t], "bf16").astype(np.float32) / np.float32(sc)
            want = np.where(np.abs(x) < 448, _torch_encode(x),       # torch: inside the range
                            np.where(x > 0, 0x7E, 0xFE))            # saturated to +-448
            assert np.array_equal(out[s // bs, s % bs], want)
    assert np.array_equal(ko[~touched], k_pool[~touched])
    assert np.array_equal(vo[~touched], v_pool[~touched])
    with pytest.raises(ValueError):
        O.reshape_and_cache_fp8_np(key[:1], val[:1], k_pool, v_pool, np.array([nb * bs]),
                                   k_scale, v_scale)


FP8_MUTANTS = {
    "exponent_bias_8": (O.e4m3_to_f64, "np.exp2(e.astype(np.float64) - 7.0)",
                        "np.exp2(e.astype(np.float64) - 8.0)"),
    "subnormal_step_2^-10": (O.e4m3_to_f64, "m * 2.0 ** -9", "m * 2.0 ** -10"),
    "mantissa_over_16": (O.e4m3_to_f64, "(1.0 + m / 8.0)", "(1.0 + m / 16.0)"),
    "scales_swapped": (O.paged_attention_fp8_np, "dequantize_e4m3(v_pool, v_scale)",
                       "dequantize_e4m3(v_pool, k_scale)"),
    "ties_away_from_zero": (O.f32_to_e4m3, "tie_pick = np.where(lo % 2 == 0, lo, hi)",
                            "tie_pick = hi"),
}


def _run_fp8_pins():
    failed = []
    for test in (test_decode_matches_torch_for_every_code, test_decode_closed_forms,
                 test_encode_ties_go_to_the_even_code, test_every_finite_code_round_trips,
                 lambda: test_fp8_attention_equals_the_bf16_oracle_on_exactly_representable_values(
                     (8, 2, 64, 4))):
        try:
            with np.errstate(all="ignore"):
                test()
        except (AssertionError, ValueError, IndexError):
            failed.append(test)
    return failed


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_mutant_fails_a_pin(name, monkeypatch):
    fn, old, new = FP8_MUTANTS[name]
    src = inspect.getsource(fn)
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(O, fn.__name__, ns[fn.__name__])
    assert _run_fp8_pins(), f"mutant {name} passed every pin"


def test_unmutated_fp8_oracle_passes_the_mutant_pins():
    assert _run_fp8_pins() == []
