"""Pins of the oracle's binary16 conversion and 4-bit group quantiser (CPU only).

Nothing here is checked against the oracle itself: the expected values are
hand-derived fixtures (tests/golden), closed forms, numpy's independent
float16 conversion, or invariants that hold for the definition
("FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 3,
Group-Wise 4-Bit Quantization).
"""
import json
import os

import numpy as np
import pytest

import oracle
import seeded_inputs as si


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _nibbles(codes_row):
    b = np.asarray(codes_row, dtype=np.uint8)
    out = np.empty(b.size * 2, dtype=np.int64)
    out[0::2] = b & 15
    out[1::2] = b >> 4
    return out


# ------------------------------------------------------------------ fp16 format ---------

def _np_half(x):
    with np.errstate(over="ignore"):
        return x.astype(np.float16).view(np.uint16)


def test_f16_decode_all_patterns_matches_numpy():
    h = np.arange(65536, dtype=np.uint16)
    ours = oracle.f16_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_f16_round_trip_all_patterns():
    h = np.arange(65536, dtype=np.uint16)
    finite = ~np.isnan(h.view(np.float16))
    back = oracle.f64_to_f16(oracle.f16_to_f64(h)).view(np.uint16)
    assert np.array_equal(back[finite], h[finite])


def test_f16_rounding_midpoints_ties_to_even():
    # all positive finite halves, their midpoints and points just off the midpoint
    h = np.arange(0, 0x7bff, dtype=np.uint16)          # 0 .. next-to-largest
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2                                  # exact in binary64
    got = oracle.f64_to_f16(mid).view(np.uint16)
    want = np.where(h % 2 == 0, h, h + 1).astype(np.uint16)  # even mantissa wins
    assert np.array_equal(got, want)
    eps = (hi - lo) * 1e-6
    assert np.array_equal(oracle.f64_to_f16(mid - eps).view(np.uint16), h)
    assert np.array_equal(oracle.f64_to_f16(mid + eps).view(np.uint16), h + 1)
    # negative side mirrors the positive side
    assert np.array_equal(oracle.f64_to_f16(-mid).view(np.uint16), want | 0x8000)


def test_f16_rounding_against_numpy_random():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 5, 200000),
                        rng.uniform(-70000, 70000, 20000)])
    assert np.array_equal(oracle.f64_to_f16(x).view(np.uint16), _np_half(x))


def test_f16_overflow_and_underflow_boundaries():
    f = lambda v: int(oracle.f64_to_f16(np.array([v]))[0].view(np.uint16))
    assert f(65504.0) == 0x7BFF
    assert f(65519.99) == 0x7BFF
    assert f(65520.0) == 0x7C00            # tie between 65504 (odd) and 2^16 (even) -> inf
    assert f(-65520.0) == 0xFC00
    assert f(2.0 ** -24) == 0x0001
    assert f(2.0 ** -25) == 0x0000         # tie between 0 and 2^-24 -> 0 (even)
    assert f(1.5 * 2.0 ** -25) == 0x0001
    assert f(-0.0) == 0x8000
    assert f(2.0 ** -14 - 2.0 ** -26) == 0x0400   # rounds up into the normal range


# ------------------------------------------------------------- hand-worked groups -------

def test_ramp_group_hand_worked(golden_dir):
    g = _load(golden_dir, "quant_ramp_group.json")
    x = np.arange(64, dtype=np.float16).reshape(1, 64)
    q = oracle.quantize(x)
    assert int(q.scales.view(np.uint16)[0, 0]) == g["scale_bits"]
    assert int(q.mins.view(np.uint16)[0, 0]) == g["min_bits"]
    want = np.repeat(np.arange(16), g["code_run_lengths"])
    assert np.array_equal(_nibbles(q.codes[0]), want)
    assert list(q.codes[0, :4]) == g["first_bytes"]
    y = oracle.dequantize(q).astype(np.float64)[0]
    assert np.array_equal(y, np.asarray(g["dequant_by_code"])[want])
    # round-trip bound: |x - deq| <= scale/2 (the fp16 rounding here is within it)
    assert np.max(np.abs(y - np.arange(64))) <= 4.19921875 / 2


def test_tie_group_half_even(golden_dir):
    g = _load(golden_dir, "quant_tie_group.json")
    x = np.array(g["input_head"] + [g["input_tail_value"]] * g["input_tail_count"], dtype=np.float16)
    q = oracle.quantize(x.reshape(1, 64))
    assert int(q.scales.view(np.uint16)[0, 0]) == g["scale_bits"]
    assert int(q.mins.view(np.uint16)[0, 0]) == g["min_bits"]
    c = _nibbles(q.codes[0])
    assert list(c[:8]) == g["codes_head"]
    assert np.all(c[8:] == g["code_tail"])


def test_signed_group_hand_worked(golden_dir):
    g = _load(golden_dir, "quant_signed_group.json")
    x = np.array(g["input_head"] + [g["input_tail_value"]] * g["input_tail_count"], dtype=np.float16)
    q = oracle.quantize(x.reshape(1, 64))
    assert int(q.scales.view(np.uint16)[0, 0]) == g["scale_bits"]
    assert int(q.mins.view(np.uint16)[0, 0]) == g["min_bits"]
    c = _nibbles(q.codes[0])
    assert list(c[:8]) == g["codes_head"]
    assert np.all(c[8:] == g["code_tail"])
    y = oracle.dequantize(q).astype(np.float64)[0]
    assert list(y[:8]) == g["dequant_head"]
    assert np.all(y[8:] == g["dequant_tail"])


# ----------------------------------------------------------------- special cases --------

@pytest.mark.parametrize("value", [0.0, -0.0, 0.5, -7.25, 65504.0, -65504.0, 2.0 ** -24])
def test_constant_group(value):
    x = np.full((1, 64), value, dtype=np.float16)
    q = oracle.quantize(x)
    assert np.all(q.codes == 0)
    assert int(q.scales.view(np.uint16)[0, 0]) == 0
    want_min = np.float16(value).view(np.uint16)
    if value == 0.0:
        want_min = np.uint16(0)                        # -0 is stored as +0
    assert q.mins.view(np.uint16)[0, 0] == want_min
    y = oracle.dequantize(q)
    assert np.array_equal(y.astype(np.float64), x.astype(np.float64))


def test_mixed_signed_zero_group_stores_plus_zero():
    x = np.where(np.arange(64) % 2 == 0, np.float16(-0.0), np.float16(0.0)).astype(np.float16)
    q = oracle.quantize(x.reshape(1, 64))
    assert int(q.mins.view(np.uint16)[0, 0]) == 0 and int(q.scales.view(np.uint16)[0, 0]) == 0
    assert np.all(q.codes == 0)


def test_scale_underflow_is_constant_group():
    # range 2^-24: (2^-24)/15 rounds to 0 in fp16 -> all codes 0, error <= range
    x = np.zeros((1, 64), dtype=np.float16)
    x[0, 5] = np.float16(2.0 ** -24)
    q = oracle.quantize(x)
    assert int(q.scales.view(np.uint16)[0, 0]) == 0 and np.all(q.codes == 0)
    assert np.max(np.abs(oracle.dequantize(q).astype(np.float64) - x.astype(np.float64))) <= 2.0 ** -24


def test_subnormal_scale_used_as_is():
    # range 2^-20: 2^-20/15 is a subnormal fp16 (nonzero) and is used as the scale
    x = np.zeros((1, 64), dtype=np.float16)
    x[0, 7] = np.float16(2.0 ** -20)
    q = oracle.quantize(x)
    s = float(q.scales.astype(np.float64)[0, 0])
    assert 0.0 < s < 2.0 ** -14
    c = _nibbles(q.codes[0])
    assert c[7] == 15 and np.all(np.delete(c, 7) == 0)


# ---------------------------------------------------------------- invariants -----------

def _check_round_trip(x2d):
    q = oracle.quantize(x2d)
    y = oracle.dequantize(q).astype(np.float64)
    x = x2d.astype(np.float64)
    G = x.reshape(-1, 64)
    Y = y.reshape(-1, 64)
    s = q.scales.astype(np.float64).reshape(-1, 1)
    mn = q.mins.astype(np.float64).reshape(-1, 1)
    codes = np.stack([q.codes.reshape(-1, 32) & 15, q.codes.reshape(-1, 32) >> 4], axis=-1).reshape(-1, 64)
    # stored min is the group minimum (exactly); constant groups are all code 0
    assert np.array_equal(mn[:, 0], G.min(axis=1) + 0.0)
    nz = s[:, 0] > 0
    assert np.all(codes[~nz] == 0)
    assert np.all(codes[nz].min(axis=1) == 0)
    # a normal fp16 scale is within 2^-11 of range/15, so the max element lands on code 15
    normal = s[:, 0] >= 2.0 ** -14
    assert np.all(codes[normal, :][np.arange(normal.sum()), G[normal].argmax(axis=1)] == 15)
    exact = mn + codes * s
    err = np.abs(G - exact)
    # |x - (min + code*scale)| <= scale/2 up to the fp32 rounding of the step ...
    assert np.all(err[normal] <= (s / 2 * (1 + 2.0 ** -16))[normal])
    # ... and, with a subnormal scale (spacing 2^-24), up to 15 half-spacings more
    assert np.all(err <= s / 2 * (1 + 2.0 ** -16) + 15 * 2.0 ** -25)
    # the stored fp16 value is that exact value rounded once to nearest
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(Y - exact) <= ulp / 2)
    # min(group) is reproduced exactly by code 0
    assert np.all(Y[np.arange(len(G)), G.argmin(axis=1)] == G.min(axis=1))
    return int((~normal & nz).sum())


def test_round_trip_bound_sweep_recipe():
    x = si.sweep_tensor(seed=0, numel=1 << 18, row=4096)
    _check_round_trip(x)


def test_round_trip_bound_wide_ranges():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((512, 64)) * 10.0 ** rng.integers(-6, 4, (512, 1))).astype(np.float16)
    assert _check_round_trip(x) > 0          # the subnormal-scale branch is exercised


def test_group_boundaries_and_dims():
    # quantising along a non-last dim equals quantising the transposed tensor along the last dim
    x = si.normal_f16(3, 99, (6, 128, 5), 1.0)
    a = oracle.quantize(x, dim=1)
    b = oracle.quantize(np.ascontiguousarray(np.transpose(x, (0, 2, 1))), dim=-1)
    assert np.array_equal(a.codes, np.transpose(b.codes, (0, 2, 1)))
    assert np.array_equal(a.mins.view(np.uint16), np.transpose(b.mins.view(np.uint16), (0, 2, 1)))
    y = oracle.dequantize(a)
    assert np.array_equal(y.view(np.uint16), np.transpose(oracle.dequantize(b).view(np.uint16), (0, 2, 1)))
    # each group of 64 is independent: quantising one group alone gives the same bytes
    x2 = si.normal_f16(4, 99, (3, 256), 1.0)
    full = oracle.quantize(x2)
    for r in range(3):
        for g in range(4):
            one = oracle.quantize(x2[r:r + 1, 64 * g:64 * (g + 1)])
            assert np.array_equal(one.codes[0], full.codes[r, 32 * g:32 * (g + 1)])
            assert one.scales.view(np.uint16)[0, 0] == full.scales.view(np.uint16)[r, g]


def test_nibble_order_low_is_even():
    x = np.zeros((1, 64), dtype=np.float16)
    x[0, 0] = 15.0   # element 0 -> low nibble of byte 0
    q = oracle.quantize(x)
    assert q.codes[0, 0] == 0x0F
    x = np.zeros((1, 64), dtype=np.float16)
    x[0, 1] = 15.0   # element 1 -> high nibble of byte 0
    q = oracle.quantize(x)
    assert q.codes[0, 0] == 0xF0


def test_rejects_non_multiple_of_64():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 96), dtype=np.float16))


# ------------------------------------------------------------------ groups of 128 -----------
# ("FlexGen Guide", section 3: groups of 64 or 128 elements)

def test_ramp_group128_hand_worked(golden_dir):
    g = _load(golden_dir, "quant_ramp_group128.json")
    x = (np.arange(128) / 2).astype(np.float16).reshape(1, 128)
    q = oracle.quantize(x, group=128)
    assert q.mins.shape == (1, 1) and q.codes.shape == (1, 64)
    assert int(q.scales.view(np.uint16)[0, 0]) == g["scale_bits"]
    assert int(q.mins.view(np.uint16)[0, 0]) == g["min_bits"]
    want = np.repeat(np.arange(16), g["code_run_lengths"])
    assert np.array_equal(_nibbles(q.codes[0]), want)
    assert list(q.codes[0, :4]) == g["first_bytes"]
    y = oracle.dequantize(q).astype(np.float64)[0]
    assert np.array_equal(y, np.asarray(g["dequant_by_code"])[want])
    assert np.max(np.abs(y - np.arange(128) / 2)) <= 4.234375 / 2 + 2.0 ** -6


def test_group128_of_two_halves_with_the_same_range_equals_group64():
    # when each 64-half of a 128-group holds the group's min and max, both groupings see the
    # same (min, max), so the scale and every code agree; a mistake in the 128-grouping
    # (a wrong stride, half, or metadata slot) breaks the equality
    rng = np.random.default_rng(5)
    x = rng.uniform(-3, 5, (4, 512)).astype(np.float16)
    for r in range(4):
        for blk in range(4):
            lo, hi = np.float16(-3.0 - r), np.float16(5.0 + blk)
            x[r, blk * 128 + 3], x[r, blk * 128 + 64 + 7] = lo, lo
            x[r, blk * 128 + 50], x[r, blk * 128 + 64 + 60] = hi, hi
    a = oracle.quantize(x, group=128)
    b = oracle.quantize(x, group=64)
    assert np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scales.view(np.uint16), b.scales.view(np.uint16)[:, ::2])
    assert np.array_equal(a.scales.view(np.uint16), b.scales.view(np.uint16)[:, 1::2])
    assert np.array_equal(a.mins.view(np.uint16), b.mins.view(np.uint16)[:, ::2])
    assert np.array_equal(oracle.dequantize(a).view(np.uint16), oracle.dequantize(b).view(np.uint16))


def test_group128_blocks_land_in_their_metadata_slots():
    # block j of 128 holds values in [j, j + 0.5]: min of slot j is j, and a 128-group never
    # mixes two blocks (with groups of 64 the same data gives two equal slots per block)
    x = np.empty((2, 640), np.float16)
    for j in range(5):
        x[:, 128 * j:128 * (j + 1)] = (j + np.linspace(0.0, 0.5, 128)).astype(np.float16)
    q = oracle.quantize(x, group=128)
    assert q.mins.shape == (2, 5)
    assert np.array_equal(q.mins.astype(np.float64), np.tile(np.arange(5.0), (2, 1)))
    # dims: along a non-last dim equals the transposed tensor along the last dim
    x3 = si.normal_f16(6, 99, (3, 256, 5), 1.0)
    a = oracle.quantize(x3, dim=1, group=128)
    b = oracle.quantize(np.ascontiguousarray(np.transpose(x3, (0, 2, 1))), dim=-1, group=128)
    assert np.array_equal(a.codes, np.transpose(b.codes, (0, 2, 1)))
    assert np.array_equal(a.scales.view(np.uint16), np.transpose(b.scales.view(np.uint16), (0, 2, 1)))


@pytest.mark.parametrize("value", [0.0, -2.5, 1000.0])
def test_constant_group128(value):
    q = oracle.quantize(np.full((1, 128), value, np.float16), group=128)
    assert np.all(q.codes == 0)
    assert q.scales.view(np.uint16)[0, 0] == 0
    assert np.all(oracle.dequantize(q) == np.float16(value))


def test_group128_round_trip_bound():
    x = si.sweep_tensor(seed=2, numel=1 << 16, row=4096)
    q = oracle.quantize(x, group=128)
    y = oracle.dequantize(q).astype(np.float64).reshape(-1, 128)
    G = x.astype(np.float64).reshape(-1, 128)
    s = q.scales.astype(np.float64).reshape(-1, 1)
    assert np.array_equal(q.mins.astype(np.float64).reshape(-1), G.min(axis=1) + 0.0)
    # |x - deq| <= scale/2 (fp32 step rounding) + half an fp16 spacing of the result
    ulp = np.spacing(np.abs(y).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(G - y) <= s / 2 * (1 + 2.0 ** -16) + ulp / 2)


def test_group128_linear_indexes_its_groups():
    # y = x deq(W)^T with W in groups of 128 along K, against numpy on the dequantised weights
    x = si.normal_f16(7, 1, (5, 384), 1.0)
    w = si.normal_f16(7, 2, (128, 384), 0.05)
    q = oracle.quantize(w, dim=1, group=128)
    ref = x.astype(np.float64) @ oracle.dequantize(q).astype(np.float64).T
    assert np.allclose(oracle.linear(x, q), ref, rtol=0, atol=1e-5 * np.max(np.abs(ref)))


def test_group_sizes_rejected():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 192), dtype=np.float16), group=128)
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 192), dtype=np.float16), group=96)


# ------------------------------------------------------------------ 8-bit codes -----------
# The same min-max scheme with 255 steps, one code per byte (INT8 beside INT4 among the
# post-training formats of the "Optimizing LLM for low memory usage" page).

def _b8_span_group(group, offset=0.0):
    # integers spanning exactly [0, 255] (both ends present), so that range/255 = 1 exactly
    x = np.concatenate([[0.0, 255.0], np.round(np.linspace(1, 254, group - 2))]) + offset
    return x.astype(np.float16).reshape(1, group)


@pytest.mark.parametrize("group,offset", [(64, 0.0), (64, 1000.0), (64, -700.0), (128, 0.0), (128, 512.0)])
def test_b8_integer_span_is_exact(group, offset):
    # scale = fp16(255 / 255) = 1, inverse 1: every code is the value minus the minimum and
    # the round trip is exact (closed form; all values are fp16 integers)
    x = _b8_span_group(group, offset)
    q = oracle.quantize(x, group=group, bits=8)
    assert q.codes.shape == (1, group)                         # one code per byte, in order
    assert float(q.scales[0, 0]) == 1.0 and float(q.mins[0, 0]) == offset
    assert np.array_equal(q.codes[0].astype(np.float64), x[0].astype(np.float64) - offset)
    assert np.array_equal(oracle.dequantize(q).view(np.uint16), x.view(np.uint16))


def test_b8_ties_round_half_even():
    # span [0, 255] -> step 1; k + 0.5 rounds to the even neighbour
    x = np.full((1, 64), 100.0)
    x[0, :2] = [0.0, 255.0]
    x[0, 2:8] = [0.5, 1.5, 2.5, 3.5, 128.5, 254.5]
    q = oracle.quantize(x.astype(np.float16), bits=8)
    assert list(q.codes[0, :8]) == [0, 255, 0, 2, 2, 4, 128, 254]
    assert np.all(q.codes[0, 8:] == 100)


@pytest.mark.parametrize("value", [0.0, -3.25, 1000.0])
def test_b8_constant_group(value):
    x = np.full((1, 64), value, dtype=np.float16)
    q = oracle.quantize(x, bits=8)
    assert np.all(q.codes == 0) and float(q.scales[0, 0]) == 0.0
    assert np.array_equal(oracle.dequantize(q).view(np.uint16), (x + np.float16(0)).view(np.uint16))


def _check_b8_round_trip(x2d, group=64):
    q = oracle.quantize(x2d, group=group, bits=8)
    y = oracle.dequantize(q).astype(np.float64).reshape(-1, group)
    G = x2d.astype(np.float64).reshape(-1, group)
    s = q.scales.astype(np.float64).reshape(-1, 1)
    mn = q.mins.astype(np.float64).reshape(-1, 1)
    codes = q.codes.reshape(-1, group).astype(np.float64)
    assert np.array_equal(mn[:, 0], G.min(axis=1) + 0.0)
    nz = s[:, 0] > 0
    assert np.all(codes[~nz] == 0) and np.all(codes[nz].min(axis=1) == 0)
    # codes follow the values: sorting a group's values sorts its codes
    order = np.argsort(G, axis=1, kind="stable")
    assert np.all(np.diff(np.take_along_axis(codes, order, axis=1), axis=1) >= 0)
    # a normal fp16 scale is within 2^-11 of range/255, so the group maximum lands on 255
    normal = s[:, 0] >= 2.0 ** -14
    assert np.all(codes[normal, :][np.arange(normal.sum()), G[normal].argmax(axis=1)] == 255)
    exact = mn + codes * s
    assert np.all(np.abs(G - exact)[normal] <= (s / 2 * (1 + 2.0 ** -16))[normal])
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(y - exact) <= ulp / 2)
    assert np.all(y[np.arange(len(G)), G.argmin(axis=1)] == G.min(axis=1))
    return int(normal.sum())


def test_b8_round_trip_bound_sweep_recipe():
    x = si.sweep_tensor(seed=5, numel=1 << 16, row=4096)
    assert _check_b8_round_trip(x) > 0
    _check_b8_round_trip(x, group=128)


def test_b8_non_last_dim_equals_transposed():
    x = si.normal_f16(6, 99, (3, 128, 5), 1.0)
    a = oracle.quantize(x, dim=1, bits=8)
    b = oracle.quantize(np.ascontiguousarray(np.transpose(x, (0, 2, 1))), dim=-1, bits=8)
    assert a.codes.shape == (3, 128, 5)
    assert np.array_equal(a.codes, np.transpose(b.codes, (0, 2, 1)))
    assert np.array_equal(oracle.dequantize(a).view(np.uint16),
                          np.transpose(oracle.dequantize(b).view(np.uint16), (0, 2, 1)))


def test_b8_codes_are_the_4bit_codes_refined():
    # with the same range, an 8-bit step is a 4-bit step / 17 (255 = 15 * 17): the integer span
    # [0, 255] quantised at 4 bits has step 17, so the 4-bit code is the 8-bit code / 17 rounded
    x = _b8_span_group(64)
    c8 = oracle.quantize(x, bits=8).codes[0].astype(np.int64)
    c4 = _nibbles(oracle.quantize(x).codes[0])
    assert float(oracle.quantize(x).scales[0, 0]) == 17.0
    assert np.array_equal(c4, np.round(c8 / 17.0).astype(np.int64))


def test_bits_rejected():
    for bits in (2, 3, 16):
        with pytest.raises(ValueError):
            oracle.quantize(np.zeros((1, 64), dtype=np.float16), bits=bits)
