"""Pins of the oracle's number formats against library casts and against the
formats' definitions (FP8 E4M3 for group scales: m.163.com article on Quant
VideoGen, section 五; bf16 storage of K/V)."""
from fractions import Fraction

import numpy as np
import pytest
import torch


def test_e4m3_decode_all_codes_match_torch(ora):
    codes = np.arange(256, dtype=np.uint8)
    ours = ora.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan_codes = (codes & 0x7F) == 0x7F
    assert np.all(np.isnan(ours[nan_codes]))
    np.testing.assert_array_equal(ours[~nan_codes], lib[~nan_codes])


def test_e4m3_decode_definition_landmarks(ora):
    # largest finite 448 = 1.75 * 2^8; smallest subnormal 2^-9; smallest normal 2^-6
    assert ora.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert ora.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert ora.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert ora.e4m3_decode(np.array([0xB0]))[0] == -0.5
    assert ora.e4m3_decode(np.array([0x38]))[0] == 1.0


def test_e4m3_encode_roundtrip_every_finite_code(ora):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = ora.e4m3_decode(codes)
    np.testing.assert_array_equal(ora.e4m3_encode(vals), codes)


def test_e4m3_encode_random_matches_torch(ora):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
        rng.uniform(-447.99, 447.99, 5000),
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 5000),
    ]).astype(np.float32)
    x = x[np.abs(x) < 448]
    ours = ora.e4m3_encode(x)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, lib)


def test_e4m3_encode_ties_to_even(ora):
    codes = np.arange(0, 0x7E, dtype=np.uint8)       # positive finite codes
    v = ora.e4m3_decode(codes).astype(np.float64)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)  # exact in fp32
    got = ora.e4m3_encode(mids).astype(int)
    lo = codes[:-1].astype(int)
    expect = np.where(lo % 2 == 0, lo, lo + 1)        # even mantissa wins
    np.testing.assert_array_equal(got, expect)
    np.testing.assert_array_equal(ora.e4m3_encode(-mids).astype(int), expect | 0x80)


def test_e4m3_encode_saturates_and_nan(ora):
    x = np.array([448, 460, 464, 500, 1e4, 3e38, np.inf, -448, -1000, -np.inf], np.float32)
    got = ora.e4m3_encode(x)
    np.testing.assert_array_equal(got, [0x7E] * 7 + [0xFE] * 3)
    assert ora.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_bf16_round_from_f32_matches_torch(ora):
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(50000) * 10.0 ** rng.uniform(-40, 38, 50000),
        rng.standard_normal(20000),
    ]).astype(np.float32)
    x = x[np.isfinite(x)]
    ours = ora.bf16_round(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, lib)


def _bf16_value(b):
    return Fraction(float(ora_bf16_to_f32(np.array([b], np.uint16))[0]))


def ora_bf16_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def test_bf16_round_from_f64_is_single_nearest_even(ora):
    """Brute force from the definition: the result is the nearer of the two
    bf16 neighbours of x in exact rational arithmetic, ties to the even
    pattern (no intermediate rounding to fp32)."""
    rng = np.random.default_rng(3)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000))
    # doubles that sit just beside a bf16 midpoint, where fp64 -> fp32 -> bf16
    # double rounding would go wrong
    for m in (1.00390625, 1.01171875, 3.0 + 2 ** -7):
        xs += [np.nextafter(m, 2), np.nextafter(m, 0), m]
    got = ora.bf16_round(np.array(xs))
    for x, g in zip(xs, got):
        ax = abs(x)
        t = np.float32(ax).view(np.uint32) >> 16           # candidate near |x|
        cands = [int(c) for c in (t - 1, t, t + 1) if 0 <= c < 0x7F80]
        fx = Fraction(ax)
        best = min(cands, key=lambda c: (abs(_bf16_value(c) - fx), c & 1))
        exp = best | (0x8000 if x < 0 else 0)
        assert int(g) == exp, (x, hex(int(g)), hex(exp))


def test_bf16_round_overflow_and_subnormal(ora):
    got = ora.bf16_round(np.array([3.4e38, -3.4e38, 2.0 ** -133, 2.0 ** -134, 1.5 * 2.0 ** -134, 0.0, -0.0]))
    np.testing.assert_array_equal(got, [0x7F80, 0xFF80, 0x0001, 0x0000, 0x0001, 0x0000, 0x8000])
