"""Pins for the oracle's number formats, against exact rational arithmetic and independent libraries."""
from fractions import Fraction

import numpy as np
import torch

import oracle as O


def rn32_exact(v: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32 (ties to even), normal range only."""
    if v == 0:
        return np.float32(0.0)
    s = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    assert -126 <= e <= 127
    m = round(a / Fraction(2) ** (e - 23))          # round-half-even on an exact rational
    return np.float32(s * float(Fraction(m) * Fraction(2) ** (e - 23)))


def _rand_f32(rng, n, lo=-20, hi=20):
    mant = rng.uniform(1.0, 2.0, n)
    exp = rng.integers(lo, hi, n)
    sign = rng.choice([-1.0, 1.0], n)
    return (sign * mant * np.exp2(exp)).astype(np.float32)


def test_fp32_single_ops_match_exact_rounding():
    rng = np.random.default_rng(1)
    a, b = _rand_f32(rng, 400), _rand_f32(rng, 400)
    for i in range(a.size):
        fa, fb = Fraction(float(a[i])), Fraction(float(b[i]))
        assert O.rn32_sub(a[i], b[i]) == rn32_exact(fa - fb)
        assert O.rn32_mul(a[i], b[i]) == rn32_exact(fa * fb)
        assert O.rn32_div(a[i], b[i]) == rn32_exact(fa / fb)


def test_fma32_single_rounding_random_and_adversarial():
    rng = np.random.default_rng(2)
    a, b, c = _rand_f32(rng, 600, -8, 8), _rand_f32(rng, 600, -8, 8), _rand_f32(rng, 600, -30, 8)
    # adversarial: c nearly cancels a*b, and products landing half an ulp from an fp32 value
    a2 = _rand_f32(rng, 300, -4, 4)
    b2 = _rand_f32(rng, 300, -4, 4)
    c2 = (-(a2.astype(np.float64) * b2)).astype(np.float32)
    a = np.concatenate([a, a2, np.float32([1.0 + 2 ** -23, 1.0, 3.0])])
    b = np.concatenate([b, b2, np.float32([1.0 + 2 ** -23, 2 ** -24, 2 ** -24 + 2 ** -47])])
    c = np.concatenate([c, c2, np.float32([-1.0, 1.0, 1.0])])
    got = O.fma32(a, b, c)
    for i in range(a.size):
        exact = Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i]))
        want = rn32_exact(exact) if exact == 0 or abs(exact) >= Fraction(2) ** -126 else None
        if want is not None:
            assert got[i] == want, (a[i], b[i], c[i], got[i], want)
    # the fused result differs from two separate roundings on a constructed case
    x = np.float32(1.0 + 2 ** -12)
    fused = O.fma32(x, x, np.float32(-1.0))
    assert fused == np.float32(2 ** -11 + 2 ** -24)
    assert O.rn32_add(O.rn32_mul(x, x), np.float32(-1.0)) == np.float32(2 ** -11)


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([_rand_f32(rng, 20000, -130, 127),
                        np.float32([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.3895314e38, 1e-45])])
    # values exactly halfway between two bf16 numbers (ties go to the even pattern)
    halves = ((rng.integers(0, 1 << 15, 2000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, halves[np.isfinite(halves)]])
    ours = O.bf16_rne_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(O.bf16_bits_to_f32(ours).view(np.uint32) & 0xFFFF, np.zeros_like(ours, np.uint32))


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    assert np.array_equal(ours[finite], ref[finite])
    assert O.e4m3_decode(np.uint8(0x7E)) == 448.0 and O.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9
    assert np.isnan(O.e4m3_decode(np.uint8(0x7F))) and np.isnan(O.e4m3_decode(np.uint8(0xFF)))


def test_e4m3_encode_round_trip_ties_and_saturation():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32)
    back = O.e4m3_encode(vals)
    assert np.array_equal(back, codes)                      # exhaustive round trip (NaN excepted)
    mags = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)  # exact midpoints, representable in fp32
    assert np.array_equal(mids.astype(np.float64), (mags[:-1] + mags[1:]) / 2)
    enc = O.e4m3_encode(mids)
    lo = np.arange(126)
    assert np.array_equal(enc, np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8))   # ties to even
    assert np.array_equal(O.e4m3_encode(-mids), enc | 0x80)
    sat = np.float32([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38])
    assert np.all(O.e4m3_encode(sat) == 0x7E) and np.all(O.e4m3_encode(-sat) == 0xFE)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.uniform(-448, 448, 50000), rng.normal(0, 1, 50000),
                        rng.normal(0, 1e-2, 20000), rng.normal(0, 1e-3, 20000)]).astype(np.float32)
    ours = O.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
