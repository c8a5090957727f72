"""Number formats the NF4 codec rounds through, each written out from its definition.

Test infrastructure (see the package docstring): only tests, smoke and the CPU baseline use it.

* fp32 single operations.  For fp32 operands a, b the exact sum, difference and product are
  representable in fp64 or, for the quotient, fp64 carries more than 2*24+2 significant bits, so
  computing in fp64 and rounding once to fp32 gives the correctly rounded fp32 result (the double
  rounding is innocuous).  These helpers are that definition.
* fp32 fused multiply-add RN32(a*b + c).  a*b is exact in fp64; the sum is formed in fp64 with
  round-to-odd and then rounded to nearest fp32.  Boldo & Melquiond ("Emulation of FMA and correctly
  rounded sums: proved algorithms using rounding to odd", IEEE Trans. Computers 2008) prove that
  round-to-odd at 53 bits followed by round-to-nearest at 24 bits equals one round-to-nearest, since
  53 >= 24 + 2.  Round-to-odd is built from the fp64 sum and its exact error (Knuth's TwoSum).
* bf16: the upper 16 bits of fp32, rounded to nearest with ties to even.
* E4M3 (OCP 8-bit floating point, "fn" variant): 1 sign, 4 exponent bits with bias 7, 3 mantissa
  bits; no infinities; S.1111.111 is NaN; largest finite magnitude 448; subnormal step 2^-9.
  Encoding rounds to nearest, ties to the even code, and saturates to +-448 ("satfinite").
"""
from __future__ import annotations

import numpy as np

F32, F64 = np.float32, np.float64
E4M3_MAX = 448.0


def _f64(x):
    return np.asarray(x, dtype=F32).astype(F64)


def rn32_add(a, b):
    return (_f64(a) + _f64(b)).astype(F32)


def rn32_sub(a, b):
    return (_f64(a) - _f64(b)).astype(F32)


def rn32_mul(a, b):
    return (_f64(a) * _f64(b)).astype(F32)


def rn32_div(a, b):
    with np.errstate(divide="ignore", invalid="ignore"):
        return (_f64(a) / _f64(b)).astype(F32)


def fma32(a, b, c):
    """RN32(a*b + c) with a single rounding, for fp32 a, b, c (finite, result in range)."""
    p = _f64(a) * _f64(b)                  # exact: two 24-bit significands fit in 53 bits
    c64 = _f64(c)
    s = p + c64                            # RN64 of the exact sum
    bb = s - p                             # TwoSum: err = (p + c) - s exactly
    err = (p - (s - bb)) + (c64 - bb)
    bits = np.asarray(s, dtype=F64).view(np.uint64)
    even = (bits & np.uint64(1)) == 0
    toward = np.where(err > 0, np.inf, -np.inf)
    s_odd = np.where((err != 0) & even, np.nextafter(s, toward), s)   # round-to-odd of the sum
    return np.asarray(s_odd, dtype=F64).astype(F32)


def bf16_rne_bits(x):
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    x = np.asarray(x, dtype=F32)
    if not np.all(np.isfinite(x)):
        raise ValueError("bf16_rne_bits: non-finite input")
    u = x.view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(F32)


def e4m3_decode(code):
    """E4M3 byte -> its exact value (fp64; NaN for S.1111.111)."""
    code = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = code >> 7
    e = (code >> 3) & 0xF
    m = code & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


# positive finite magnitudes in code order 0x00..0x7E; E4M3 codes increase with magnitude
_MAG = e4m3_decode(np.arange(127, dtype=np.uint8))
assert np.all(np.diff(_MAG) > 0)


def e4m3_encode(t):
    """fp32 -> E4M3 byte: round to nearest, ties to the even code, saturate to +-448."""
    t = np.asarray(t, dtype=F32)
    if not np.all(np.isfinite(t)):
        raise ValueError("e4m3_encode: non-finite input")
    a = np.abs(t.astype(F64))
    lo = np.clip(np.searchsorted(_MAG, a, side="right") - 1, 0, 126)   # largest code with |value| <= a
    hi = np.minimum(lo + 1, 126)
    d_lo = a - _MAG[lo]                     # exact: both are short dyadic numbers of similar size
    d_hi = _MAG[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= E4M3_MAX, 126, pick)                          # satfinite
    sign = np.signbit(t).astype(np.int64)
    return (pick | (sign << 7)).astype(np.uint8)
