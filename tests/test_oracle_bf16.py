"""Pins of the oracle's bf16 conversions against the format's definition (CPU only).

bf16 is 1 sign bit, 8 exponent bits (bias 127) and 7 mantissa bits, with
subnormals at exponent 0 and inf / NaN at exponent 255.  Conversions to it round
to the nearest value, ties to the even mantissa, and overflow to inf from the
midpoint between the largest finite value and 2^128 up.  The oracle rounds fp64
results in two steps, fp64 -> fp32 -> bf16, each to nearest (reading R11: the
residual and the layer outputs); a worked value separates that from one rounding.
"""
import math

import numpy as np
import pytest

from oracle import svdq_oracle as O


def _bf16_definition(bits: int) -> float:
    """The value of a bf16 bit pattern, from the format's fields."""
    sign = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    f = bits & 0x7F
    if e == 0xFF:
        return sign * math.inf if f == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(f, -133)              # (f / 128) * 2^-126
    return sign * math.ldexp(128 + f, e - 134)         # (1 + f / 128) * 2^(e - 127)


# every finite non-negative bf16 value, in bit order (which is value order)
_POS_BITS = np.arange(0, 0x7F80, dtype=np.int64)
_POS_VALUES = np.array([_bf16_definition(int(b)) for b in _POS_BITS], dtype=np.float64)


def _round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Nearest bf16 bit pattern of finite fp32-representable values, ties to even.

    The candidates are the two neighbouring bf16 values of |v| (2^128 above the
    largest, standing for inf).  The distances are exact in fp64: |v| has a
    24-bit significand and the neighbours lie in its binade or at its ends, so
    each difference is a multiple of |v|'s fp32 ulp below 2^53 of them.
    """
    a = np.abs(v)
    lo_i = np.searchsorted(_POS_VALUES, a, side="right") - 1
    lo = _POS_VALUES[lo_i]
    hi = np.where(lo_i + 1 < len(_POS_VALUES), _POS_VALUES[np.minimum(lo_i + 1, len(_POS_VALUES) - 1)],
                  math.ldexp(1.0, 128))
    d_lo, d_hi = a - lo, hi - a
    assert np.array_equal(lo + d_lo, a) and np.array_equal(hi - d_hi, a)
    lo_even = (_POS_BITS[lo_i] & 1) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    bits = np.where(take_hi, _POS_BITS[lo_i] + 1, _POS_BITS[lo_i])       # lo + 1 past the end is inf, 0x7F80
    bits = np.where(np.signbit(v), bits | 0x8000, bits)
    return bits.astype(np.uint16)


def test_bf16_decode_every_pattern():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):                 # signalling NaN patterns widen quietly
        got = O.bf16_to_f32(bits).astype(np.float64)
    want = np.array([_bf16_definition(int(b)) for b in bits], dtype=np.float64)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.array_equal(np.signbit(got[finite]), np.signbit(want[finite]))      # -0 decodes to -0
    inf = np.isinf(want)
    assert np.array_equal(got[inf], want[inf])
    assert np.all(np.isnan(got[np.isnan(want)]))
    assert np.array_equal(O.bf16_to_f64(bits[finite]), want[finite])


def _rounding_cases() -> np.ndarray:
    rng = np.random.default_rng(2024)
    # every midpoint between neighbouring finite bf16 values, and the fp32 values
    # one ulp either side of it (the midpoints are exact in fp32)
    mid = ((_POS_VALUES[:-1] + _POS_VALUES[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (_POS_VALUES[:-1] + _POS_VALUES[1:]) / 2)
    around = np.concatenate([mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0))])
    # the overflow edge: the largest finite bf16, the midpoint to 2^128, and fp32 values around it
    top = np.float32(math.ldexp(255.5, 120))
    edge = np.array([_POS_VALUES[-1], top, np.nextafter(top, np.float32(0)), np.nextafter(top, np.float32(np.inf)),
                     np.finfo(np.float32).max], dtype=np.float32)
    # random finite fp32 bit patterns and exact bf16 values
    raw = rng.integers(0, 0x7F800000, size=200_000, dtype=np.uint32).view(np.float32)
    exact = _POS_VALUES.astype(np.float32)
    pos = np.concatenate([around, edge, raw, exact, np.array([0.0], np.float32)])
    return np.concatenate([pos, -pos])


def test_f32_to_bf16_nearest_ties_even():
    v = _rounding_cases()
    got = O.f32_to_bf16(v)
    want = _round_to_bf16(v.astype(np.float64))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(v[i]), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]


def test_f32_to_bf16_worked_values():
    # 1 + 2^-8 lies halfway between 1 (mantissa 0, even) and 1 + 2^-7 (odd): ties to 1;
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): ties up
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.3895313892515355e38, 3.4e38, -0.0, 1e-45],
                 dtype=np.float32)
    got = O.f32_to_bf16(v)
    assert [hex(int(g)) for g in got] == ["0x3f80", "0x3f82", "0xbf80", "0x7f7f", "0x7f80", "0x8000", "0x0"]


def test_f64_to_bf16_rounds_through_fp32():
    # 1 + 2^-8 + 2^-30: rounded once it is past the midpoint and goes up to 1 + 2^-7
    # (0x3F81); rounded to fp32 first it becomes the midpoint 1 + 2^-8 exactly, which
    # ties to 1.0 (0x3F80).  The oracle takes the two-step reading.
    v = np.array([1 + 2 ** -8 + 2 ** -30, -(1 + 2 ** -8 + 2 ** -30)], dtype=np.float64)
    assert [hex(int(g)) for g in O.f64_to_bf16(v)] == ["0x3f80", "0xbf80"]
    rng = np.random.default_rng(7)
    x = rng.standard_normal(100_000) * np.exp2(rng.integers(-140, 120, size=100_000))
    want = _round_to_bf16(x.astype(np.float32).astype(np.float64))      # numpy's fp64 -> fp32, then the definition
    assert np.array_equal(O.f64_to_bf16(x), want)
