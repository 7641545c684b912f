"""Exact-arithmetic helpers for the pins (rationals, no floating point)."""
from fractions import Fraction

import numpy as np


def round_f32(q: Fraction) -> Fraction:
    """Round a rational to the nearest IEEE binary32 value, ties to even.

    Covers normal and subnormal results; overflow is not needed here.
    """
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                     # below 2^-126 the spacing stays 2^-149
    ulp = Fraction(2) ** (e - 23)
    k = a / ulp
    n = k.numerator // k.denominator
    rem = k - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def frac(x) -> Fraction:
    """Exact rational value of a float / numpy float."""
    return Fraction(float(x))


def f32(q: Fraction) -> np.float32:
    """A rational that is exactly a binary32 value, as np.float32."""
    v = np.float32(float(q))
    assert Fraction(float(v)) == q
    return v


def round_bits(q: Fraction, mant_bits: int, min_exp: int) -> Fraction:
    """Round a rational to the nearest binary float with `mant_bits` fraction
    bits and smallest normal exponent `min_exp`, ties to even (no overflow)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, min_exp)
    ulp = Fraction(2) ** (e - mant_bits)
    k = a / ulp
    n = k.numerator // k.denominator
    rem = k - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def round_bf16(q: Fraction) -> Fraction:
    """Nearest bfloat16 value (7 fraction bits, fp32 exponent range), ties to even."""
    return round_bits(q, 7, -126)
