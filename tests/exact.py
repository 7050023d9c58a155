"""Exact-rational helpers used to pin the oracle (pure Python, no oracle code)."""
from __future__ import annotations

import math
import struct
from fractions import Fraction


def floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def round_to_precision(q: Fraction, mant_bits: int, min_exp: int, max_exp: int) -> float:
    """Round an exact rational to a binary float with `mant_bits` fraction bits,
    normal exponents in [min_exp, max_exp] and gradual underflow; ties to even."""
    if q == 0:
        return 0.0
    sign = -1.0 if q < 0 else 1.0
    a = abs(q)
    e = max(floor_log2(a), min_exp)
    ulp_exp = e - mant_bits
    t = a / (Fraction(2) ** ulp_exp) if ulp_exp >= 0 else a * (2 ** (-ulp_exp))
    n = t.numerator // t.denominator
    rem = t - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = Fraction(n) * (Fraction(2) ** ulp_exp)
    if v >= Fraction(2) ** (max_exp + 1):
        return sign * math.inf
    return sign * float(v)


def bf16_exact(q: Fraction) -> float:
    return round_to_precision(q, 7, -126, 127)


def f32_exact(q: Fraction) -> float:
    return round_to_precision(q, 23, -126, 127)


def bf16_bits(x: float) -> int:
    """Bit pattern of a float that is exactly representable in bf16."""
    u = struct.unpack("<I", struct.pack("<f", x))[0]
    assert u & 0xFFFF == 0, x
    return u >> 16
