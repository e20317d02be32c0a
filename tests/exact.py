"""Exact rational helpers for pinning the oracle (independent of oracle.c).

Everything here uses Python's ``fractions.Fraction`` so that the expected
values carry no rounding except the single rounding the definition asks for.
"""
from __future__ import annotations

from fractions import Fraction
import math
import struct

import numpy as np


def bf16_bits_to_fraction(h: int) -> Fraction:
    f = struct.unpack("<f", struct.pack("<I", (int(h) & 0xFFFF) << 16))[0]
    return Fraction(f)


def _round_half_even(x: Fraction) -> int:
    fl = math.floor(x)
    rem = x - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def fraction_to_bf16_bits(x: Fraction) -> int:
    """Nearest bf16 value of an exact rational, ties to even (finite inputs)."""
    if x == 0:
        return 0
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    # exponent of the leading bit: 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp_e = max(e - 7, -133)
    n = _round_half_even(a / (Fraction(2) ** ulp_e))
    val = Fraction(n) * (Fraction(2) ** ulp_e)
    if val > Fraction(255) * Fraction(2) ** 120:
        return sign | 0x7F80
    bits = struct.unpack("<I", struct.pack("<f", float(val)))[0]
    return sign | ((bits >> 16) & 0x7FFF)


def exact_cube_mean_bits(x_bits: np.ndarray, n: int) -> int:
    """bf16 of (correctly rounded double of (exact sum / n)): the definition
    'sum over the valid tokens, divide by the count, cast back to bf16'
    with the division done in IEEE double."""
    if n == 0:
        return 0
    s = sum((bf16_bits_to_fraction(int(v)) for v in x_bits[:n]), Fraction(0))
    # test data keep the exact sum representable in double, so the only
    # roundings are the IEEE double division and the final bf16 rounding
    assert Fraction(float(s)) == s, "test data must keep the cube sum exact in double"
    q = float(s) / float(n)
    return fraction_to_bf16_bits(Fraction(q))
