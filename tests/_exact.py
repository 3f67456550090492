"""Exact rational arithmetic and IEEE-754 rounding from the definition, for the oracle's pins.

Nothing here is the method: these helpers only round an exact rational number to the nearest
binary32 / binary16 value (ties to the even significand), so a test can evaluate a tiny case
exactly and independently of the oracle's C code.
"""
from fractions import Fraction

import numpy as np


def _round(x: Fraction, p: int, emin: int, emax: int):
    """Nearest value with p significand bits and exponents in [emin, emax]; ties to even.
    Returns a Fraction, or +-inf as a float when it overflows."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    spacing = Fraction(2) ** (e - p + 1)
    q = a / spacing
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = n * spacing
    largest = (2 - Fraction(2) ** (1 - p)) * Fraction(2) ** emax
    if v > largest:
        return float("inf") * sign
    return sign * v


def round_f32(x: Fraction) -> np.float32:
    r = _round(x, 24, -126, 127)
    return np.float32(float(r))


def round_f16(x: Fraction) -> np.float16:
    r = _round(x, 11, -14, 15)
    return np.float16(float(r))


def frac(v) -> Fraction:
    return Fraction(float(v))
