"""Exact-arithmetic helpers for the oracle pins (Python integers and fractions)."""
from fractions import Fraction

import numpy as np


def frac(x) -> Fraction:
    """The exact rational value of a float32 / float64 / float16 number."""
    return Fraction(float(x))


def rn_f32(q: Fraction) -> np.float32:
    """Round a rational to the nearest float32, ties to even (normal and subnormal range)."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    sp = max(e - 23, -149)
    m = a / (Fraction(2) ** sp)
    r = round(m)  # Fraction.__round__: nearest, ties to even
    return np.float32(sign * r * 2.0 ** sp)


def argmin_code(d: Fraction, s: Fraction) -> int:
    """argmin over q in [-127, 127] of |d - q s|; equal distances go away from zero."""
    den = d.denominator * s.denominator
    dn = d.numerator * s.denominator
    sn = s.numerator * d.denominator
    best_q, best_e = None, None
    for q in range(-127, 128):
        err = abs(dn - q * sn)
        if best_e is None or err < best_e or (err == best_e and abs(q) > abs(best_q)):
            best_q, best_e = q, err
    assert den > 0
    return best_q


def near_half(d: Fraction, s: Fraction, rel: float = 2.0 ** -21) -> bool:
    """True when d/s lies within rel*|d/s| of a half-integer (rounding may legitimately tip)."""
    y = d / s
    base = Fraction(y.__floor__()) + Fraction(1, 2)  # the half-integer inside [floor y, floor y + 1)
    for h in (base - 1, base, base + 1):
        if abs(y - h) <= abs(y) * Fraction(rel) + Fraction(1, 2**40):
            return True
    return False
