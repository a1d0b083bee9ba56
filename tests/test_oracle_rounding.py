"""Pins of the oracle's two rounding rules, on inputs where the wrong rule
gives a different answer.

1. The quotient.  A code is roundf(RN(d / s)): the IEEE round-to-nearest
   quotient, then round half away from zero.  Multiplying by a rounded
   reciprocal, RN(d * RN(1/s)), lands on the other side of a half-integer for
   some d when s is not a power of two (0.3, 0.8, 1.2, 1.5 and most anchor
   scales), and the code then differs by one.
2. The reconstruction.  A value is RN(a + RN(q * s)): the product and the sum
   each rounded to nearest, no fused multiply-add.  One rounding,
   RN(a + q * s), differs when q * s is not representable.

Every expected value below is derived here in exact rational arithmetic
(tests/exact.py: Fraction values of the floats, rn_f32 = round to the nearest
float32, ties to even), never by calling the oracle.  The cases are the ones the
GPU parity test tests/test_gpu_rounding.py feeds through the kernels.
"""
from fractions import Fraction

import numpy as np
import pytest

from exact import frac, rn_f32

S03 = Fraction(10066330, 2**25)    # 0.3f  = 0x3E99999A
S08 = Fraction(13421773, 2**24)    # 0.8f  = 0x3F4CCCCD
S12 = Fraction(10066330, 2**23)    # 1.2f  = 0x3F99999A
S15 = Fraction(3, 2)               # 1.5f, exact


def _half_away(y: Fraction) -> int:
    """roundf: nearest integer, halves away from zero."""
    a = abs(y)
    r = int(a + Fraction(1, 2))
    return r if y >= 0 else -r


def _code_by_division(d: Fraction, s: Fraction) -> int:
    return max(-127, min(127, _half_away(frac(rn_f32(d / s)))))


def _code_by_reciprocal(d: Fraction, s: Fraction) -> int:
    r = frac(rn_f32(1 / s))
    return max(-127, min(127, _half_away(frac(rn_f32(d * r)))))


def test_step_constants_are_the_float32_roundings():
    assert frac(np.float32(0.3)) == S03
    assert frac(np.float32(0.8)) == S08
    assert frac(np.float32(1.2)) == S12
    assert frac(np.float32(1.5)) == S15


# (d, s, code by IEEE division, code a reciprocal multiply would give)
QUOTIENT_CASES = [
    # 2.25 / 0.3f = 37748736 / 5033165 = 7.49999970..., whose nearest float is
    # 7.5 - 2^-21 (7.5 itself is 2.98e-7 away, more than half a spacing
    # 2^-21 / 2), so the code is 7; 2.25 * RN(1/0.3f) = 7.49999982... rounds to
    # 7.5 and would give 8.
    (Fraction(9, 4), S03, 7, 8),
    (Fraction(-9, 4), S03, -7, -8),
    (Fraction(15, 4), S03, 12, 13),
    (Fraction(33, 4), S03, 27, 28),
    # 9 / 1.2f: the same quotient one binade up.
    (Fraction(9), S12, 7, 8),
    (Fraction(15), S12, 12, 13),
    # 15728639 * 2^-22 / 1.5 = 2.4999998..., nearest float below 2.5 -> 2;
    # RN(1/1.5f) = 0.6666667 (above 2/3) lifts the product to 2.5 -> 3.
    (Fraction(15728639, 2**22), S15, 2, 3),
    # 5452595 * 2^-20 / 0.8f -> 6.4999997..., code 6; reciprocal 1.25 exactly
    # gives 6.4999998 * 1.25 rounding to 6.5 -> 7.
    (Fraction(5452595, 2**20), S08, 6, 7),
]


@pytest.mark.parametrize("d,s,want,rcp", QUOTIENT_CASES)
def test_delta_code_is_ieee_quotient_then_half_away(oracle_lib, d, s, want, rcp):
    assert _code_by_division(d, s) == want
    assert _code_by_reciprocal(d, s) == rcp != want  # the case separates the two rules
    # x - a = d exactly (a = 0), so the oracle's code must be the division's
    assert oracle_lib.delta_code(float(d), 0.0, float(s)) == want
    # with a non-zero reconstructed anchor a: x = d + a, both float32 values, so
    # that x - a = d exactly
    a = next(a for a in (Fraction(1, 2), Fraction(1, 8), Fraction(1, 2**20))
             if frac(rn_f32(d + a)) == d + a)
    assert oracle_lib.delta_code(float(d + a), float(a), float(s)) == want


@pytest.mark.parametrize("d,s,want,rcp", QUOTIENT_CASES)
def test_anchor_code_is_ieee_quotient_then_half_away(oracle_lib, d, s, want, rcp):
    # The anchor code divides x - zp by the channel's scale the same way.
    assert oracle_lib.anchor_code(float(d), 0.0, float(s)) == want
    z = next(z for z in (Fraction(-3, 4), Fraction(-1, 8), Fraction(-1, 2**20))
             if frac(rn_f32(d + z)) == d + z)
    assert oracle_lib.anchor_code(float(d + z), float(z), float(s)) == want


def test_anchor_code_of_a_realistic_channel(oracle_lib):
    # Anchors lo = -7.68359375, hi = 4.46484375 (fp16 values), zp =
    # RN(RN(lo + hi) / 2) = -1.609375, scale = RN(RN(hi - lo) / 254), and the
    # anchor x = 1.427734375: RN((x - zp) / scale) is the float just above
    # 63.5, so the code is 64, while the reciprocal product rounds below 63.5.
    lo, hi, x = Fraction(-7.68359375), Fraction(4.46484375), Fraction(1.427734375)
    zp = rn_f32(frac(rn_f32(lo + hi)) * Fraction(1, 2))
    sc = rn_f32(frac(rn_f32(hi - lo)) / 254)
    d = frac(rn_f32(x - frac(zp)))
    want = _code_by_division(d, frac(sc))
    assert want != _code_by_reciprocal(d, frac(sc))
    assert want == 64
    z, s = oracle_lib.anchor_params(np.array([float(lo), float(hi), float(x)], np.float32))
    assert z == zp and s == sc
    assert oracle_lib.anchor_code(float(x), z, s) == want


# (a, q, s, value with two roundings RN(a + RN(q s)), value with one RN(a + q s))
RECON_CASES = [
    # 25 * 0.8f = 20 + 5 * 2^-24; float32 spacing at 20 is 2^-19, so
    # RN(-25 * 0.8f) = -20 and 20 + (-20) = +0 exactly.  One rounding keeps
    # the residue: RN(20 - 20 - 5 * 2^-24) = -5 * 2^-24 (fp16 0x8005).
    (Fraction(20), -25, S08, Fraction(0), Fraction(-5, 2**24)),
    (Fraction(36), -45, S08, Fraction(0), Fraction(-9, 2**24)),
    (Fraction(64), -80, S08, Fraction(0), Fraction(-16, 2**24)),
]


def test_recon_cases_are_derived_exactly():
    for a, q, s, two, one in RECON_CASES:
        assert frac(rn_f32(a + frac(rn_f32(q * s)))) == two
        assert frac(rn_f32(a + q * s)) == one
        assert two != one


@pytest.mark.parametrize("a,q,s,two,one", RECON_CASES)
def test_delta_value_rounds_product_then_sum(oracle_lib, a, q, s, two, one):
    got = oracle_lib.delta_value(q, float(a), float(s))
    assert frac(got) == two and not np.signbit(got)
    assert oracle_lib.f32_to_f16([got])[0] == 0x0000
    assert oracle_lib.f32_to_f16([np.float32(float(one))])[0] != 0x0000


@pytest.mark.parametrize("a,q,s,two,one", RECON_CASES)
def test_anchor_value_rounds_product_then_sum(oracle_lib, a, q, s, two, one):
    got = oracle_lib.anchor_value(q, float(a), float(s))
    assert frac(got) == two and not np.signbit(got)


def test_recon_with_a_many_bit_anchor(oracle_lib):
    # a = 2.046875, q = -55, s = 1.2f: RN(-55 * 1.2f) = -66.00000262... rounded
    # to the float spacing 2^-17 at 66, then the sum; one rounding ends on the
    # other side of an fp16 rounding boundary.
    a, q, s = Fraction(2.046875), -55, S12
    two = rn_f32(a + frac(rn_f32(q * s)))
    one = rn_f32(a + q * s)
    assert two != one
    assert np.float16(two) != np.float16(one)
    got = oracle_lib.delta_value(q, float(a), float(s))
    assert got == two
    assert oracle_lib.f32_to_f16([got])[0] == np.float16(two).view(np.uint16)


def test_anchor_recon_of_a_realistic_channel(oracle_lib):
    # Anchors lo = -3.90625, hi = 7.62890625 and x = -0.021484375: code -41,
    # and RN(zp + RN(-41 * scale)) and RN(zp - 41 * scale) round to different
    # fp16 values.
    lo, hi, x = Fraction(-3.90625), Fraction(7.62890625), Fraction(-0.021484375)
    zp = rn_f32(frac(rn_f32(lo + hi)) * Fraction(1, 2))
    sc = rn_f32(frac(rn_f32(hi - lo)) / 254)
    c = _code_by_division(frac(rn_f32(x - frac(zp))), frac(sc))
    assert c == -41
    two = rn_f32(frac(zp) + frac(rn_f32(c * frac(sc))))
    one = rn_f32(frac(zp) + c * frac(sc))
    assert np.float16(two) != np.float16(one)
    z, s = oracle_lib.anchor_params(np.array([float(lo), float(hi), float(x)], np.float32))
    assert oracle_lib.anchor_code(float(x), z, s) == c
    got = oracle_lib.anchor_value(c, z, s)
    assert got == two


def test_chunk_path_uses_both_rules(oracle_lib):
    # The same cases through the chunk quantiser and the container round trip:
    # 3 layers at the high level (steps 0.3 / 0.8 / 1.2 by third), one head of
    # 16 channels, one 20-token chunk (anchors at tokens 0 and 10).
    kv = np.zeros((3, 2, 20, 1, 16), dtype=np.float16)
    kv[0, 0, 1, 0, 0] = 2.25    # step 0.3: code 7 (a reciprocal gives 8)
    kv[0, 0, 2, 0, 0] = -2.25   # -7
    kv[0, 0, 3, 0, 0] = 3.75    # 12
    kv[2, 0, 1, 0, 0] = 9.0     # step 1.2: 7
    kv[2, 0, 2, 0, 0] = 15.0    # 12
    kv[1, 0, :, 0, 1] = 20.0    # constant anchors 20 at step 0.8 ...
    kv[1, 0, 3, 0, 1] = 0.0     # ... and a delta token 0: code -25, value +0
    kv[1, 0, :, 0, 2] = 36.0
    kv[1, 0, 4, 0, 2] = 0.0     # code -45, value +0
    h = kv.view(np.uint16)
    rc, sym, zp, sc = oracle_lib.quantize_chunk(h, 0, 20, 0)
    assert rc == 0
    q = sym.astype(int) - 127
    assert [q[0, 0, t, 0, 0] for t in (1, 2, 3)] == [7, -7, 12]
    assert [q[2, 0, t, 0, 0] for t in (1, 2)] == [7, 12]
    assert q[1, 0, 3, 0, 1] == -25 and q[1, 0, 4, 0, 2] == -45
    rc, cont = oracle_lib.encode_chunk(h, 0, 20, 0)
    assert rc == 0
    rc, out, n, _ = oracle_lib.decode_chunk(cont, 3, 1, 16, 20, 0)
    assert rc == 0
    assert out[1, 0, 3, 0, 1] == 0x0000 and out[1, 0, 4, 0, 2] == 0x0000
    # 7 * 0.3f and 12 * 0.3f rounded to fp16
    for t, c in ((1, 7), (2, -7), (3, 12)):
        want = np.float16(rn_f32(c * S03)).view(np.uint16)
        assert out[0, 0, t, 0, 0] == want
