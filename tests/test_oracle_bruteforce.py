"""Brute-force pin of the oracle's quantiser on a 2-layer, 1-head, 8-dim, 20-token
KV cache: every code must be the argmin over all 255 codes of the reconstruction
distance (equal distances away from zero), every zero point / scale must span the
anchors' range, and every decoded value must be the fp16 of the reconstruction.
Where the exact quotient lies so close to a half-integer that the float32
quotient may round onto either side, the code must be the one the definition
gives: roundf of the round-to-nearest float32 quotient (computed here in exact
rationals), and every decoded value must be the two-rounding reconstruction
RN(a + RN(q * s)) of the codes.
"""
from fractions import Fraction

import numpy as np
import pytest

from exact import argmin_code, frac, near_half, rn_f32


def _defn_code(d: Fraction, s: Fraction) -> int:
    """clamp(roundf(RN(d / s))): the float32 quotient, halves away from zero."""
    y = frac(rn_f32(d / s))
    r = int(abs(y) + Fraction(1, 2))
    return max(-127, min(127, r if y >= 0 else -r))

L, H, D, T = 2, 1, 8, 20


def _kv(seed):
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(L, 2, T, H, D)).cumsum(axis=2) * 0.7
    x[0, 0, :, 0, 0] = 0.375          # a constant channel: scale 0
    x[1, 1, :, 0, 3] *= 60.0          # an outlier channel: deltas clamp at +-127
    x[0, 1, 5, 0, 2] = x[0, 1, 0, 0, 2]  # exact repeat of an anchor value
    return x.astype(np.float16).view(np.uint16)


def _expected_chunk(kv, t0, C, level, oracle_lib):
    """Quantise one chunk with exact arithmetic and exhaustive search."""
    n = min(C, T - t0)
    vals = kv.view(np.float16).astype(np.float32)
    sym = np.zeros((L, 2, n, H, D), dtype=np.int64)
    dec = np.zeros((L, 2, n, H, D), dtype=np.float32)
    zps = np.zeros((L, 2, H, D), dtype=np.float32)
    scs = np.zeros((L, 2, H, D), dtype=np.float32)
    fuzzy = np.zeros((L, 2, n, H, D), dtype=bool)
    defn = np.zeros((L, 2, n, H, D), dtype=np.int64)
    for l in range(L):
        s = frac(oracle_lib.step(level, l, L))
        for kv_ in range(2):
            for d in range(D):
                col = vals[l, kv_, t0:t0 + n, 0, d]
                anchors = col[::10]
                lo, hi = frac(anchors.min()), frac(anchors.max())
                zp = rn_f32(frac(rn_f32(lo + hi)) * Fraction(1, 2))
                sc = rn_f32(frac(rn_f32(hi - lo)) / 254)
                zps[l, kv_, 0, d], scs[l, kv_, 0, d] = zp, sc
                for g0 in range(0, n, 10):
                    xa = frac(col[g0])
                    if sc == 0:
                        c = dfc = 0
                    else:
                        da = xa - frac(zp)
                        c = argmin_code(da, frac(sc))
                        fuzzy[l, kv_, g0, 0, d] = near_half(frac(rn_f32(da)), frac(sc))
                        dfc = _defn_code(frac(rn_f32(da)), frac(sc))
                        if fuzzy[l, kv_, g0, 0, d]:
                            c = dfc  # the definition decides near a half
                    defn[l, kv_, g0, 0, d] = dfc
                    ahat = rn_f32(frac(zp) + frac(rn_f32(c * frac(sc))))
                    sym[l, kv_, g0, 0, d] = c
                    dec[l, kv_, g0, 0, d] = ahat
                    for t in range(g0 + 1, min(g0 + 10, n)):
                        dd = frac(col[t]) - frac(ahat)
                        q = argmin_code(dd, s)
                        fuzzy[l, kv_, t, 0, d] = near_half(frac(rn_f32(dd)), s)
                        defn[l, kv_, t, 0, d] = _defn_code(frac(rn_f32(dd)), s)
                        if fuzzy[l, kv_, t, 0, d]:
                            q = defn[l, kv_, t, 0, d]
                        sym[l, kv_, t, 0, d] = q
                        dec[l, kv_, t, 0, d] = rn_f32(frac(ahat) + frac(rn_f32(q * s)))
    return sym, dec, zps, scs, fuzzy, defn


@pytest.mark.parametrize("C", [20, 16])
@pytest.mark.parametrize("level", [0, 1, 2])
@pytest.mark.parametrize("seed", [11, 12])
def test_bruteforce_tiny_cache(oracle_lib, C, level, seed):
    kv = _kv(seed)
    for t0 in range(0, T, C):
        esym, edec, ezp, esc, fuzzy, defn = _expected_chunk(kv, t0, C, level, oracle_lib)
        rc, sym, zp, sc = oracle_lib.quantize_chunk(kv, t0, C, level)
        assert rc == 0
        assert np.array_equal(zp.view(np.uint32), ezp.view(np.uint32))
        assert np.array_equal(sc.view(np.uint32), esc.view(np.uint32))
        got = sym.astype(np.int64) - 127
        exact = ~fuzzy
        assert np.array_equal(got[exact], esym[exact])
        assert np.all(np.abs(got[fuzzy] - esym[fuzzy]) <= 1)
        assert np.array_equal(got, defn)  # the float32 quotient decides every code
        # the container round trip reproduces the reconstruction of these codes
        rc, cont = oracle_lib.encode_chunk(kv, t0, C, level)
        assert rc == 0
        rc, out, n, start = oracle_lib.decode_chunk(cont, L, H, D, C, level)
        assert rc == 0 and n == min(C, T - t0) and start == t0
        assert np.array_equal(out, edec.astype(np.float16).view(np.uint16))


def test_anchor_range_is_spanned(oracle_lib):
    # the channel's largest anchor gets code +127, the smallest -127, and every
    # anchor is reconstructed within half a scale step
    kv = _kv(3)
    vals = kv.view(np.float16).astype(np.float32)
    rc, sym, zp, sc = oracle_lib.quantize_chunk(kv, 0, 20, 1)
    assert rc == 0
    for l in range(L):
        for k in range(2):
            for d in range(D):
                a = vals[l, k, 0:20:10, 0, d]
                codes = sym[l, k, 0:20:10, 0, d].astype(int) - 127
                if sc[l, k, 0, d] == 0:
                    assert np.all(codes == 0) and zp[l, k, 0, d] == a[0]
                    continue
                assert codes[np.argmax(a)] == 127 and codes[np.argmin(a)] == -127
                rec = zp[l, k, 0, d] + codes.astype(np.float64) * sc[l, k, 0, d]
                assert np.all(np.abs(rec - a) <= 0.5 * sc[l, k, 0, d] * (1 + 1e-5))


def test_ties_round_half_away_from_zero(oracle_lib):
    # Exact ties: anchors all 0 (scale 0, reconstructed anchor 0); delta x = +-0.25
    # at step 0.5 is exactly half a step -> +-1; 1.25 -> 2.5 steps -> 3 (not 2).
    kv = np.zeros((3, 2, 10, 1, 16), dtype=np.float16)
    vals = [0.25, -0.25, 0.75, -0.75, 1.25, -1.25, 0.125, 0.0, 63.75, -63.75, 64.0, 100.0,
            0.2, -0.3, 1.0, 0.5]
    kv[0, 0, 1, 0, :] = np.array(vals, dtype=np.float16)
    rc, sym, zp, sc = oracle_lib.quantize_chunk(kv.view(np.uint16), 0, 10, 1)  # balanced
    assert rc == 0 and oracle_lib.step(1, 0, 3) == np.float32(0.5)
    q = sym[0, 0, 1, 0, :].astype(int) - 127
    expect = [1, -1, 2, -2, 3, -3, 0, 0, 127, -127, 127, 127, 0, -1, 2, 1]
    assert q.tolist() == expect
    # 0.125 / 0.5 = 0.25 -> 0; 63.75 / 0.5 = 127.5 -> 128 -> clamp 127; 0.2/0.5 = 0.4 -> 0
    # -0.3/0.5 = -0.6 -> -1


def test_constant_channel_is_exact(oracle_lib):
    kv = np.full((1, 2, 23, 1, 16), 0.7, dtype=np.float16)
    rc, cont = oracle_lib.encode_chunk(kv.view(np.uint16), 0, 23, 2)
    assert rc == 0
    rc, out, n, _ = oracle_lib.decode_chunk(cont, 1, 1, 16, 23, 2)
    assert rc == 0 and np.array_equal(out.ravel(), kv.view(np.uint16).ravel())
