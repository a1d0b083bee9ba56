"""Pins of the oracle's format 2: deltas between adjacent tokens ([Practice] 1
read literally).  Inside a group the anchor is coded as in format 1; token t is
quantised against the reconstruction of token t - 1, x^_t = x^_(t-1) + q_t s,
and the chain restarts at every anchor.

Pinned against exact rational arithmetic with exhaustive search over the 255
codes (each step given the previous reconstruction), exact integer walks whose
codes are known in closed form, the per-token error bound, and the container
format (version field, sections shared with format 1)."""
from fractions import Fraction

import numpy as np
import pytest

from exact import argmin_code, frac, near_half, rn_f32

L, H, D, T = 2, 1, 8, 20


def _kv(seed):
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(L, 2, T, H, D)).cumsum(axis=2) * 0.7
    x[0, 0, :, 0, 0] = 0.375          # a constant channel: scale 0
    x[1, 1, :, 0, 3] *= 60.0          # an outlier channel: some deltas clamp
    return x.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("C", [20, 16])
@pytest.mark.parametrize("level", [0, 1, 2])
@pytest.mark.parametrize("seed", [11, 12])
def test_bruteforce_chain(oracle_lib, C, level, seed):
    kv = _kv(seed)
    vals = kv.view(np.float16).astype(np.float32)
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        rc, sym, zp, sc = oracle_lib.quantize_chunk(kv, t0, C, level, adjacent=True)
        assert rc == 0
        rc1, sym1, zp1, sc1 = oracle_lib.quantize_chunk(kv, t0, C, level)
        assert rc1 == 0
        # the anchor part is format 1's (pinned by its own brute-force test)
        assert np.array_equal(zp.view(np.uint32), zp1.view(np.uint32))
        assert np.array_equal(sc.view(np.uint32), sc1.view(np.uint32))
        assert np.array_equal(sym[:, :, ::10], sym1[:, :, ::10])
        q = sym.astype(np.int64) - 127
        expect_dec = np.zeros((L, 2, n, H, D), dtype=np.float32)
        for l in range(L):
            s = frac(oracle_lib.step(level, l, L))
            for k in range(2):
                for d in range(D):
                    col = vals[l, k, t0:t0 + n, 0, d]
                    for g0 in range(0, n, 10):
                        ref = rn_f32(frac(zp[l, k, 0, d]) +
                                     frac(rn_f32(int(q[l, k, g0, 0, d]) * frac(sc[l, k, 0, d]))))
                        expect_dec[l, k, g0, 0, d] = ref
                        for t in range(g0 + 1, min(g0 + 10, n)):
                            dd = frac(col[t]) - frac(ref)
                            want = argmin_code(dd, s)
                            got = int(q[l, k, t, 0, d])
                            if near_half(frac(rn_f32(dd)), s):
                                assert abs(got - want) <= 1
                            else:
                                assert got == want, (l, k, d, t)
                            # the next token builds on this token's reconstruction
                            ref = rn_f32(frac(ref) + frac(rn_f32(got * s)))
                            expect_dec[l, k, t, 0, d] = ref
        rc, cont = oracle_lib.encode_chunk(kv, t0, C, level, adjacent=True)
        assert rc == 0
        rc, out, nn, start = oracle_lib.decode_chunk(cont, L, H, D, C, level, adjacent=True)
        assert rc == 0 and nn == n and start == t0
        assert np.array_equal(out, expect_dec.astype(np.float16).view(np.uint16))


def _walk_cache(steps_per_layer, k):
    """Anchors of every channel equal A (scale 0, so the reconstructed anchor is
    A exactly); token t of a group holds A + k_t s with k the integer walk."""
    A = np.float16(3.0)
    Lw = len(steps_per_layer)
    n = k.shape[0]
    x = np.zeros((Lw, 2, n, 1, k.shape[1]), dtype=np.float64)
    for l, s in enumerate(steps_per_layer):
        x[l, :, :, 0, :] = float(A) + k * s
    kv = x.astype(np.float16)
    assert np.array_equal(kv.astype(np.float64), x)  # every value exact in fp16
    return kv.view(np.uint16)


def test_integer_walk_codes_in_closed_form(oracle_lib):
    # 3 layers at the balanced level: steps 0.5 / 1.0 / 1.5 (all exact in fp16)
    steps = [0.5, 1.0, 1.5]
    assert [float(oracle_lib.step(1, l, 3)) for l in range(3)] == steps
    rng = np.random.default_rng(4)
    n, Dw = 30, 16
    inc = rng.integers(-60, 61, size=(n, Dw))
    inc[::10] = 0                      # anchors: k = 0
    k = np.zeros((n, Dw), dtype=np.int64)
    for t in range(n):
        k[t] = 0 if t % 10 == 0 else k[t - 1] + inc[t]
    kv = _walk_cache(steps, k)
    rc2, sym2, _, _ = oracle_lib.quantize_chunk(kv, 0, n, 1, adjacent=True)
    rc1, sym1, _, _ = oracle_lib.quantize_chunk(kv, 0, n, 1)
    assert rc1 == 0 and rc2 == 0
    for l in range(3):
        for kvi in range(2):
            q2 = sym2[l, kvi, :, 0, :].astype(np.int64) - 127
            q1 = sym1[l, kvi, :, 0, :].astype(np.int64) - 127
            # format 2 codes the increments, format 1 the (clamped) offsets
            assert np.array_equal(q2, inc)
            assert np.array_equal(q1, np.clip(k, -127, 127))
    # format 2 reconstructs the walk exactly, also where format 1 had to clamp
    assert np.abs(k).max() > 127
    rc, cont = oracle_lib.encode_chunk(kv, 0, n, 1, adjacent=True)
    assert rc == 0
    rc, out, _, _ = oracle_lib.decode_chunk(cont, 3, 1, Dw, n, 1, adjacent=True)
    assert rc == 0 and np.array_equal(out, kv.reshape(out.shape))
    rc, cont1 = oracle_lib.encode_chunk(kv, 0, n, 1)
    rc, out1, _, _ = oracle_lib.decode_chunk(cont1, 3, 1, Dw, n, 1)
    assert rc == 0 and not np.array_equal(out1, kv.reshape(out1.shape))


def test_first_delta_of_each_group_matches_format_1(oracle_lib):
    # token 1 of a group is a delta to the reconstructed anchor in both formats
    kv = _kv(5)
    rc1, s1, _, _ = oracle_lib.quantize_chunk(kv, 0, 20, 2)
    rc2, s2, _, _ = oracle_lib.quantize_chunk(kv, 0, 20, 2, adjacent=True)
    assert rc1 == 0 and rc2 == 0
    assert np.array_equal(s1[:, :, 1::10], s2[:, :, 1::10])
    assert not np.array_equal(s1, s2)


def test_error_bound_per_token(oracle_lib):
    # |x - x^| <= s/2 (+ rounding) for every unclamped delta, however far the
    # token is from its anchor: the chain re-references every token
    rng = np.random.default_rng(8)
    Lb, Hb, Db, Tb = 3, 2, 16, 64
    x = rng.normal(0, 1, size=(Lb, 2, Tb, Hb, Db)).cumsum(axis=2) * 0.4
    kv = x.astype(np.float16).view(np.uint16)
    vals = kv.view(np.float16).astype(np.float64)
    for level in range(3):
        rc, cont = oracle_lib.encode_chunk(kv, 0, Tb, level, adjacent=True)
        assert rc == 0
        rc, out, _, _ = oracle_lib.decode_chunk(cont, Lb, Hb, Db, Tb, level, adjacent=True)
        assert rc == 0
        rc, sym, _, _ = oracle_lib.quantize_chunk(kv, 0, Tb, level, adjacent=True)
        dec = out.view(np.float16).astype(np.float64)
        q = sym.astype(np.int64) - 127
        for l in range(Lb):
            s = float(oracle_lib.step(level, l, Lb))
            err = np.abs(vals[l] - dec[l])
            ulp = np.spacing(np.abs(dec[l]).astype(np.float16)).astype(np.float64)
            delta = np.ones(Tb, dtype=bool)
            delta[::10] = False
            m = delta[None, :, None, None] & (np.abs(q[l]) < 127)
            bound = s / 2 * (1 + 1e-6) + ulp / 2 + 1e-6
            assert np.all(err[m] <= np.broadcast_to(bound, err.shape)[m])


def test_container_format_2(oracle_lib):
    kv = _kv(6)
    rc1, c1 = oracle_lib.encode_chunk(kv, 0, 20, 1)
    rc2, c2 = oracle_lib.encode_chunk(kv, 0, 20, 1, adjacent=True)
    assert rc1 == 0 and rc2 == 0
    assert int(c1[4]) | (int(c1[5]) << 8) == 1
    assert int(c2[4]) | (int(c2[5]) << 8) == 2
    secs = oracle_lib.sections(L, H, D, 20)
    # same header fields apart from the version, same zero points and scales
    assert np.array_equal(c1[:4], c2[:4]) and np.array_equal(c1[6:40], c2[6:40])
    assert np.array_equal(c1[secs[0]:secs[2]], c2[secs[0]:secs[2]])
    # each decoder takes only its own format
    assert oracle_lib.decode_chunk(c2, L, H, D, 20, 1)[0] == oracle_lib.MISMATCH
    assert oracle_lib.decode_chunk(c1, L, H, D, 20, 1, adjacent=True)[0] == oracle_lib.MISMATCH
    bad = c2.copy()
    bad[4] = 3  # no format 3
    assert oracle_lib.decode_chunk(bad, L, H, D, 20, 1, adjacent=True)[0] == oracle_lib.CORRUPT


def test_format_2_streams_and_entropy_bound(oracle_lib):
    # every stream of a format-2 container decodes to the format-2 symbols under
    # tables built from those symbols, and the payload sits within 1 % (+ the
    # per-stream flush) of the tables' information content, as in format 1
    import struct
    from kv_cache_compression_cachegen_b200 import synth
    Lc, Hc, Dc, Tc = 4, 8, 128, 1536
    kv = synth.generate_cpu(Lc, Hc, Dc, Tc, seed=1)
    rc, cont = oracle_lib.encode_chunk(kv, 0, Tc, 1, adjacent=True)
    assert rc == 0
    rc, sym, _, _ = oracle_lib.quantize_chunk(kv, 0, Tc, 1, adjacent=True)
    assert rc == 0
    secs = oracle_lib.sections(Lc, Hc, Dc, Tc)
    freq = np.frombuffer(cont[secs[2]:secs[3]].tobytes(), np.uint16).reshape(Lc, 2, Hc, 256)
    assert np.array_equal(freq, oracle_lib.tables_of(sym))
    payload = struct.unpack_from("<Q", bytes(cont[40:48]))[0]
    offs = np.frombuffer(cont[secs[3]:secs[3] + 4 * (2 * Lc * Tc + 1)].tobytes(), np.uint32)
    body = cont[secs[4]:secs[4] + payload]
    for s in (0, 1, Tc - 1, Tc, 2 * Lc * Tc - 1):  # first, last and boundary streams
        l, k, t = s // (2 * Tc), (s // Tc) % 2, s % Tc
        words = np.frombuffer(body[offs[s]:offs[s + 1]].tobytes(), np.uint16)
        rc, got = oracle_lib.rans_decode(words, Hc * Dc, Dc, freq[l, k])
        assert rc == 0 and np.array_equal(got, sym[l, k, t].ravel())
    f = np.take_along_axis(freq.astype(np.float64)[:, :, None, :, :].repeat(Tc, axis=2),
                           sym.astype(np.int64).reshape(Lc, 2, Tc, Hc, Dc), axis=4)
    info = float(np.sum(-np.log2(f / 4096.0)))
    assert info <= 8 * payload <= 1.01 * info + 48 * 2 * Lc * Tc
    # on this smooth AR(1) cache the adjacent differences carry less information
    # than the differences to the anchor (the purpose of the format)
    rc1, cont1 = oracle_lib.encode_chunk(kv, 0, Tc, 1)
    assert rc1 == 0 and cont.size < cont1.size
