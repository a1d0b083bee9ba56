"""Pin the oracle's own fp32 <-> fp16 conversions to numpy's IEEE conversions."""
import numpy as np


def test_f16_to_f32_all_patterns(oracle_lib):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle_lib.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f16_round_trip_is_identity(oracle_lib):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    back = oracle_lib.f32_to_f16(oracle_lib.f16_to_f32(h))
    finite = (h & 0x7C00) != 0x7C00
    assert np.array_equal(back[finite], h[finite])
    inf = ((h & 0x7FFF) == 0x7C00)
    assert np.array_equal(back[inf], h[inf])


def _stratified_floats(rng):
    # Every sign x fp32 exponent that can land near the fp16 range x every top-10
    # mantissa pattern, with the low 13 bits at the rounding-critical values
    # (exact, just above/below half an fp16 ulp, exactly half) plus random ones.
    sign = np.array([0, 1], dtype=np.uint32)
    exp = np.arange(98, 145, dtype=np.uint32)          # 2^-29 .. 2^17
    top = np.arange(1024, dtype=np.uint32)
    low = np.array([0, 1, 0x0FFF, 0x1000, 0x1001, 0x1FFF], dtype=np.uint32)
    s, e, t, lo = np.meshgrid(sign, exp, top, low, indexing="ij")
    bits = (s << 31) | (e << 23) | (t << 13) | lo
    rnd = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    special = np.array([0x00000000, 0x80000000, 0x7F800000, 0xFF800000, 0x477FE000,
                        0x477FEFFF, 0x477FF000, 0x477FF001, 0x33000000, 0x33000001,
                        0x32FFFFFF, 0x387FC000, 0x38800000], dtype=np.uint32)
    return np.concatenate([bits.ravel(), rnd, special]).view(np.float32)


def test_f32_to_f16_matches_numpy(oracle_lib):
    x = _stratified_floats(np.random.default_rng(7))
    ours = oracle_lib.f32_to_f16(x)
    with np.errstate(over="ignore", invalid="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.all((ours[nan] & 0x7C00) == 0x7C00) and np.all((ours[nan] & 0x3FF) != 0)
