"""The input generator: Philox4x32-10 known-answer vectors (Random123's published
test vectors) and the statistics of the synthetic KV caches."""
import numpy as np

from kv_cache_compression_cachegen_b200 import synth

KAT = [  # counter (4 words), key (2 words) -> output (4 words)
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


def test_philox_known_answers():
    for ctr, key, want in KAT:
        got = synth.philox4x32_10(*[np.array([c], np.uint64) for c in ctr], *key)
        assert tuple(int(g[0]) for g in got) == want


def test_generator_is_deterministic_and_shaped():
    a = synth.generate_cpu(2, 2, 16, 50, seed=5)
    b = synth.generate_cpu(2, 2, 16, 50, seed=5)
    c = synth.generate_cpu(2, 2, 16, 50, seed=6)
    assert a.shape == (2, 2, 50, 2, 16) and a.dtype == np.uint16
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_generator_statistics():
    rho, p = 0.95, 0.05
    kv = synth.generate_cpu(2, 4, 64, 400, seed=1, rho=rho, p_out=p, m_out=8.0)
    x = kv.view(np.float16).astype(np.float64).transpose(0, 1, 3, 4, 2).reshape(-1, 400)
    x = x - x.mean(axis=1, keepdims=True)
    r1 = (x[:, 1:] * x[:, :-1]).sum(axis=1) / (x * x).sum(axis=1)
    assert abs(np.median(r1) - rho) < 0.05            # AR(1) lag-1 correlation
    amp = np.sqrt((x * x).mean(axis=1))
    frac_out = np.mean(amp > 4 * np.median(amp))
    assert 0.01 < frac_out < 0.12                     # ~p of the channels are x8 outliers


def test_level_schedule():
    s = synth.level_schedule(52, seed=3)
    assert len(s) == 52 and set(s) <= {0, 1, 2} and len(set(s)) == 3
    assert s == synth.level_schedule(52, seed=3)
