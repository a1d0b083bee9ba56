"""Pins of the oracle's rANS coder: hand-worked streams, a closed form for the
stream length, lossless round trips, the entropy bound, and corrupt streams."""
import math

import numpy as np
import pytest

from kv_cache_compression_cachegen_b200 import synth  # noqa: F401  (package import check)


def _table(fs):
    f = np.zeros(256, dtype=np.uint16)
    for u, v in fs.items():
        f[u] = v
    assert f.sum() == 4096
    return f


def test_hand_worked_one_symbol_stream(oracle_lib):
    # f = {0: 4095, 1: 1}; encode [1] from x = 2^15: no renormalisation (32768 < 1 << 19),
    # x = 32768 * 4096 + 0 + 4095 = 0x08000FFF -> words [0x0800, 0x0FFF].
    f = _table({0: 4095, 1: 1})
    w = oracle_lib.rans_encode(np.array([1], np.uint8), 1, f)
    assert w.tolist() == [0x0800, 0x0FFF]
    rc, s = oracle_lib.rans_decode(w, 1, 1, f)
    assert rc == 0 and s.tolist() == [1]


def test_hand_worked_two_symbol_stream(oracle_lib):
    # encode [0, 0] with f0 = 4095: 32768 = 8*4095 + 8 -> 8*4096 + 8 = 32776
    # = 8*4095 + 16 -> 8*4096 + 16 = 32784 = 0x8010 -> words [0x0000, 0x8010].
    f = _table({0: 4095, 1: 1})
    w = oracle_lib.rans_encode(np.array([0, 0], np.uint8), 2, f)
    assert w.tolist() == [0x0000, 0x8010]
    rc, s = oracle_lib.rans_decode(w, 2, 2, f)
    assert rc == 0 and s.tolist() == [0, 0]


def test_single_symbol_table_costs_only_the_state(oracle_lib):
    f = _table({42: 4096})
    w = oracle_lib.rans_encode(np.full(4096, 42, np.uint8), 4096, f)
    assert w.tolist() == [0, 0x8000]  # the state never moves from 2^15


@pytest.mark.parametrize("N", [1, 3, 4, 5, 8, 1023, 1024, 4096])
def test_uniform_sixteen_symbol_closed_form(oracle_lib, N):
    # 16 symbols at f = 256: each step multiplies the state by 16, so from 2^15 the
    # state reaches 2^27 = 256 << 19 after three symbols and renormalises before every
    # fourth: floor(N/4) words plus the two words of the final state.
    f = _table({u: 256 for u in range(16)})
    rng = np.random.default_rng(N)
    s = rng.integers(0, 16, size=N).astype(np.uint8)
    w = oracle_lib.rans_encode(s, N, f)
    assert w.size == 2 + N // 4
    rc, back = oracle_lib.rans_decode(w, N, N, f)
    assert rc == 0 and np.array_equal(back, s)


def _random_table(rng, k):
    c = np.zeros(255, dtype=np.uint64)
    sup = rng.choice(255, size=k, replace=False)
    c[sup] = rng.integers(1, 1000, size=k)
    return c


@pytest.mark.parametrize("seed", range(8))
def test_round_trip_multi_table(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    per_table, ntab = 128, 8
    freqs, syms = [], []
    for _ in range(ntab):
        c = _random_table(rng, int(rng.integers(1, 60)))
        f = oracle_lib.normalize(c)
        freqs.append(f)
        p = f[:255].astype(np.float64) / 4096
        syms.append(rng.choice(255, size=per_table, p=p))
    freq = np.stack(freqs).astype(np.uint16)
    s = np.concatenate(syms).astype(np.uint8)
    w = oracle_lib.rans_encode(s, per_table, freq)
    rc, back = oracle_lib.rans_decode(w, s.size, per_table, freq)
    assert rc == 0 and np.array_equal(back, s)
    # Entropy bound: the stream costs the symbols' information content under the
    # table (within 1%) plus at most 48 bits of state flush and tail.
    info = sum(-math.log2(freq[j // per_table][s[j]] / 4096) for j in range(s.size))
    assert 16 * w.size <= 1.01 * info + 48


def test_corrupt_streams_are_rejected(oracle_lib):
    rng = np.random.default_rng(5)
    f = oracle_lib.normalize(_random_table(rng, 40))
    p = f[:255].astype(np.float64) / 4096
    s = rng.choice(255, size=1024, p=p).astype(np.uint8)
    w = oracle_lib.rans_encode(s, 1024, f)
    assert oracle_lib.rans_decode(w[:-1], 1024, 1024, f)[0] == oracle_lib.CORRUPT
    assert oracle_lib.rans_decode(np.append(w, 7), 1024, 1024, f)[0] == oracle_lib.CORRUPT
    bad = f.copy()
    bad[np.argmax(bad)] -= 1  # sums to 4095
    assert oracle_lib.rans_decode(w, 1024, 1024, bad)[0] == oracle_lib.CORRUPT


def test_symbol_absent_from_table_cannot_be_encoded(oracle_lib):
    f = _table({0: 4096})
    with pytest.raises(ValueError):
        oracle_lib.rans_encode(np.array([1], np.uint8), 1, f)
