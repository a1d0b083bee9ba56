"""Pins of the 12-bit frequency-table normalisation: closed forms, hand-worked
examples of the two repair rules, and invariants on random histograms."""
import numpy as np
import pytest


def test_single_symbol_takes_everything(oracle_lib):
    c = np.zeros(255, dtype=np.uint64)
    c[127] = 1536 * 128
    f = oracle_lib.normalize(c)
    assert f[127] == 4096 and f.sum() == 4096


@pytest.mark.parametrize("k", [1, 2, 4, 8, 16, 64, 128])
def test_equal_counts_split_evenly(oracle_lib, k):
    c = np.zeros(255, dtype=np.uint64)
    c[:k] = 1000
    f = oracle_lib.normalize(c)
    assert np.all(f[:k] == 4096 // k) and f[k:].sum() == 0


def test_rare_symbol_gets_one(oracle_lib):
    c = np.zeros(255, dtype=np.uint64)
    c[3], c[200] = 1, 99_999
    f = oracle_lib.normalize(c)
    assert f[3] == 1 and f[200] == 4095


def test_excess_taken_from_the_largest(oracle_lib):
    # 200 symbols seen once and one symbol seen N-200 times, N = 10000:
    # floor shares 1 (x200) and floor(9800*4096/10000) = 4014, sum 4214, excess 118,
    # all taken from the largest: 4014 - 118 = 3896.
    c = np.zeros(255, dtype=np.uint64)
    c[:100] = 1
    c[101:201] = 1
    c[100] = 9800
    f = oracle_lib.normalize(c)
    assert f[100] == 3896
    assert np.all(f[:100] == 1) and np.all(f[101:201] == 1) and f.sum() == 4096


def test_excess_alternates_between_tied_maxima(oracle_lib):
    # u=10 and u=20 seen 5000 times, 99 others once (N = 10099): shares 2027, 2027
    # and 99 ones, sum 4153, excess 57.  Ties go to the smaller u first, so u=10 loses
    # 29 and u=20 loses 28.
    c = np.zeros(255, dtype=np.uint64)
    c[10] = c[20] = 5000
    rare = [u for u in range(255) if u not in (10, 20)][:99]
    c[rare] = 1
    f = oracle_lib.normalize(c)
    assert (int(f[10]), int(f[20])) == (1998, 1999)
    assert f.sum() == 4096


def test_deficit_goes_to_the_most_frequent(oracle_lib):
    # counts 3, 3, 1 (N = 7): shares 1755, 1755, 585 = 4095; the missing 1 goes to the
    # most frequent symbol, ties to the smaller u.
    c = np.zeros(255, dtype=np.uint64)
    c[5], c[9], c[200] = 3, 3, 1
    f = oracle_lib.normalize(c)
    assert (int(f[5]), int(f[9]), int(f[200])) == (1756, 1755, 585)


@pytest.mark.parametrize("seed", range(20))
def test_random_histogram_invariants(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    k = int(rng.integers(1, 256))
    support = rng.choice(255, size=min(k, 255), replace=False)
    c = np.zeros(255, dtype=np.uint64)
    # heavy-tailed counts so that many symbols are rare
    c[support] = np.maximum(1, (rng.pareto(0.8, size=support.size) * 3).astype(np.uint64))
    N = int(c.sum())
    f = oracle_lib.normalize(c).astype(np.int64)
    assert f.sum() == 4096 and f[255] == 0
    assert np.array_equal(f[:255] > 0, c > 0)                       # present <=> f >= 1
    order = np.argsort(-c.astype(np.int64), kind="stable")          # more frequent never smaller
    fs = f[:255][order]
    cs = c[order]
    for i in range(254):
        if cs[i] > cs[i + 1]:
            assert fs[i] >= fs[i + 1]
    # every frequency stays within the repair budget of its exact share
    share = c.astype(np.float64) * 4096 / N
    budget = 255 + 1
    assert np.all(np.abs(f[:255] - share) <= budget)
