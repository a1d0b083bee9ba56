"""Pins of the layer-dependent step table and the thirds map.

The values come from tests/golden/steps.txt, which copies the numbers printed in
"CacheGen实战：KV缓存压缩与流式传输在大型语言模型服务中的高效应用" section 3.1.
"""
from pathlib import Path

import numpy as np
import pytest

GOLDEN = Path(__file__).with_name("golden") / "steps.txt"


def _golden():
    rows = {}
    for line in GOLDEN.read_text(encoding="utf-8").splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lvl, *vals = line.split()
        rows[int(lvl)] = [np.float32(v) for v in vals]
    return rows


def test_golden_has_three_levels():
    g = _golden()
    assert sorted(g) == [0, 1, 2]
    assert all(len(v) == 3 for v in g.values())


@pytest.mark.parametrize("L", [2, 3, 4, 32, 48, 80])
def test_step_per_layer_matches_printed_table(oracle_lib, L):
    g = _golden()
    for level in range(3):
        for l in range(L):
            third = (3 * l) // L
            assert oracle_lib.step(level, l, L) == g[level][third]


def test_thirds_of_the_configs(oracle_lib):
    # 32 layers: 11 / 11 / 10; 48 layers: 16 each; 4 layers: {0,0,1,2}; 2 layers: {0,1}.
    def counts(L):
        t = [oracle_lib.layer_third(l, L) for l in range(L)]
        return [t.count(k) for k in range(3)], t
    assert counts(32)[0] == [11, 11, 10]
    assert counts(48)[0] == [16, 16, 16]
    assert counts(4)[1] == [0, 0, 1, 2]
    assert counts(2)[1] == [0, 1]


def test_shallow_layers_get_the_finer_step(oracle_lib):
    # [Practice] section 1: shallow layers are more sensitive (0.5 shallow, 1.5 deep).
    for level in range(3):
        s = [oracle_lib.step(level, l, 32) for l in range(32)]
        assert all(a <= b for a, b in zip(s, s[1:]))
        assert s[0] < s[-1]
    assert oracle_lib.step(1, 0, 32) == np.float32(0.5)
    assert oracle_lib.step(1, 31, 32) == np.float32(1.5)
