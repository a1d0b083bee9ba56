"""The sender's level choice ([Practice] 2.2): thresholds at 5 and 1 Gbit/s,
read as >= 5 -> high, [1, 5) -> balanced, < 1 -> fast.  Host logic, no GPU."""
import pytest

from kv_cache_compression_cachegen_b200 import LEVELS
from kv_cache_compression_cachegen_b200 import streaming as st


@pytest.mark.parametrize("gbps,level", [
    (100.0, "high"), (5.0, "high"), (4.999, "balanced"), (2.5, "balanced"), (1.0, "balanced"),
    (0.999, "fast"), (0.1, "fast"), (0.0, "fast"),
])
def test_select_level_thresholds(gbps, level):
    assert st.select_level(gbps) == LEVELS[level]


def test_plan_follows_a_bandwidth_drop_and_recovery():
    # the page's example: a link falling from 5 Gbps to 100 Mbps, then recovering
    trace = [10, 5, 3, 1, 0.1, 0.1, 2, 6]
    assert st.plan_levels(trace) == [0, 0, 1, 1, 2, 2, 1, 0]
