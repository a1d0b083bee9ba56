"""GPU parity on inputs built to sit on the rounding decisions.

The cache below carries, channel by channel, the cases pinned on the CPU in
tests/test_oracle_rounding.py:
  * delta quotients that a rounded reciprocal would put on the other side of a
    half-integer (2.25 at step 0.3 -> 7, 9.0 at step 1.2 -> 7, ...): the
    quantiser's fast path cannot decide them and must fall back to the
    IEEE division;
  * exact half-step ties at the balanced level (0.25 at step 0.5 -> 1, 63.75
    -> 127.5 -> clamped to 127);
  * anchor codes of realistic channels on both sides of a half;
  * reconstructions where one rounding and two roundings give different fp16
    (a = 20, q = -25 at step 0.8: +0 with two roundings, -5 * 2^-24 with one).
Containers must equal the oracle's byte for byte and decoded fp16 bit for bit,
at all three levels, and the decoded values of the pinned cases must be the
pinned ones.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_cachegen_b200 import Shape
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu

L, H, D, T, C = 3, 2, 16, 30, 30   # three layers: one per third; anchors at tokens 0, 10, 20

NEAR_HALF_03 = [2.25, -2.25, 3.75, 8.25, 15.75, 17.25, 18.75, 29.25, 30.75]
NEAR_HALF_12 = [9.0, 15.0, 33.0, 63.0, 69.0, 75.0, 117.0, 123.0, -9.0]
TIES_05 = [0.25, -0.25, 0.75, -0.75, 1.25, -1.25, 63.75, -63.75, 64.0]


def _crafted_cache() -> np.ndarray:
    rng = np.random.default_rng(7)
    kv = (rng.normal(0.0, 1.0, size=(L, 2, T, H, D)).cumsum(axis=2) * 0.4).astype(np.float32)
    for l in range(L):
        for k in range(2):
            c = kv[l, k, :, 0, :]
            # ch 0: constant anchors 0; the deltas are the near-half quotients
            c[:, 0] = 0.0
            for g in range(3):
                c[10 * g + 1:10 * g + 10, 0] = NEAR_HALF_03 if l != 2 else NEAR_HALF_12
            # ch 1-3: constant anchors 20 / 36 / 64 with delta tokens 0 -> q = -25 / -45 / -80
            # at step 0.8, whose two-rounding value is +0
            for ch, a in ((1, 20.0), (2, 36.0), (3, 64.0)):
                c[:, ch] = a
                c[[3, 14, 27], ch] = 0.0
            # ch 4: exact half-step ties at step 0.5
            c[:, 4] = 0.0
            for g in range(3):
                c[10 * g + 1:10 * g + 10, 4] = TIES_05
            # ch 5: anchors whose code IEEE division puts at 64 and a reciprocal at 63
            c[[0, 10, 20], 5] = [-7.68359375, 4.46484375, 1.427734375]
            # ch 6: an anchor (-0.021484375, code -41) whose reconstruction differs
            # in fp16 between one and two roundings
            c[[0, 10, 20], 6] = [-3.90625, 7.62890625, -0.021484375]
            # ch 7: constant anchors 2.046875, deltas at q = -55 for step 1.2
            c[:, 7] = 2.046875
            c[[1, 11, 21], 7] = -63.96875
    return kv.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("level", [0, 1, 2])
def test_rounding_cases_match_oracle(level):
    kv_h = _crafted_cache()
    kv = torch.from_numpy(kv_h.view(np.int16).copy()).cuda()
    shape = Shape(L, H, D)
    enc = ta.encode(kv, C, level)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    ref = gu.oracle_containers(kv_h, C, level, [0])
    got = gu.gpu_containers(enc, [0])
    assert np.array_equal(got[0], ref[0])
    out, st = ta.decode(enc.data, enc.stride, shape, C, level, 1)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    dref = gu.oracle_decodes(ref, shape, C, level)
    vals = gu.host(gu.chunk_slot(out, shape, C, 0, T))
    assert np.array_equal(vals, dref[0])
    if level == 0:
        # high level: step 0.3 (layer 0), 0.8 (layer 1), 1.2 (layer 2)
        for k in range(2):
            # q = -25 / -45 / -80 at step 0.8 reconstruct to +0 exactly
            for ch in (1, 2, 3):
                assert (vals[1, k, [3, 14, 27], 0, ch] == 0x0000).all()
            # 2.25 / 0.3f -> code 7 -> fp16(RN(7 * 0.3f))
            assert vals[0, k, 1, 0, 0] == np.float16(np.float32(7) * np.float32(0.3)).view(np.uint16)
            assert vals[2, k, 1, 0, 0] == np.float16(np.float32(7) * np.float32(1.2)).view(np.uint16)
    if level == 1:
        # 0.25 at step 0.5 is a tie -> 1 -> 0.5; 63.75 -> 127.5 -> clamp 127 -> 63.5
        assert vals[0, 0, 1, 0, 4] == np.float16(0.5).view(np.uint16)
        assert vals[0, 0, 7, 0, 4] == np.float16(63.5).view(np.uint16)
