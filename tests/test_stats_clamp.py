"""The clamp-rate measurement (stats.clamp_counts) against an exact count on a
small cache with outlier channels: a delta value is clamped when the rounded
quotient of its difference to the reconstructed anchor leaves [-127, 127]."""
from fractions import Fraction

import numpy as np
import torch

from exact import frac, rn_f32
from kv_cache_compression_cachegen_b200 import stats


def _exact_clamped(kv_h, zp, sc, sym, C, level, oracle_lib):
    L, _, T, H, D = kv_h.shape
    vals = kv_h.view(np.float16).astype(np.float32)
    count = 0
    for l in range(L):
        s = frac(oracle_lib.step(level, l, L))
        for k in range(2):
            for h in range(H):
                for d in range(D):
                    zpf, scf = frac(zp[l, k, h, d]), frac(sc[l, k, h, d])
                    for t0 in range(0, T, 10):
                        c = int(sym[l, k, t0, h, d]) - 127
                        ahat = frac(rn_f32(zpf + frac(rn_f32(c * scf))))
                        for t in range(t0 + 1, min(t0 + 10, T)):
                            y = frac(rn_f32(frac(rn_f32(frac(vals[l, k, t, h, d]) - ahat)) / s))
                            r = int(abs(y) + Fraction(1, 2))
                            count += r > 127
    return count


def test_clamp_counts_match_exact_count(oracle_lib):
    rng = np.random.default_rng(5)
    L, H, D, T = 3, 2, 16, 40
    x = rng.normal(0, 1, size=(L, 2, T, H, D)).cumsum(axis=2)
    x[:, :, :, 1, 3] *= 90.0     # an outlier channel whose deltas overflow 127 steps
    x[1, 0, 7, 0, 5] = 500.0     # one isolated spike on a delta token
    kv_h = x.astype(np.float16).view(np.uint16)
    level = 2
    rc, sym, zp, sc = oracle_lib.quantize_chunk(kv_h, 0, T, level)
    assert rc == 0
    rc, cont = oracle_lib.encode_chunk(kv_h, 0, T, level)
    rc2, out, n, _ = oracle_lib.decode_chunk(cont, L, H, D, T, level)
    assert rc == 0 and rc2 == 0
    want = _exact_clamped(kv_h, zp, sc, sym, T, level, oracle_lib)
    assert want > 0
    got, deltas = stats.clamp_counts(torch.from_numpy(kv_h.view(np.int16).copy()),
                                     torch.from_numpy(out.view(np.int16).copy()), T, level)
    assert got == want
    assert deltas == L * 2 * H * D * (T - 4)


def test_clamp_counts_zero_without_outliers(oracle_lib):
    rng = np.random.default_rng(6)
    L, H, D, T, C = 2, 1, 16, 45, 20
    kv_h = (rng.normal(0, 0.2, size=(L, 2, T, H, D)).cumsum(axis=2)).astype(np.float16)
    kv_h = kv_h.view(np.uint16)
    outs = []
    for k0 in range(0, T, C):
        rc, cont = oracle_lib.encode_chunk(kv_h, k0, C, 1)
        rc2, out, n, _ = oracle_lib.decode_chunk(cont, L, H, D, C, 1)
        assert rc == 0 and rc2 == 0
        outs.append(out)
    dec = np.concatenate(outs, axis=2)
    got, deltas = stats.clamp_counts(torch.from_numpy(kv_h.view(np.int16).copy()),
                                     torch.from_numpy(dec.view(np.int16).copy()), C, 1)
    assert got == 0
    # anchors at local tokens 0, 10 of each 20-token chunk (and 40 of the last)
    assert deltas == L * 2 * H * D * (T - 5)
