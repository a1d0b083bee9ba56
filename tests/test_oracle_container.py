"""Pins of the oracle's container: section arithmetic, header, offsets, streams,
error statuses, the reconstruction error bound and the entropy bound."""
import math
import struct

import numpy as np
import pytest

from kv_cache_compression_cachegen_b200 import synth


def test_sections_by_hand(oracle_lib):
    # L=1, H=1, D=16, n=10: 32 channels -> zp [64,192), scale [192,320), freq 2 tables
    # of 512 B [320,1344), 21 offsets [1344,1428) padded to 1440 = payload.
    assert oracle_lib.sections(1, 1, 16, 10) == [64, 192, 320, 1344, 1440]


def _header(buf):
    f = struct.unpack_from("<4sHBBIIIIIIQQQQ", bytes(buf[:64]))
    keys = ["magic", "version", "level", "group", "L", "H", "D", "C", "n", "prob_bits",
            "token_start", "payload", "total", "reserved"]
    return dict(zip(keys, f))


@pytest.mark.parametrize("T,C,t0", [(256, 256, 0), (23, 16, 16), (45, 20, 40), (1, 8, 0)])
def test_container_structure(oracle_lib, T, C, t0):
    L, H, D = 3, 2, 16
    kv = synth.generate_cpu(L, H, D, T, seed=T + C)
    rc, cont = oracle_lib.encode_chunk(kv, t0, C, 1)
    assert rc == 0
    n = min(C, T - t0)
    h = _header(cont)
    assert h["magic"] == b"CGK1" and h["version"] == 1 and h["level"] == 1 and h["group"] == 10
    assert (h["L"], h["H"], h["D"], h["C"], h["n"], h["prob_bits"]) == (L, H, D, C, n, 12)
    assert h["token_start"] == t0 and h["reserved"] == 0
    secs = oracle_lib.sections(L, H, D, n)
    assert h["total"] == cont.size == ((secs[4] + h["payload"] + 15) // 16) * 16
    assert not cont[secs[4] + h["payload"]:].any()                 # trailing padding is zero
    offs = np.frombuffer(cont[secs[3]:secs[3] + 4 * (2 * L * n + 1)].tobytes(), np.uint32)
    assert offs[0] == 0 and offs[-1] == h["payload"] and np.all(np.diff(offs.astype(np.int64)) >= 4)
    assert not cont[secs[3] + 4 * (2 * L * n + 1):secs[4]].any()   # offsets padding is zero
    rc, sym, zp, sc = oracle_lib.quantize_chunk(kv, t0, C, 1)
    assert np.array_equal(np.frombuffer(cont[secs[0]:secs[1]].tobytes(), np.float32), zp.ravel())
    assert np.array_equal(np.frombuffer(cont[secs[1]:secs[2]].tobytes(), np.float32), sc.ravel())
    freq = np.frombuffer(cont[secs[2]:secs[3]].tobytes(), np.uint16).reshape(L, 2, H, 256)
    assert np.array_equal(freq, oracle_lib.tables_of(sym))
    payload = cont[secs[4]:secs[4] + h["payload"]]
    for l in range(L):
        for k in range(2):
            for t in range(n):
                s = (l * 2 + k) * n + t
                words = np.frombuffer(payload[offs[s]:offs[s + 1]].tobytes(), np.uint16)
                rc, got = oracle_lib.rans_decode(words, H * D, D, freq[l, k])
                assert rc == 0 and np.array_equal(got, sym[l, k, t].ravel())


def test_nonfinite_input_is_rejected(oracle_lib):
    kv = synth.generate_cpu(2, 1, 16, 30, seed=9)
    for bad in (0x7C00, 0xFC00, 0x7E00):
        k2 = kv.copy()
        k2[1, 0, 17, 0, 5] = bad
        assert oracle_lib.encode_chunk(k2, 0, 30, 0)[0] == oracle_lib.NONFINITE


def test_decode_status_codes(oracle_lib):
    L, H, D, T = 2, 1, 16, 40
    kv = synth.generate_cpu(L, H, D, T, seed=4)
    rc, cont = oracle_lib.encode_chunk(kv, 0, 40, 2)
    assert rc == 0
    dec = oracle_lib.decode_chunk
    assert dec(cont, L, H, D, 40, 1)[0] == oracle_lib.MISMATCH      # wrong level
    assert dec(cont, L, H, D, 32, 2)[0] == oracle_lib.MISMATCH      # wrong chunk size
    assert dec(cont, L, 2, D, 40, 2)[0] == oracle_lib.MISMATCH      # wrong shape
    assert dec(cont[:-16], L, H, D, 40, 2)[0] == oracle_lib.CORRUPT  # truncated
    bad = cont.copy()
    bad[0] ^= 1
    assert dec(bad, L, H, D, 40, 2)[0] == oracle_lib.CORRUPT         # magic
    secs = oracle_lib.sections(L, H, D, 40)
    bad = cont.copy()
    bad[secs[4] + 40] ^= 0x10                                          # a payload bit
    assert dec(bad, L, H, D, 40, 2)[0] == oracle_lib.CORRUPT
    bad = cont.copy()
    bad[secs[2]] ^= 1                                                   # freq table sum != 4096
    assert dec(bad, L, H, D, 40, 2)[0] == oracle_lib.CORRUPT


@pytest.mark.parametrize("level", [0, 1, 2])
def test_reconstruction_error_bound(oracle_lib, level):
    # For unclamped deltas |x - xhat| <= s/2 (+ the fp32 roundings) + half an fp16 ulp of
    # xhat; the anchor's own error does not enter because deltas are coded against the
    # reconstructed anchor.  Anchors: |x - xhat| <= scale/2 (+ roundings) + half an ulp.
    L, H, D, T = 4, 2, 64, 256
    kv = synth.generate_cpu(L, H, D, T, seed=0)
    rc, cont = oracle_lib.encode_chunk(kv, 0, 256, level)
    assert rc == 0
    rc, out, n, _ = oracle_lib.decode_chunk(cont, L, H, D, 256, level)
    rc2, sym, zp, sc = oracle_lib.quantize_chunk(kv, 0, 256, level)
    x = kv.view(np.float16).astype(np.float64)
    xh = out.view(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(out.view(np.float16))).astype(np.float64)
    err = np.abs(x - xh)
    q = sym.astype(np.int64) - 127
    anchor = np.zeros(T, bool)
    anchor[::10] = True
    for l in range(L):
        s = float(oracle_lib.step(level, l, L))
        e, u, qq = err[l][:, ~anchor], ulp[l][:, ~anchor], q[l][:, ~anchor]
        unclamped = np.abs(qq) < 127
        bound = s / 2 * (1 + 1e-5) + 0.5 * u + 1e-6 * np.abs(x[l][:, ~anchor])
        assert np.all(e[unclamped] <= bound[unclamped])
        ea, ua = err[l][:, anchor], ulp[l][:, anchor]
        scl = sc[l][:, None, :, :]
        assert np.all(ea <= scl / 2 * (1 + 1e-5) + 0.5 * ua + 1e-6 * np.abs(x[l][:, anchor]))


def test_payload_within_one_percent_of_table_entropy(oracle_lib):
    L, H, D, T = 4, 8, 128, 1536
    kv = synth.generate_cpu(L, H, D, T, seed=1)
    rc, cont = oracle_lib.encode_chunk(kv, 0, T, 1)
    assert rc == 0
    rc, sym, _, _ = oracle_lib.quantize_chunk(kv, 0, T, 1)
    freq = oracle_lib.tables_of(sym).astype(np.float64)
    # information content of every symbol under its (l, kv, h) table
    f = np.take_along_axis(freq[:, :, None, :, :].repeat(T, axis=2),
                           sym.astype(np.int64).reshape(L, 2, T, H, D), axis=4)
    info = float(np.sum(-np.log2(f / 4096.0)))
    payload = struct.unpack_from("<Q", bytes(cont[40:48]))[0]
    streams = L * 2 * T
    assert 8 * payload <= 1.01 * info + 48 * streams
    assert 8 * payload >= info  # no code beats the model's entropy
