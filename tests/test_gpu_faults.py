"""Corrupt or mismatched containers must come back as a status code from the
decoder, never as a fault: every read is bounds-checked against the container
and every write against the destination."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_cachegen_b200 import Shape
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu

L, H, D, T, C = 3, 2, 32, 64, 32


def _encoded():
    kv = gu.gen(L, H, D, T, seed=21)
    enc = ta.encode(kv, C, 1)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    return kv, enc


def _decode_status(buf: torch.Tensor, stride: int, level=1, chunk=C, nch=2, into=False, T_=T):
    shape = Shape(L, H, D)
    if into:
        kv = torch.zeros((L, 2, T_, H, D), dtype=torch.int16, device="cuda")
        st = ta.decode_into(buf, stride, shape, chunk, level, nch, kv)
    else:
        _, st = ta.decode(buf, stride, shape, chunk, level, nch)
    torch.cuda.synchronize()
    return ta.status_of(st)


def test_mismatches():
    _, enc = _encoded()
    assert _decode_status(enc.data, enc.stride, level=2) == oracle.MISMATCH
    assert _decode_status(enc.data, enc.stride, chunk=16, nch=1) == oracle.MISMATCH
    assert _decode_status(enc.data, enc.stride, into=True, T_=T - 1) == oracle.MISMATCH


def _padding_ranges(size0, secs):
    """Byte ranges of chunk 0's container that hold only zero padding: after the
    offsets array up to the payload, and after the payload up to total_bytes."""
    offs_end = secs[3] + 4 * (2 * L * C + 1)
    return [(offs_end, secs[4])]


def test_truncated_and_flipped_containers():
    _, enc = _encoded()
    size0 = int(enc.sizes[0])
    secs = oracle.sections(L, H, D, C)
    # a stride smaller than the container: header claims more bytes than readable
    small = enc.data[:enc.stride].clone()
    assert _decode_status(small[: (size0 // 16 - 1) * 16].clone(), (size0 // 16 - 1) * 16,
                          nch=1) == oracle.CORRUPT
    host0 = enc.data[:enc.stride].cpu().numpy()
    payload_bytes = int(host0[40:48].view(np.uint64)[0])
    pad = _padding_ranges(size0, secs) + [(secs[4] + payload_bytes, size0)]
    token_start = (32, 40)  # ignored by the chunk-slot decode (only cg_decode_into uses it)
    rng = np.random.default_rng(0)
    checked = {"header": 0, "freq": 0, "offsets": 0, "payload": 0}
    for region, lo, hi in (("header", 0, 64), ("freq", secs[2], secs[3]),
                           ("offsets", secs[3], secs[4]), ("payload", secs[4], size0)):
        for trial in range(10):
            buf = enc.data.clone()
            pos = int(rng.integers(lo, hi))
            bit = int(rng.integers(0, 8))
            buf[pos] ^= 1 << bit
            st = _decode_status(buf, enc.stride)
            in_pad = any(a <= pos < b for a, b in pad)
            if in_pad:
                assert st == 0, (region, pos, st)  # padding is not read
                continue
            checked[region] += 1
            if region == "header" and token_start[0] <= pos < token_start[1]:
                assert st == 0, (region, pos, st)
                # the same flip is caught by the full-KV decode when it moves the
                # chunk out of the cache, and is otherwise a valid other position
                continue
            if region == "payload":
                # the decoder's verdict on a damaged stream is the oracle's
                flipped = host0.copy()
                flipped[pos] ^= 1 << bit
                rc, *_ = oracle.decode_chunk(flipped, L, H, D, C, 1)
                assert (st == 0) == (rc == 0), (pos, bit, st, rc)
                assert st in (0, oracle.CORRUPT)
            else:
                # every header field but token_start, every frequency and every
                # offset is checked: a flip there is never decoded as valid
                assert st in (oracle.CORRUPT, oracle.MISMATCH), (region, pos, bit, st)
    assert min(checked.values()) >= 5, checked
    # garbage everywhere after the header
    buf = enc.data.clone()
    buf[64:] = torch.randint(0, 256, (buf.numel() - 64,), dtype=torch.uint8, device="cuda")
    assert _decode_status(buf, enc.stride) != 0
    # all-zero input
    assert _decode_status(torch.zeros_like(enc.data), enc.stride) == oracle.CORRUPT


def test_value_sections_are_not_checksummed():
    """A flip in the zero points or scales decodes with status 0 and changes the
    channel's values: the container carries no checksum, and the decoder checks
    structure (header, tables, offsets, stream ends), not values."""
    _, enc = _encoded()
    secs = oracle.sections(L, H, D, C)
    shape = Shape(L, H, D)
    ref, st = ta.decode(enc.data, enc.stride, shape, C, 1, 2)
    buf = enc.data.clone()
    buf[secs[0] + 4 * 5 + 2] ^= 0x40  # zp of channel 5 of (layer 0, K, head 0)
    out, st2 = ta.decode(buf, enc.stride, shape, C, 1, 2)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0 and ta.status_of(st2) == 0
    assert not torch.equal(out, ref)


def test_payload_flip_is_detected():
    _, enc = _encoded()
    secs = oracle.sections(L, H, D, C)
    buf = enc.data.clone()
    buf[secs[4] + 100] ^= 0x10
    assert _decode_status(buf, enc.stride) == oracle.CORRUPT
