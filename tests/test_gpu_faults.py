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


def test_truncated_and_flipped_containers():
    _, enc = _encoded()
    size0 = int(enc.sizes[0])
    secs = oracle.sections(L, H, D, C)
    # a stride smaller than the container: header claims more bytes than readable
    small = enc.data[:enc.stride].clone()
    assert _decode_status(small[: (size0 // 16 - 1) * 16].clone(), (size0 // 16 - 1) * 16,
                          nch=1) == oracle.CORRUPT
    rng = np.random.default_rng(0)
    for region, lo, hi in (("header", 0, 64), ("freq", secs[2], secs[3]),
                           ("offsets", secs[3], secs[4]), ("payload", secs[4], size0)):
        for trial in range(6):
            buf = enc.data.clone()
            pos = int(rng.integers(lo, hi))
            buf[pos] ^= int(1 << rng.integers(0, 8))
            st = _decode_status(buf, enc.stride)
            if region == "payload":
                assert st in (0, oracle.CORRUPT)
            else:
                assert st in (0, oracle.CORRUPT, oracle.MISMATCH), (region, pos, st)
    # garbage everywhere after the header
    buf = enc.data.clone()
    buf[64:] = torch.randint(0, 256, (buf.numel() - 64,), dtype=torch.uint8, device="cuda")
    assert _decode_status(buf, enc.stride) != 0
    # all-zero input
    assert _decode_status(torch.zeros_like(enc.data), enc.stride) == oracle.CORRUPT


def test_payload_flip_is_detected():
    _, enc = _encoded()
    secs = oracle.sections(L, H, D, C)
    buf = enc.data.clone()
    buf[secs[4] + 100] ^= 0x10
    assert _decode_status(buf, enc.stride) == oracle.CORRUPT
