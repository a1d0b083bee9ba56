"""GPU parity: libcachegen containers must equal the oracle's byte for byte and
decoded fp16 must equal the oracle's bit for bit (0 ULP), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_cachegen_b200 import CG_ERR_MISMATCH, Shape
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu


def _roundtrip_parity(kv, C, level, chunks=None, check_into=True, check_tables=True):
    L, _, T, H, D = kv.shape
    shape = Shape(L, H, D)
    nchunks = -(-T // C)
    chunks = list(range(nchunks)) if chunks is None else chunks
    enc = ta.encode(kv, C, level)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    kv_h = gu.host(kv)
    ref = gu.oracle_containers(kv_h, C, level, chunks)
    got = gu.gpu_containers(enc, chunks)
    for k in chunks:
        assert got[k].size == ref[k].size, f"chunk {k} size"
        assert np.array_equal(got[k], ref[k]), f"chunk {k} bytes differ"
    # decode the GPU's containers on the GPU, compare with the oracle's decode
    out, st = ta.decode(enc.data, enc.stride, shape, C, level, nchunks)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    dref = gu.oracle_decodes(ref, shape, C, level)
    for k in chunks:
        n = min(C, T - k * C)
        assert np.array_equal(gu.host(gu.chunk_slot(out, shape, C, k, n)), dref[k]), k
    if check_into:
        kv2 = torch.full_like(kv, 0x7E00)
        st = ta.decode_into(enc.data, enc.stride, shape, C, level, nchunks, kv2)
        torch.cuda.synchronize()
        assert ta.status_of(st) == 0
        for k in range(nchunks):
            n = min(C, T - k * C)
            assert torch.equal(kv2[:, :, k * C:k * C + n], gu.chunk_slot(out, shape, C, k, n))
    if check_tables:
        tables, tb, st = ta.build_tables(kv, C, level)
        torch.cuda.synchronize()
        assert ta.status_of(st) == 0
        secs = oracle.sections(L, H, D, 1)
        th = tables.cpu().numpy()
        for k in chunks:
            assert np.array_equal(th[k * tb:(k + 1) * tb], ref[k][64:secs[2] + L * 2 * H * 512])
        enc2 = ta.encode(kv, C, level, tables=tables)
        torch.cuda.synchronize()
        assert ta.status_of(enc2.status) == 0
        got2 = gu.gpu_containers(enc2, chunks)
        for k in chunks:
            assert np.array_equal(got2[k], ref[k])
    return enc


@pytest.mark.parametrize("level", [0, 1, 2])
def test_tiny_config_all_levels(level):
    kv = gu.gen(4, 2, 64, 256, seed=0)
    _roundtrip_parity(kv, 256, level)


RAGGED = [  # L, H, D, T, C
    (2, 1, 16, 20, 20),
    (2, 1, 16, 20, 16),
    (3, 2, 32, 45, 20),
    (1, 1, 16, 1, 8),
    (2, 1, 16, 9, 9),
    (5, 3, 48, 301, 128),
    (2, 4, 256, 37, 37),
    (2, 64, 16, 25, 10),
    (3, 2, 64, 300, 300),
    (2, 1, 16, 1000, 512),
    (4, 5, 80, 333, 100),
    # the implementation's maxima: chunk of 16,384 tokens; 1,024 layers;
    # 64 heads x head_dim 256 (streams of 16,384 symbols)
    (1, 1, 16, 16384, 16384),
    (1024, 1, 16, 12, 12),
    (1, 64, 256, 12, 12),
]


@pytest.mark.parametrize("L,H,D,T,C", RAGGED)
def test_ragged_shapes(L, H, D, T, C):
    for level in range(3):
        kv = gu.gen(L, H, D, T, seed=L * 1000 + T + level, p_out=0.05)
        _roundtrip_parity(kv, C, level)


@pytest.mark.parametrize("level", [0, 1, 2])
def test_mistral7b_shape_all_levels(level):
    kv = gu.gen(32, 8, 128, 1536, seed=1)
    _roundtrip_parity(kv, 1536, level)


def test_degenerate_inputs():
    # constant channels (scale 0), single-symbol heads, zeros, huge outliers (clamping)
    L, H, D, T = 3, 2, 32, 50
    kv = gu.gen(L, H, D, T, seed=5, p_out=0.2, m_out=2000.0)
    kv[0] = torch.tensor(np.float16(0.5).view(np.int16), device="cuda")   # whole layer constant
    kv[1, 0, :, 1, :] = 0                                                   # one head all zero
    kv[2, 1, ::3, 0, :5] = torch.tensor(np.float16(6e4).view(np.int16), device="cuda")
    for level in range(3):
        _roundtrip_parity(kv.contiguous(), 20, level)


def test_nonfinite_input_sets_status():
    kv = gu.gen(2, 1, 16, 40, seed=3)
    kv[1, 0, 17, 0, 3] = torch.tensor(np.uint16(0x7C00).view(np.int16), device="cuda")
    enc = ta.encode(kv, 40, 1)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == oracle.NONFINITE
    kv[1, 0, 17, 0, 3] = torch.tensor(np.uint16(0x7E01).view(np.int16), device="cuda")
    kv[1, 0, 10, 0, 3] = 0  # NaN on a delta token, not on an anchor
    enc = ta.encode(kv, 40, 1)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == oracle.NONFINITE


def test_supplied_tables_missing_symbol_is_mismatch():
    kv = gu.gen(2, 1, 16, 40, seed=3)
    tables, tb, st = ta.build_tables(torch.zeros_like(kv), 40, 1)
    enc = ta.encode(kv, 40, 1, tables=tables)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == CG_ERR_MISMATCH


def test_capacity_status():
    kv = gu.gen(2, 1, 16, 40, seed=3)
    shape = Shape(2, 1, 16)
    secs = oracle.sections(2, 1, 16, 40)
    enc = ta.encode(kv, 40, 1, out_stride=((secs[4] + 64) // 16) * 16)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == oracle.CAPACITY
    full = ta.encode(kv, 40, 1)
    torch.cuda.synchronize()
    assert int(enc.sizes[0]) == int(full.sizes[0])  # the required size is reported
    del shape


def test_destination_only_16_byte_aligned():
    # The decoder writes 32-byte pieces when the destination allows it and
    # 16-byte pieces otherwise; both must give the same bytes.
    L, H, D, T, C = 3, 2, 64, 250, 96
    kv = gu.gen(L, H, D, T, seed=11)
    shape = Shape(L, H, D)
    nch = -(-T // C)
    enc = ta.encode(kv, C, 1)
    ref, st = ta.decode(enc.data, enc.stride, shape, C, 1, nch)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    flat = torch.empty(ref.numel() + 8, dtype=torch.int16, device=kv.device)
    out = flat[8:]
    assert out.data_ptr() % 32 == 16
    out, st = ta.decode(enc.data, enc.stride, shape, C, 1, nch, out=out)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    for k in range(nch):  # the written part of each chunk slot
        n = min(C, T - k * C)
        assert torch.equal(gu.chunk_slot(out, shape, C, k, n), gu.chunk_slot(ref, shape, C, k, n))
    flat2 = torch.full((kv.numel() + 8,), 0x7E00, dtype=torch.int16, device=kv.device)
    kv2 = flat2[8:].view(kv.shape)
    assert kv2.data_ptr() % 32 == 16
    st = ta.decode_into(enc.data, enc.stride, shape, C, 1, nch, kv2)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    for k in range(nch):
        n = min(C, T - k * C)
        assert torch.equal(kv2[:, :, k * C:k * C + n], gu.chunk_slot(ref, shape, C, k, n))


def test_decode_into_paged_pool():
    # A shuffled block table: decoding into the paged pool must put every token's
    # row exactly where the flat decode_into puts it, page by page.
    L, H, D, T, C, P = 3, 2, 64, 250, 96, 16
    kv = gu.gen(L, H, D, T, seed=13)
    shape = Shape(L, H, D)
    nch = -(-T // C)
    enc = ta.encode(kv, C, 2)
    flat = torch.full_like(kv, 0x7E00)
    st = ta.decode_into(enc.data, enc.stride, shape, C, 2, nch, flat)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    npages_logical = -(-T // P)
    num_pages = npages_logical + 5
    g = torch.Generator().manual_seed(3)
    table = torch.randperm(num_pages, generator=g)[:npages_logical].to(torch.int32).cuda()
    pool = torch.full((L, 2, num_pages, P, H, D), 0x7E00, dtype=torch.int16, device="cuda")
    st = ta.decode_into_paged(enc.data, enc.stride, shape, C, 2, nch, pool, P, table, T)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    tab = table.cpu().tolist()
    for lp in range(npages_logical):
        a, b = lp * P, min(T, (lp + 1) * P)
        assert torch.equal(pool[:, :, tab[lp], :b - a], flat[:, :, a:b]), lp
    # every logical token's row also equals the oracle's decode of its chunk
    conts = gu.gpu_containers(enc, range(nch))
    dref = gu.oracle_decodes(conts, shape, C, 2)
    logical = gu.host(pool[:, :, table.long()].reshape(L, 2, npages_logical * P, H, D))
    for k in range(nch):
        n = min(C, T - k * C)
        assert np.array_equal(logical[:, :, k * C:k * C + n], dref[k]), k
    # pages no logical page maps to stay untouched
    unused = sorted(set(range(num_pages)) - set(tab))
    assert bool((pool[:, :, unused] == 0x7E00).all())
    # a block-table entry outside the pool is a mismatch
    bad = table.clone()
    bad[2] = num_pages
    st = ta.decode_into_paged(enc.data, enc.stride, shape, C, 2, nch, pool, P, bad, T)
    torch.cuda.synchronize()
    assert ta.status_of(st) == CG_ERR_MISMATCH
