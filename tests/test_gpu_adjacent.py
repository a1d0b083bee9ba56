"""GPU parity of format 2 (deltas between adjacent tokens) through the C ABI:
containers byte-identical to the oracle's format 2, decoded fp16 bit-identical
(0 ULP) to the oracle's format-2 decode, for chunk slots and the full KV."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_cachegen_b200 import CG_ERR_MISMATCH, Shape, synth
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu


def _oracle_v2(kv_h, C, level, chunks):
    def one(k):
        rc, buf = oracle.encode_chunk(kv_h, k * C, C, level, adjacent=True)
        assert rc == 0, f"oracle encode chunk {k}: {rc}"
        return buf
    return dict(zip(chunks, gu.pmap(one, list(chunks))))


def _oracle_v2_decodes(containers, shape, C, level):
    L, H, D = shape.num_layers, shape.num_kv_heads, shape.head_dim

    def one(k):
        rc, vals, n, start = oracle.decode_chunk(containers[k], L, H, D, C, level, adjacent=True)
        assert rc == 0, f"oracle decode chunk {k}: {rc}"
        return vals
    keys = list(containers)
    return dict(zip(keys, gu.pmap(one, keys)))


def _parity(kv, C, level, chunks=None):
    L, _, T, H, D = kv.shape
    shape = Shape(L, H, D)
    nch = -(-T // C)
    chunks = list(range(nch)) if chunks is None else chunks
    enc = ta.encode(kv, C, level, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    ref = _oracle_v2(gu.host(kv), C, level, chunks)
    got = gu.gpu_containers(enc, chunks)
    for k in chunks:
        assert got[k].size == ref[k].size, f"chunk {k} size"
        assert np.array_equal(got[k], ref[k]), f"chunk {k} bytes differ"
    out, st = ta.decode(enc.data, enc.stride, shape, C, level, nch, adjacent=True)
    kv2 = torch.full_like(kv, 0x7E00)
    st2 = ta.decode_into(enc.data, enc.stride, shape, C, level, nch, kv2, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0 and ta.status_of(st2) == 0
    dref = _oracle_v2_decodes(ref, shape, C, level)
    for k in chunks:
        n = min(C, T - k * C)
        assert np.array_equal(gu.host(gu.chunk_slot(out, shape, C, k, n)), dref[k]), k
    for k in range(nch):
        n = min(C, T - k * C)
        assert torch.equal(kv2[:, :, k * C:k * C + n], gu.chunk_slot(out, shape, C, k, n))
    return enc


@pytest.mark.parametrize("level", [0, 1, 2])
def test_tiny_config_all_levels(level):
    kv = gu.gen(4, 2, 64, 256, seed=0)
    _parity(kv, 256, level)


@pytest.mark.parametrize("L,H,D,T,C", [
    (2, 1, 16, 20, 20),
    (2, 1, 16, 20, 16),
    (3, 2, 32, 45, 20),
    (1, 1, 16, 1, 8),
    (2, 1, 16, 9, 9),
    (5, 3, 48, 301, 128),
    (2, 4, 256, 37, 37),
    (2, 64, 16, 25, 10),
    (4, 5, 80, 333, 100),
    (1, 1, 16, 16384, 16384),
])
def test_ragged_shapes(L, H, D, T, C):
    for level in range(3):
        kv = gu.gen(L, H, D, T, seed=L * 1000 + T + level + 17, p_out=0.05)
        _parity(kv, C, level)


def test_degenerate_inputs():
    # constant layer (one-symbol tables in the symbol pass), a zero head,
    # clamping outliers that the chain has to walk back from
    L, H, D, T = 3, 2, 32, 50
    kv = gu.gen(L, H, D, T, seed=5, p_out=0.2, m_out=2000.0)
    kv[0] = torch.tensor(np.float16(0.5).view(np.int16), device="cuda")
    kv[1, 0, :, 1, :] = 0
    kv[2, 1, ::3, 0, :5] = torch.tensor(np.float16(6e4).view(np.int16), device="cuda")
    for level in range(3):
        _parity(kv.contiguous(), 20, level)


def test_mistral7b_shape_all_levels():
    kv = gu.gen(32, 8, 128, 1536, seed=1)
    for level in range(3):
        _parity(kv, 1536, level)


def test_llama2_7b_full_size_and_ratio():
    w = synth.WORKLOADS["llama2_7b"]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(w.L, w.H, w.D)
    nch = w.num_chunks
    enc2 = ta.encode(kv, w.C, 1, adjacent=True)
    out = torch.full_like(kv, 0x7E00)
    st = ta.decode_into(enc2.data, enc2.stride, shape, w.C, 1, nch, out, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(enc2.status) == 0 and ta.status_of(st) == 0
    sampled = [0, nch - 1]
    ref = _oracle_v2(gu.host(kv), w.C, 1, sampled)
    got = gu.gpu_containers(enc2, sampled)
    for k in sampled:
        assert np.array_equal(got[k], ref[k]), f"chunk {k} container differs"
    dref = _oracle_v2_decodes(ref, shape, w.C, 1)
    for k in sampled:
        assert np.array_equal(gu.host(out[:, :, k * w.C:(k + 1) * w.C]), dref[k]), k
    slots, st2 = ta.decode(enc2.data, enc2.stride, shape, w.C, 1, nch, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(st2) == 0
    for k in range(nch):
        assert torch.equal(out[:, :, k * w.C:(k + 1) * w.C],
                           gu.chunk_slot(slots, shape, w.C, k, w.C))
    # both formats are plausible compressions of this cache
    fp16 = kv.numel() * 2
    enc1 = ta.encode(kv, w.C, 1)
    torch.cuda.synchronize()
    r1, r2 = fp16 / int(enc1.sizes.sum()), fp16 / int(enc2.sizes.sum())
    assert 2.0 < r1 < 12.0 and 2.0 < r2 < 12.0, (r1, r2)


def test_formats_are_not_interchangeable():
    L, H, D, T, C = 2, 2, 32, 60, 30
    kv = gu.gen(L, H, D, T, seed=9)
    shape = Shape(L, H, D)
    e1 = ta.encode(kv, C, 1)
    e2 = ta.encode(kv, C, 1, adjacent=True)
    torch.cuda.synchronize()
    _, s12 = ta.decode(e1.data, e1.stride, shape, C, 1, 2, adjacent=True)
    _, s21 = ta.decode(e2.data, e2.stride, shape, C, 1, 2)
    torch.cuda.synchronize()
    assert ta.status_of(s12) == CG_ERR_MISMATCH
    assert ta.status_of(s21) == CG_ERR_MISMATCH
    # the anchor sections agree between the formats
    secs = oracle.sections(L, H, D, C)
    a = e1.data[:secs[2]].cpu().numpy()
    b = e2.data[:secs[2]].cpu().numpy()
    assert np.array_equal(a[secs[0]:], b[secs[0]:])


def test_corrupt_format2_containers_report_a_status():
    # both passes of the format-2 decode bound every read by the container and
    # every write by the destination: damage comes back as a status
    L, H, D, T, C = 3, 2, 32, 64, 32
    kv = gu.gen(L, H, D, T, seed=21)
    shape = Shape(L, H, D)
    enc = ta.encode(kv, C, 1, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    size0 = int(enc.sizes[0])
    secs = oracle.sections(L, H, D, C)

    def status(buf, stride, nch=2, into=False):
        if into:
            out = torch.zeros_like(kv)
            st = ta.decode_into(buf, stride, shape, C, 1, nch, out, adjacent=True)
        else:
            _, st = ta.decode(buf, stride, shape, C, 1, nch, adjacent=True)
        torch.cuda.synchronize()
        return ta.status_of(st)

    cut = (size0 // 16 - 1) * 16
    assert status(enc.data[:cut].clone(), cut, nch=1) == oracle.CORRUPT
    rng = np.random.default_rng(1)
    for lo, hi in ((0, 64), (secs[2], secs[3]), (secs[3], secs[4]), (secs[4], size0)):
        for _ in range(4):
            buf = enc.data.clone()
            buf[int(rng.integers(lo, hi))] ^= int(1 << rng.integers(0, 8))
            for into in (False, True):
                assert status(buf, enc.stride, into=into) in (0, oracle.CORRUPT,
                                                              oracle.MISMATCH)
    buf = enc.data.clone()
    buf[secs[4] + 100] ^= 0x10
    assert status(buf, enc.stride) == oracle.CORRUPT
    assert status(torch.zeros_like(enc.data), enc.stride, into=True) == oracle.CORRUPT


def test_format2_into_paged_pool():
    # Format-2 containers decoded into a paged pool through a shuffled block
    # table: every logical token's row equals the oracle's format-2 decode.
    L, H, D, T, C, P = 3, 2, 64, 250, 96, 16
    kv = gu.gen(L, H, D, T, seed=21)
    shape = Shape(L, H, D)
    nch = -(-T // C)
    enc = ta.encode(kv, C, 1, adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    npages_logical = -(-T // P)
    num_pages = npages_logical + 3
    g = torch.Generator().manual_seed(5)
    table = torch.randperm(num_pages, generator=g)[:npages_logical].to(torch.int32).cuda()
    pool = torch.full((L, 2, num_pages, P, H, D), 0x7E00, dtype=torch.int16, device="cuda")
    st = ta.decode_into_paged(enc.data, enc.stride, shape, C, 1, nch, pool, P, table, T,
                              adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    conts = gu.gpu_containers(enc, range(nch))
    dref = _oracle_v2_decodes(conts, shape, C, 1)
    logical = gu.host(pool[:, :, table.long()].reshape(L, 2, npages_logical * P, H, D))
    for k in range(nch):
        n = min(C, T - k * C)
        assert np.array_equal(logical[:, :, k * C:k * C + n], dref[k]), k
    tab = table.cpu().tolist()
    unused = sorted(set(range(num_pages)) - set(tab))
    assert bool((pool[:, :, unused] == 0x7E00).all())

    # Logical page 3 (tokens 48..63) unmapped: its rows are not written, the
    # call reports a mismatch, and the later tokens of the groups it cuts
    # (the group of tokens 60..69 continues on page 4) still decode exactly.
    bad = table.clone()
    bad[3] = num_pages
    pool2 = torch.full_like(pool, 0x7E00)
    st = ta.decode_into_paged(enc.data, enc.stride, shape, C, 1, nch, pool2, P, bad, T,
                              adjacent=True)
    torch.cuda.synchronize()
    assert ta.status_of(st) == CG_ERR_MISMATCH
    badtab = bad.cpu().tolist()
    for lp in range(npages_logical):
        a, b = lp * P, min(T, (lp + 1) * P)
        if lp == 3:
            continue
        assert torch.equal(pool2[:, :, badtab[lp], :b - a], pool[:, :, tab[lp], :b - a]), lp
    # the physical page logical page 3 used to map to was never written
    assert bool((pool2[:, :, tab[3]] == 0x7E00).all())
