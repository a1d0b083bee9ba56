"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: every chunk is encoded and decoded on the GPU in one call; sampled
chunks are compared byte for byte / bit for bit with the oracle, and every
chunk is checked against properties that hold at any size (a clean status,
decode_into equal to the per-chunk decode, the streamed pipeline equal to the
batched decode)."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_cachegen_b200 import Shape, synth
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu


def _compare_sampled(kv, enc, C, level, chunks):
    L, _, T, H, D = kv.shape
    shape = Shape(L, H, D)
    kv_h = gu.host(kv)
    ref = gu.oracle_containers(kv_h, C, level, chunks)
    got = gu.gpu_containers(enc, chunks)
    for k in chunks:
        assert np.array_equal(got[k], ref[k]), f"chunk {k} container differs"
    dref = gu.oracle_decodes(ref, shape, C, level)
    return dref


def test_llama2_7b_full_size():
    w = synth.WORKLOADS["llama2_7b"]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(w.L, w.H, w.D)
    nch = w.num_chunks
    enc = ta.encode(kv, w.C, 1)
    out = torch.full_like(kv, 0x7E00)
    st = ta.decode_into(enc.data, enc.stride, shape, w.C, 1, nch, out)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0 and ta.status_of(st) == 0
    ratio = kv.numel() * 2 / int(enc.sizes.sum())
    assert 2.0 < ratio < 12.0
    sampled = [0, nch - 1]
    dref = _compare_sampled(kv, enc, w.C, 1, sampled)
    for k in sampled:
        got = gu.host(out[:, :, k * w.C:(k + 1) * w.C])
        assert np.array_equal(got, dref[k]), f"chunk {k} decode differs"
    # every chunk: decode_into equals the per-chunk decode
    slots, st2 = ta.decode(enc.data, enc.stride, shape, w.C, 1, nch)
    torch.cuda.synchronize()
    assert ta.status_of(st2) == 0
    for k in range(nch):
        assert torch.equal(out[:, :, k * w.C:(k + 1) * w.C],
                           gu.chunk_slot(slots, shape, w.C, k, w.C))


def test_llama2_7b_paged_pool_full_size():
    """The bench workload decoded into a pool of 16-token pages through a shuffled
    block table: every logical token's row equals the flat cg_decode_into."""
    w = synth.WORKLOADS["llama2_7b"]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(w.L, w.H, w.D)
    nch, P = w.num_chunks, 16
    enc = ta.encode(kv, w.C, 1)
    flat = torch.full_like(kv, 0x7E00)
    st = ta.decode_into(enc.data, enc.stride, shape, w.C, 1, nch, flat)
    npages = -(-w.T // P) + 3
    table = torch.randperm(npages, generator=torch.Generator().manual_seed(5))
    table = table[:-(-w.T // P)].to(torch.int32).cuda()
    pool = torch.full((w.L, 2, npages, P, w.H, w.D), 0x7E00, dtype=torch.int16, device="cuda")
    st2 = ta.decode_into_paged(enc.data, enc.stride, shape, w.C, 1, nch, pool, P, table, w.T)
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0 and ta.status_of(st) == 0 and ta.status_of(st2) == 0
    logical = pool[:, :, table.long()].reshape(w.L, 2, table.numel() * P, w.H, w.D)
    assert torch.equal(logical[:, :, :w.T], flat)
    unused = sorted(set(range(npages)) - set(table.cpu().tolist()))
    assert bool((pool[:, :, unused] == 0x7E00).all())
    # sampled chunks of the pool's logical view against the oracle's decode
    sampled = [0, 3, nch - 1]
    dref = gu.oracle_decodes(gu.gpu_containers(enc, sampled), shape, w.C, 1)
    for k in sampled:
        got = gu.host(logical[:, :, k * w.C:(k + 1) * w.C])
        assert np.array_equal(got, dref[k]), f"chunk {k} paged decode differs from the oracle"


def test_llama34b_streamed_decode_with_level_schedule():
    """Pre-encode every chunk at the three levels, keep the containers in pinned
    host memory, then decode chunk by chunk with cg_decode_into on one stream while
    a second stream copies the next chunk's container to the device."""
    w = synth.WORKLOADS["llama34b"]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(w.L, w.H, w.D)
    nch = w.num_chunks
    sched = synth.level_schedule(nch, w.seed)
    host = {}
    batch = 13
    for level in range(3):
        for k0 in range(0, nch, batch):
            nb = min(batch, nch - k0)
            enc = ta.encode(kv, w.C, level, token_start=k0 * w.C, num_chunks=nb)
            torch.cuda.synchronize()
            assert ta.status_of(enc.status) == 0
            sizes = enc.sizes.cpu().tolist()
            for j in range(nb):
                buf = torch.empty(sizes[j], dtype=torch.uint8, pin_memory=True)
                buf.copy_(enc.data[j * enc.stride:j * enc.stride + sizes[j]])
                host[(level, k0 + j)] = buf
            if level == 1 and k0 == 0:  # sampled oracle parity: two chunks of the balanced set
                dref = _compare_sampled(kv, enc, w.C, level, [0, 5])
    # streamed decode following the per-chunk level schedule
    out = torch.full_like(kv, 0x7E00)
    status = ta.new_status(kv.device)
    comp, copy = torch.cuda.Stream(), torch.cuda.Stream()
    maxb = max(b.numel() for b in host.values())
    stage = [torch.empty(((maxb + 15) // 16) * 16, dtype=torch.uint8, device="cuda")
             for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    for k in range(nch):
        s = k % 2
        buf = host[(sched[k], k)]
        with torch.cuda.stream(copy):
            copy.wait_event(done[s])
            stage[s][:buf.numel()].copy_(buf, non_blocking=True)
            ready[s].record(copy)
        comp.wait_event(ready[s])
        ta.decode_into(stage[s], stage[s].numel(), shape, w.C, sched[k], 1, out, status,
                       stream=comp)
        done[s].record(comp)
    torch.cuda.synchronize()
    assert ta.status_of(status) == 0
    # each streamed chunk equals the batched decode of the same level's containers
    for level in range(3):
        ks = [k for k in range(nch) if sched[k] == level][:4]
        for k in ks:
            buf = host[(level, k)].cuda()
            slot, st = ta.decode(buf, buf.numel(), shape, w.C, level, 1)
            torch.cuda.synchronize()
            assert ta.status_of(st) == 0
            assert torch.equal(out[:, :, k * w.C:(k + 1) * w.C],
                               gu.chunk_slot(slot, shape, w.C, 0, w.C))
    if sched[0] == 1:
        assert np.array_equal(gu.host(out[:, :, :w.C]), dref[0])


@pytest.mark.parametrize("dist", ["sweep_smooth", "sweep_rough"])
def test_chunk_size_and_distribution_sweep(dist):
    w = synth.WORKLOADS[dist]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(w.L, w.H, w.D)
    for C in w.chunk_sizes:
        nch = -(-w.T // C)
        for level in range(3):
            enc = ta.encode(kv, C, level)
            out = torch.full_like(kv, 0x7E00)
            st = ta.decode_into(enc.data, enc.stride, shape, C, level, nch, out)
            torch.cuda.synchronize()
            assert ta.status_of(enc.status) == 0 and ta.status_of(st) == 0
            last = nch - 1  # ragged tail for C = 1536 (32768 = 21 * 1536 + 512)
            dref = _compare_sampled(kv, enc, C, level, [last])
            n = w.T - last * C
            assert np.array_equal(gu.host(out[:, :, last * C:last * C + n]), dref[last])


def test_bandwidth_adaptive_stream_decode():
    """Three versions per chunk, a bandwidth trace picks each chunk's version, the
    chunks stream in (copy of the next overlapping the decode of the current),
    and every chunk equals the decode of the version that was sent."""
    from kv_cache_compression_cachegen_b200 import streaming
    L, H, D, C = 4, 2, 64, 256
    T = 7 * C + 100
    kv = gu.gen(L, H, D, T, seed=21)
    shape = Shape(L, H, D)
    store = streaming.encode_all_levels(kv, C)
    trace = [8.0, 3.0, 0.5, 6.0, 1.0, 0.2, 4.0, 9.0]
    levels = streaming.plan_levels(trace)
    assert len(levels) == store.num_chunks
    out = torch.full_like(kv, 0x7E00)
    status = streaming.stream_decode(store, levels, out)
    torch.cuda.synchronize()
    assert ta.status_of(status) == 0
    for k in range(store.num_chunks):
        buf = store.containers[(levels[k], k)].cuda()
        slot, st = ta.decode(buf, buf.numel(), shape, C, levels[k], 1)
        torch.cuda.synchronize()
        assert ta.status_of(st) == 0
        n = min(C, T - k * C)
        assert torch.equal(out[:, :, k * C:k * C + n], gu.chunk_slot(slot, shape, C, 0, n))
    # every streamed chunk equals the oracle's decode of the container that was
    # sent, and every sent container is the oracle's encoding of that chunk
    kv_h = gu.host(kv)
    got_all = gu.host(out)

    def check(k):
        lvl = levels[k]
        rc, ref = oracle.encode_chunk(kv_h, k * C, C, lvl)
        assert rc == 0
        sent = store.containers[(lvl, k)].numpy()
        assert np.array_equal(sent[:ref.size], ref) and not sent[ref.size:].any(), k
        rc, vals, n, start = oracle.decode_chunk(ref, L, H, D, C, lvl)
        assert rc == 0 and start == k * C
        assert np.array_equal(got_all[:, :, k * C:k * C + n], vals), k
    gu.pmap(check, list(range(store.num_chunks)))


def test_stream_decode_on_a_side_stream():
    """stream_decode given a stream other than the current one: its staging
    buffers are released while the side stream still uses them, and the
    current stream immediately allocates and overwrites memory; the decoded
    cache must still equal the decode on the current stream."""
    from kv_cache_compression_cachegen_b200 import streaming
    L, H, D, C = 4, 2, 64, 256
    T = 5 * C + 37
    kv = gu.gen(L, H, D, T, seed=23)
    store = streaming.encode_all_levels(kv, C)
    levels = streaming.plan_levels([6.0, 2.0, 0.3, 7.0, 1.5, 0.8])
    assert len(levels) == store.num_chunks
    ref = torch.full_like(kv, 0x7E00)
    st = streaming.stream_decode(store, levels, ref)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    side = torch.cuda.Stream()
    out = torch.full_like(kv, 0x7E00)
    torch.cuda.synchronize()
    st2 = streaming.stream_decode(store, levels, out, stream=side)
    # churn the current stream's allocator while the side stream works
    junk = [torch.full((store.size(levels[k], k),), 0xAB, dtype=torch.uint8, device="cuda")
            for k in range(store.num_chunks) for _ in range(4)]
    del junk
    side.synchronize()
    torch.cuda.synchronize()
    assert ta.status_of(st2) == 0
    assert torch.equal(out, ref)
