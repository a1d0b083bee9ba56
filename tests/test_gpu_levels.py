"""cg_encode_levels: the three versions of every chunk ([Practice] 2.1) from one
quantiser pass.  Each level's containers must be byte for byte those of
cg_encode at that level, and hence the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_cachegen_b200 import CG_ERR_CAPACITY, Shape, synth
from kv_cache_compression_cachegen_b200 import torch_api as ta

import gpu_util as gu

pytestmark = pytest.mark.gpu


def _levels_vs_single(kv, C, token_start=0, num_chunks=None, oracle_chunks=()):
    L, _, T, H, D = kv.shape
    views = ta.encode_levels(kv, C, token_start=token_start, num_chunks=num_chunks)
    torch.cuda.synchronize()
    assert ta.status_of(views[0].status) == 0
    nch = views[0].num_chunks
    kv_h = gu.host(kv) if oracle_chunks else None
    for level in range(3):
        single = ta.encode(kv, C, level, token_start=token_start, num_chunks=nch)
        torch.cuda.synchronize()
        assert ta.status_of(single.status) == 0
        assert torch.equal(views[level].sizes, single.sizes), f"level {level} sizes"
        got = gu.gpu_containers(views[level], range(nch))
        ref = gu.gpu_containers(single, range(nch))
        for k in range(nch):
            assert np.array_equal(got[k], ref[k]), f"level {level} chunk {k}"
        if oracle_chunks:
            want = {}
            for k in oracle_chunks:
                rc, buf = oracle.encode_chunk(kv_h, token_start + k * C, C, level)
                assert rc == 0
                want[k] = buf
            for k in oracle_chunks:
                assert np.array_equal(got[k], want[k]), f"level {level} chunk {k} vs oracle"
    return views


def test_tiny_config_levels_vs_oracle():
    kv = gu.gen(4, 2, 64, 256, seed=0)
    _levels_vs_single(kv, 256, oracle_chunks=[0])


@pytest.mark.parametrize("L,H,D,T,C", [
    (2, 1, 16, 20, 20),
    (2, 1, 16, 20, 16),
    (3, 2, 32, 45, 20),
    (1, 1, 16, 1, 8),
    (5, 3, 48, 301, 128),
    (2, 4, 256, 37, 37),
    (2, 64, 16, 25, 10),
    (4, 5, 80, 333, 100),
])
def test_ragged_shapes_levels(L, H, D, T, C):
    kv = gu.gen(L, H, D, T, seed=7 * L + T, p_out=0.05)
    nch = -(-T // C)
    _levels_vs_single(kv, C, oracle_chunks=[0, nch - 1])


def test_degenerate_inputs_levels():
    L, H, D, T = 3, 2, 32, 50
    kv = gu.gen(L, H, D, T, seed=5, p_out=0.2, m_out=2000.0)
    kv[0] = torch.tensor(np.float16(0.5).view(np.int16), device="cuda")
    kv[1, 0, :, 1, :] = 0
    kv[2, 1, ::3, 0, :5] = torch.tensor(np.float16(6e4).view(np.int16), device="cuda")
    _levels_vs_single(kv.contiguous(), 20, oracle_chunks=[0, 2])


def test_mistral7b_shape_levels():
    kv = gu.gen(32, 8, 128, 3072, seed=1)
    _levels_vs_single(kv, 1536, oracle_chunks=[1])


def test_llama34b_batch_levels_full_size():
    """One 13-chunk batch of the Llama-34B-shaped pre-encode at full size,
    from a token offset inside the cache."""
    w = synth.WORKLOADS["llama34b"]
    kv = gu.gen(w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    _levels_vs_single(kv, w.C, token_start=13 * w.C, num_chunks=13, oracle_chunks=[12])


def test_levels_decode_round_trip():
    L, H, D, T, C = 4, 2, 64, 700, 256
    kv = gu.gen(L, H, D, T, seed=11)
    shape = Shape(L, H, D)
    views = ta.encode_levels(kv, C)
    nch = views[0].num_chunks
    for level in range(3):
        out = torch.full_like(kv, 0x7E00)
        st = ta.decode_into(views[level].data, views[level].stride, shape, C, level, nch, out)
        torch.cuda.synchronize()
        assert ta.status_of(st) == 0
        ref = gu.oracle_decodes(gu.gpu_containers(views[level], range(nch)), shape, C, level)
        for k in range(nch):
            n = min(C, T - k * C)
            assert np.array_equal(gu.host(out[:, :, k * C:k * C + n]), ref[k]), (level, k)


def test_levels_nonfinite_and_capacity():
    kv = gu.gen(2, 1, 16, 40, seed=3)
    kv[1, 0, 17, 0, 3] = torch.tensor(np.uint16(0x7C00).view(np.int16), device="cuda")
    views = ta.encode_levels(kv, 40)
    torch.cuda.synchronize()
    assert ta.status_of(views[0].status) == oracle.NONFINITE
    kv = gu.gen(2, 1, 16, 40, seed=3)
    secs = oracle.sections(2, 1, 16, 40)
    small = ((secs[4] + 64) // 16) * 16
    views = ta.encode_levels(kv, 40, out_stride=small)
    full = ta.encode_levels(kv, 40)
    torch.cuda.synchronize()
    assert ta.status_of(views[0].status) == CG_ERR_CAPACITY
    for level in range(3):  # the required sizes are reported
        assert torch.equal(views[level].sizes, full[level].sizes)
