"""cg_encode_static: the encoder for callers that cannot allocate device memory
(a server that has reserved the whole GPU for its own pool, a plugin whose
enqueue step must not call cudaMalloc, a path that cannot take an allocation's
implicit synchronisation).  It must produce exactly what cg_encode produces
with a caller-provided workspace, call after call, although every call reuses
the same library-owned scratch block.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_compression_cachegen_b200 as cg

pytestmark = pytest.mark.gpu


def _inputs(L, H, D, T, seed):
    from kv_cache_compression_cachegen_b200 import synth
    kv = torch.empty((L, 2, T, H, D), dtype=torch.int16, device="cuda")
    synth.generate_gpu(kv, L, H, D, T, seed)
    return kv


def _encode_with_workspace(kv, C, level, nch, stride):
    L, _, T, H, D = kv.shape
    shape = cg.Shape(L, H, D)
    wsb = cg.cg_encode_workspace_bytes(shape, C, nch)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.zeros(stride * nch, dtype=torch.uint8, device="cuda")
    sizes = torch.zeros(nch, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cg.check(cg.cg_encode(shape, kv, T, 0, nch, C, level, None, out, stride, sizes, st, ws, wsb))
    return out, sizes, st


def _encode_static(kv, C, level, nch, stride):
    L, _, T, H, D = kv.shape
    shape = cg.Shape(L, H, D)
    out = torch.zeros(stride * nch, dtype=torch.uint8, device="cuda")
    sizes = torch.zeros(nch, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # through the C ABI directly (ctypes), no Python-side buffers beyond the outputs
    lib = cg.library()
    rc = lib.cg_encode_static(ctypes.byref(shape), ctypes.c_void_p(kv.data_ptr()), T, 0, nch, C,
                              level, None, ctypes.c_void_p(out.data_ptr()), stride,
                              ctypes.c_void_p(sizes.data_ptr()), ctypes.c_void_p(st.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    cg.check(rc, "cg_encode_static")
    return out, sizes, st


def test_static_scratch_encode_matches_workspace_encode_twice():
    cases = [((4, 2, 64, 256), 256, 1, 0), ((32, 2, 128, 1000), 512, 2, 7)]
    for (L, H, D, T), C, level, seed in cases:
        kv = _inputs(L, H, D, T, seed)
        nch = -(-T // C)
        stride = cg.cg_encoded_bound(cg.Shape(L, H, D), C)
        ref, rsz, rst = _encode_with_workspace(kv, C, level, nch, stride)
        for _ in range(2):  # two calls in a row reuse the same scratch block
            got, gsz, gst = _encode_static(kv, C, level, nch, stride)
            torch.cuda.synchronize()
            assert int(gst.item()) == 0 and int(rst.item()) == 0
            assert torch.equal(gsz, rsz)
            for k in range(nch):
                n = int(rsz[k])
                assert torch.equal(got[k * stride:k * stride + n], ref[k * stride:k * stride + n])


def test_static_scratch_rejects_oversized_requests():
    kv = _inputs(32, 8, 128, 1536, 1)
    shape = cg.Shape(32, 8, 128)
    stride = cg.cg_encoded_bound(shape, 1536)
    out = torch.zeros(stride, dtype=torch.uint8, device="cuda")
    sizes = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert cg.cg_encode_workspace_bytes(shape, 1536, 1) > (128 << 20)
    rc = cg.cg_encode_static(shape, kv, 1536, 0, 1, 1536, 1, None, out, stride, sizes, st)
    assert rc == cg.CG_ERR_CAPACITY
