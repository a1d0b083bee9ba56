"""cg_encode of two or more chunks runs its second half on the library's side
stream, forked from the caller's stream and joined back into it.  These tests
check that the split is invisible: the same bytes as one call per chunk, a
decode queued right after the encode on the same stream sees finished
containers, and CUDA graph capture works with the side stream in place and in
a fresh process where it does not exist yet (the call then runs on the
capturing stream alone)."""
import os
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest
import torch

import gpu_util as gu
from kv_cache_compression_cachegen_b200 import Shape
from kv_cache_compression_cachegen_b200 import torch_api as ta

pytestmark = pytest.mark.gpu
ROOT = Path(__file__).resolve().parents[1]


def _containers(enc: ta.Encoded) -> list[np.ndarray]:
    sizes = enc.sizes.cpu().tolist()
    data = enc.data.cpu().numpy()
    return [data[k * enc.stride:k * enc.stride + sizes[k]].copy() for k in range(enc.num_chunks)]


@pytest.mark.parametrize("adjacent", [False, True])
def test_two_halves_equal_one_call_per_chunk(adjacent):
    L, H, D, C = 4, 2, 64, 256
    T = 4 * C + 100  # five chunks, the last one ragged
    kv = gu.gen(L, H, D, T, seed=11)
    whole = _containers(ta.encode(kv, C, 1, adjacent=adjacent))
    torch.cuda.synchronize()
    nch = -(-T // C)
    assert len(whole) == nch
    for k in range(nch):
        one = ta.Encoder(Shape(L, H, D), C, 1, kv.device)
        e = one.encode(kv, 1, token_start=k * C, adjacent=adjacent)
        torch.cuda.synchronize()
        assert ta.status_of(e.status) == 0
        assert np.array_equal(_containers(e)[0], whole[k]), k


def test_decode_on_the_same_stream_sees_both_halves():
    L, H, D, C = 8, 8, 128, 1536
    T = 4 * C
    kv = gu.gen(L, H, D, T, seed=12)
    shape = Shape(L, H, D)
    ref_enc = ta.encode(kv, C, 1)
    torch.cuda.synchronize()
    ref = torch.empty_like(kv)
    st = ta.decode_into(ref_enc.data, ref_enc.stride, shape, C, 1, 4, ref)
    torch.cuda.synchronize()
    assert ta.status_of(st) == 0
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        enc = ta.Encoder(shape, C, 4, kv.device)
        out = torch.empty_like(kv)
        for _ in range(3):  # no synchronisation between the encode and the decode
            enc.out.zero_()
            out.zero_()
            e = enc.encode(kv, 1, stream=s)
            st2 = ta.decode_into(e.data, e.stride, shape, C, 1, 4, out, stream=s)
            s.synchronize()
            assert ta.status_of(e.status) == 0 and ta.status_of(st2) == 0
            assert torch.equal(out, ref)


def test_graph_capture_with_the_side_stream():
    L, H, D, C = 4, 4, 64, 512
    T = 3 * C + 7
    kv = gu.gen(L, H, D, T, seed=13)
    shape = Shape(L, H, D)
    enc = ta.Encoder(shape, C, -(-T // C), kv.device)
    eager = _containers(enc.encode(kv, 2))  # also creates the side stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        enc.encode(kv, 2)
    enc.out.zero_()
    enc.sizes.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert ta.status_of(enc.status) == 0
    got = _containers(ta.Encoded(enc.out, enc.sizes, enc.stride, enc.num_chunks, C, 2, shape,
                                 enc.status))
    assert all(np.array_equal(a, b) for a, b in zip(got, eager))
    del g


_FRESH = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import gpu_util as gu
from kv_cache_compression_cachegen_b200 import Shape
from kv_cache_compression_cachegen_b200 import torch_api as ta
L, H, D, C = 4, 4, 64, 512
T = 3 * C + 7
kv = gu.gen(L, H, D, T, seed=14)
shape = Shape(L, H, D)
enc = ta.Encoder(shape, C, -(-T // C), kv.device)
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):   # the first encode of the process: no side stream yet
    enc.encode(kv, 0)
g.replay()
torch.cuda.synchronize()
assert ta.status_of(enc.status) == 0
sizes = enc.sizes.cpu().tolist()
captured = [enc.out[k * enc.stride:k * enc.stride + sizes[k]].cpu().numpy() for k in range(len(sizes))]
ref = ta.encode(kv, C, 0)
torch.cuda.synchronize()
rs = ref.sizes.cpu().tolist()
eager = [ref.data[k * ref.stride:k * ref.stride + rs[k]].cpu().numpy() for k in range(len(rs))]
assert all(np.array_equal(a, b) for a, b in zip(captured, eager))
del g
print("fresh-capture-ok")
"""


def test_graph_capture_before_the_side_stream_exists():
    env = dict(os.environ)
    res = subprocess.run([sys.executable, "-c", _FRESH, str(ROOT)], capture_output=True,
                         text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "fresh-capture-ok" in res.stdout


def test_concurrent_calls_from_two_host_threads():
    # The side stream and its fork/join events are shared by every call on the
    # device: calls from two host threads on two streams must still produce
    # their own bytes (ctypes releases the GIL inside the C call).
    import threading
    L, H, D, C = 4, 4, 64, 256
    T = 3 * C + 40
    kvs = [gu.gen(L, H, D, T, seed=30 + i) for i in range(2)]
    shape = Shape(L, H, D)
    refs = []
    for kv in kvs:
        refs.append(_containers(ta.encode(kv, C, 1)))
        torch.cuda.synchronize()
    encs = [ta.Encoder(shape, C, -(-T // C), kvs[0].device) for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    errors = []

    def worker(i):
        try:
            with torch.cuda.stream(streams[i]):
                for _ in range(20):
                    encs[i].encode(kvs[i], 1, stream=streams[i])
            streams[i].synchronize()
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    for i in range(2):
        assert ta.status_of(encs[i].status) == 0
        got = _containers(ta.Encoded(encs[i].out, encs[i].sizes, encs[i].stride,
                                     encs[i].num_chunks, C, 1, shape, encs[i].status))
        assert all(np.array_equal(a, b) for a, b in zip(got, refs[i])), i
