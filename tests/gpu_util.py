"""Helpers shared by the GPU parity tests: device inputs, host copies, and
threaded oracle calls (ctypes releases the GIL, so oracle chunks run in parallel)."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from kv_cache_compression_cachegen_b200 import Shape, synth
from kv_cache_compression_cachegen_b200 import torch_api as ta

THREADS = max(1, min(32, (os.cpu_count() or 2)))


def gen(L, H, D, T, seed, rho=0.95, p_out=0.01, m_out=8.0) -> torch.Tensor:
    kv = torch.empty(L * 2 * T * H * D, dtype=torch.int16, device="cuda")
    synth.generate_gpu(kv, L, H, D, T, seed, rho, p_out, m_out)
    return kv.view(L, 2, T, H, D)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint16)


def pmap(fn, items):
    with ThreadPoolExecutor(THREADS) as ex:
        return list(ex.map(fn, items))


def oracle_containers(kv_h: np.ndarray, C: int, level: int, chunks):
    def one(k):
        rc, buf = oracle.encode_chunk(kv_h, k * C, C, level)
        assert rc == 0, f"oracle encode chunk {k}: {rc}"
        return buf
    return dict(zip(chunks, pmap(one, list(chunks))))


def oracle_decodes(containers: dict, shape: Shape, C: int, level: int):
    L, H, D = shape.num_layers, shape.num_kv_heads, shape.head_dim

    def one(k):
        rc, vals, n, start = oracle.decode_chunk(containers[k], L, H, D, C, level)
        assert rc == 0, f"oracle decode chunk {k}: {rc}"
        return vals
    keys = list(containers)
    return dict(zip(keys, pmap(one, keys)))


def gpu_containers(enc: ta.Encoded, chunks):
    sizes = enc.sizes.cpu().numpy()
    out = {}
    for k in chunks:
        out[k] = enc.data[k * enc.stride:k * enc.stride + int(sizes[k])].cpu().numpy()
    return out


def chunk_slot(out: torch.Tensor, shape: Shape, C: int, k: int, n: int) -> torch.Tensor:
    L, H, D = shape.num_layers, shape.num_kv_heads, shape.head_dim
    slot = L * 2 * C * H * D
    return out[k * slot:k * slot + L * 2 * n * H * D].view(L, 2, n, H, D)
