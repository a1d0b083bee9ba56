"""Seeded synthetic fp16 KV caches: the inputs of the tests and the benchmark.

This module holds none of the codec's arithmetic.  It draws per-channel AR(1)
random walks with log-normal channel scales and a fraction of outlier
channels -- smooth along tokens, as the KV caches the CacheGen pages describe
("adjacent tokens are as similar as consecutive video frames": [Practice] 1 of
"CacheGen实战：KV缓存压缩与流式传输在大型语言模型服务中的高效应用") -- with the
shapes of the workloads below.  No dataset or trained model is involved.

Definition (the CUDA kernel in kvsynth.cu computes the same thing):
  key = (seed mod 2^32, seed div 2^32); channel ch = ((l*2 + kv)*H + h)*D + d
  Philox4x32-10 (Salmon et al., SC'11) at counter (ch, k, 0, tag):
    tag 1, k = 0: amplitude = exp(0.5 z) * (u3 < p_out ? m_out : 1)
    tag 2, k    : normals e_{2k}, e_{2k+1} (Box-Muller)
  u1 = (r0 + 1) 2^-32, u2 = r1 2^-32, u3 = r2 2^-32
  rad = sqrt(-2 ln u1); z0 = rad cos(2 pi u2); z1 = rad sin(2 pi u2)
  x_0 = e_0, x_t = rho x_{t-1} + sigma e_t, sigma = sqrt(1 - rho^2)
  kv[l][kv][t][h][d] = fp16_rn(amplitude * x_t)      (fp64 throughout)
The two implementations agree except where the platforms' fp64 log/cos/sin
differ by an ulp near an fp16 rounding boundary; tests that compare the codec
with the oracle always feed both the very same buffer.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass, field
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_LIB = _HERE / "libkvsynth.so"

M0, M1 = 0xD2511F53, 0xCD9E8D57
W0, W1 = 0x9E3779B9, 0xBB67AE85
_MASK = 0xFFFFFFFF
_TWO_M32 = 2.0 ** -32
_TWO_PI = 6.283185307179586


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox4x32 with 10 rounds; returns four uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK for c in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    k0, k1 = np.uint64(k0 & _MASK), np.uint64(k1 & _MASK)
    m0, m1, mask = np.uint64(M0), np.uint64(M1), np.uint64(_MASK)
    s32 = np.uint64(32)
    for _ in range(10):
        p0 = c0 * m0
        p1 = c2 * m1
        c0, c1, c2, c3 = ((p1 >> s32) ^ c1 ^ k0, p1 & mask, (p0 >> s32) ^ c3 ^ k1, p0 & mask)
        k0 = (k0 + np.uint64(W0)) & mask
        k1 = (k1 + np.uint64(W1)) & mask
    return tuple(np.asarray(c, dtype=np.uint32) for c in (c0, c1, c2, c3))


def _key(seed: int) -> tuple[int, int]:
    return seed & _MASK, (seed >> 32) & _MASK


def _box_muller(a, b):
    u1 = (a.astype(np.float64) + 1.0) * _TWO_M32
    u2 = b.astype(np.float64) * _TWO_M32
    rad = np.sqrt(-2.0 * np.log(u1))
    th = _TWO_PI * u2
    return rad * np.cos(th), rad * np.sin(th)


def generate_cpu(L: int, H: int, D: int, T: int, seed: int, rho: float = 0.95,
                 p_out: float = 0.01, m_out: float = 8.0) -> np.ndarray:
    """The KV cache as a uint16 (fp16 bits) array of shape [L, 2, T, H, D]."""
    k0, k1 = _key(seed)
    chans = L * 2 * H * D
    ch = np.arange(chans, dtype=np.uint64)
    r = philox4x32_10(ch, 0, 0, 1, k0, k1)
    z, _ = _box_muller(r[0], r[1])
    u3 = r[2].astype(np.float64) * _TWO_M32
    amp = np.exp(0.5 * z) * np.where(u3 < p_out, m_out, 1.0)
    sigma = math.sqrt(1.0 - rho * rho)
    out = np.empty((T, chans), dtype=np.float16)
    x = None
    for k in range((T + 1) // 2):
        r = philox4x32_10(ch, k, 0, 2, k0, k1)
        e0, e1 = _box_muller(r[0], r[1])
        t = 2 * k
        x = e0 if t == 0 else rho * x + sigma * e0
        out[t] = (amp * x).astype(np.float16)
        if t + 1 < T:
            x = rho * x + sigma * e1
            out[t + 1] = (amp * x).astype(np.float16)
    out = out.reshape(T, L * 2, H * D).transpose(1, 0, 2).reshape(L, 2, T, H, D)
    return np.ascontiguousarray(out).view(np.uint16)


def _load():
    if not _LIB.exists():
        raise RuntimeError(f"{_LIB.name} is not built; run "
                           "kv_cache_compression_cachegen_b200.build.build_all()")
    lib = ctypes.CDLL(str(_LIB))
    lib.kvsynth_generate.restype = ctypes.c_int
    lib.kvsynth_generate.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int64, ctypes.c_uint64, ctypes.c_double,
                                     ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
    return lib


_lib = None


def generate_gpu(out, L: int, H: int, D: int, T: int, seed: int, rho: float = 0.95,
                 p_out: float = 0.01, m_out: float = 8.0, stream=None) -> None:
    """Fill `out` (a CUDA tensor of L*2*T*H*D 16-bit elements) on its device."""
    global _lib
    if _lib is None:
        _lib = _load()
    import torch
    if out.numel() != L * 2 * T * H * D or out.element_size() != 2 or not out.is_cuda:
        raise ValueError("out must be a CUDA tensor of L*2*T*H*D 16-bit elements")
    s = stream if stream is not None else torch.cuda.current_stream(out.device)
    rc = _lib.kvsynth_generate(ctypes.c_void_p(out.data_ptr()), L, H, D, T, seed, rho, p_out,
                               m_out, ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"kvsynth_generate failed ({rc})")


def level_schedule(num_chunks: int, seed: int) -> list[int]:
    """Per-chunk level drawn uniformly from {0, 1, 2}: Philox counter (k, 0, 0, 3)."""
    k0, k1 = _key(seed)
    r = philox4x32_10(np.arange(num_chunks, dtype=np.uint64), 0, 0, 3, k0, k1)
    return [int(v) % 3 for v in r[0]]


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: KV shape, sequence, chunking, generator knobs."""
    name: str
    L: int
    H: int
    D: int
    T: int
    C: int
    seed: int
    rho: float = 0.95
    p_out: float = 0.01
    m_out: float = 8.0
    levels: tuple = (0, 1, 2)
    chunk_sizes: tuple = field(default=())

    @property
    def num_chunks(self) -> int:
        return -(-self.T // self.C)

    @property
    def fp16_bytes(self) -> int:
        return self.L * 2 * self.T * self.H * self.D * 2


# The workloads the CacheGen pages describe, as synthetic stand-ins: a tiny
# case, a Mistral-7B-shaped GQA cache in one 1.5K chunk, a Llama-2-7B-shaped
# MHA cache of 10.5K tokens in seven chunks, a Llama-34B-shaped GQA cache of
# 78K tokens streamed chunk by chunk, and a chunk-size / distribution sweep.
WORKLOADS = {
    "tiny": Workload("tiny", 4, 2, 64, 256, 256, seed=0, levels=(1,)),
    "mistral7b": Workload("mistral7b", 32, 8, 128, 1536, 1536, seed=1),
    "llama2_7b": Workload("llama2_7b", 32, 32, 128, 10752, 1536, seed=2, levels=(1,)),
    "llama34b": Workload("llama34b", 48, 8, 128, 79872, 1536, seed=3, rho=0.97),
    "sweep_smooth": Workload("sweep_smooth", 32, 8, 128, 32768, 1536, seed=4,
                             chunk_sizes=(512, 1024, 1536, 2048)),
    "sweep_rough": Workload("sweep_rough", 32, 8, 128, 32768, 1536, seed=4, rho=0.8,
                            p_out=0.05, m_out=16.0, chunk_sizes=(512, 1024, 1536, 2048)),
}
