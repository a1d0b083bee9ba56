"""TEST INFRASTRUCTURE ONLY: ctypes wrapper of the plain CPU oracle.

The oracle (cachegen_oracle.c) is a slow, single-threaded C restatement of the
CacheGen codec, written from the pages' description and the readings fixed in
include/cachegen.h.  It shares no code with the CUDA library.  Only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package; the library and its Python binding never do.
"""
from __future__ import annotations

import ctypes
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SOURCE = HERE / "cachegen_oracle.c"
HEADER = HERE / "cachegen_oracle.h"
LIBPATH = HERE / "liboracle.so"
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]

OK, INVALID, CAPACITY, CORRUPT, MISMATCH, NONFINITE = 0, 1, 2, 3, 4, 5


def build(force: bool = False) -> Path:
    stale = (not LIBPATH.exists() or LIBPATH.stat().st_mtime < SOURCE.stat().st_mtime
             or LIBPATH.stat().st_mtime < HEADER.stat().st_mtime)
    if force or stale:
        subprocess.run(["gcc", *CFLAGS, "-o", str(LIBPATH), str(SOURCE), "-lm"], check=True,
                       cwd=HERE)
    return LIBPATH


_lib = None
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")
_c = ctypes


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(LIBPATH))
        sig = {
            "orc_f16_to_f32": (_c.c_float, [_c.c_uint16]),
            "orc_f32_to_f16": (_c.c_uint16, [_c.c_float]),
            "orc_f32_to_f16_array": (None, [_f32p, _u16p, _c.c_int64]),
            "orc_f16_to_f32_array": (None, [_u16p, _f32p, _c.c_int64]),
            "orc_layer_third": (_c.c_int, [_c.c_int, _c.c_int]),
            "orc_step": (_c.c_float, [_c.c_int, _c.c_int, _c.c_int]),
            "orc_anchor_params": (None, [_f32p, _c.c_int, _c.POINTER(_c.c_float),
                                         _c.POINTER(_c.c_float)]),
            "orc_anchor_code": (_c.c_int, [_c.c_float, _c.c_float, _c.c_float]),
            "orc_anchor_value": (_c.c_float, [_c.c_int, _c.c_float, _c.c_float]),
            "orc_delta_code": (_c.c_int, [_c.c_float, _c.c_float, _c.c_float]),
            "orc_delta_value": (_c.c_float, [_c.c_int, _c.c_float, _c.c_float]),
            "orc_normalize": (None, [_u32p, _c.c_uint64, _u16p]),
            "orc_rans_encode": (_c.c_int64, [_u8p, _c.c_int, _c.c_int, _u16p, _u16p,
                                             _c.c_int64]),
            "orc_rans_decode": (_c.c_int, [_u16p, _c.c_int64, _c.c_int, _c.c_int, _u16p, _u8p]),
            "orc_sections": (None, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _u64p]),
            "orc_encoded_bound": (_c.c_uint64, [_c.c_int, _c.c_int, _c.c_int, _c.c_int]),
            "orc_quantize_chunk": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _u16p, _c.c_int64,
                                              _c.c_int64, _c.c_int, _c.c_int, _u8p, _f32p,
                                              _f32p]),
            "orc_tables_of": (None, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _u8p, _u16p]),
            "orc_encode_chunk": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _u16p, _c.c_int64,
                                            _c.c_int64, _c.c_int, _c.c_int, _u8p, _c.c_uint64,
                                            _c.POINTER(_c.c_uint64)]),
            "orc_decode_chunk": (_c.c_int, [_u8p, _c.c_uint64, _c.c_int, _c.c_int, _c.c_int,
                                            _c.c_int, _c.c_int, _u16p, _c.c_uint64,
                                            _c.POINTER(_c.c_int64), _c.POINTER(_c.c_int64)]),
            "orc_quantize_chunk_v": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _u16p, _c.c_int64,
                                                _c.c_int64, _c.c_int, _c.c_int, _c.c_int, _u8p,
                                                _f32p, _f32p]),
            "orc_encode_chunk_v": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _u16p, _c.c_int64,
                                              _c.c_int64, _c.c_int, _c.c_int, _c.c_int, _u8p,
                                              _c.c_uint64, _c.POINTER(_c.c_uint64)]),
            "orc_decode_chunk_v": (_c.c_int, [_u8p, _c.c_uint64, _c.c_int, _c.c_int, _c.c_int,
                                              _c.c_int, _c.c_int, _c.c_int, _u16p, _c.c_uint64,
                                              _c.POINTER(_c.c_int64), _c.POINTER(_c.c_int64)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---- fp16 -------------------------------------------------------------------
def f32_to_f16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, dtype=np.uint16)
    lib().orc_f32_to_f16_array(x, out, x.size)
    return out


def f16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16).ravel()
    out = np.empty(h.size, dtype=np.float32)
    lib().orc_f16_to_f32_array(h, out, h.size)
    return out


# ---- quantiser ----------------------------------------------------------------
def layer_third(l: int, L: int) -> int:
    return lib().orc_layer_third(l, L)


def step(level: int, l: int, L: int) -> np.float32:
    return np.float32(lib().orc_step(level, l, L))


def anchor_params(anchors) -> tuple[np.float32, np.float32]:
    a = np.ascontiguousarray(anchors, dtype=np.float32)
    zp, sc = _c.c_float(), _c.c_float()
    lib().orc_anchor_params(a, a.size, _c.byref(zp), _c.byref(sc))
    return np.float32(zp.value), np.float32(sc.value)


def anchor_code(x, zp, scale) -> int:
    return lib().orc_anchor_code(float(np.float32(x)), float(np.float32(zp)),
                                 float(np.float32(scale)))


def anchor_value(c: int, zp, scale) -> np.float32:
    return np.float32(lib().orc_anchor_value(int(c), float(np.float32(zp)),
                                             float(np.float32(scale))))


def delta_code(x, ahat, step_) -> int:
    return lib().orc_delta_code(float(np.float32(x)), float(np.float32(ahat)),
                                float(np.float32(step_)))


def delta_value(q: int, ahat, step_) -> np.float32:
    return np.float32(lib().orc_delta_value(int(q), float(np.float32(ahat)),
                                            float(np.float32(step_))))


# ---- tables and rANS ----------------------------------------------------------
def normalize(counts, total: int | None = None) -> np.ndarray:
    c = np.zeros(255, dtype=np.uint32)
    src = np.asarray(counts, dtype=np.uint64)
    c[: src.size] = src
    if total is None:
        total = int(src.sum())
    f = np.zeros(256, dtype=np.uint16)
    lib().orc_normalize(c, total, f)
    return f


def rans_encode(sym, per_table: int, freq) -> np.ndarray:
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    fq = np.ascontiguousarray(freq, dtype=np.uint16)
    cap = s.size + 2
    words = np.zeros(cap, dtype=np.uint16)
    m = lib().orc_rans_encode(s, s.size, per_table, fq, words, cap)
    if m < 0:
        raise ValueError(f"orc_rans_encode failed ({m})")
    return words[:m].copy()


def rans_decode(words, nsym: int, per_table: int, freq) -> tuple[int, np.ndarray]:
    w = np.ascontiguousarray(words, dtype=np.uint16)
    if w.size == 0:
        w = np.zeros(1, dtype=np.uint16)[:0]
    fq = np.ascontiguousarray(freq, dtype=np.uint16)
    sym = np.zeros(nsym, dtype=np.uint8)
    rc = lib().orc_rans_decode(np.ascontiguousarray(w), w.size, nsym, per_table, fq, sym)
    return rc, sym


# ---- container ----------------------------------------------------------------
def sections(L: int, H: int, D: int, n: int) -> list[int]:
    offs = np.zeros(5, dtype=np.uint64)
    lib().orc_sections(L, H, D, n, offs)
    return [int(v) for v in offs]


def encoded_bound(L: int, H: int, D: int, C: int) -> int:
    return int(lib().orc_encoded_bound(L, H, D, C))


def quantize_chunk(kv: np.ndarray, token_start: int, C: int, level: int,
                   adjacent: bool = False):
    """kv: uint16 [L, 2, T, H, D].  Returns (status, sym [L,2,n,H,D], zp, scale).
    adjacent=True: format 2, deltas to the previous token's reconstruction."""
    L, _, T, H, D = kv.shape
    n = min(C, T - token_start)
    sym = np.zeros((L, 2, n, H, D), dtype=np.uint8)
    zp = np.zeros((L, 2, H, D), dtype=np.float32)
    sc = np.zeros((L, 2, H, D), dtype=np.float32)
    rc = lib().orc_quantize_chunk_v(L, H, D, np.ascontiguousarray(kv, dtype=np.uint16), T,
                                    token_start, C, level, int(adjacent), sym, zp, sc)
    return rc, sym, zp, sc


def tables_of(sym: np.ndarray) -> np.ndarray:
    L, _, n, H, D = sym.shape
    freq = np.zeros((L, 2, H, 256), dtype=np.uint16)
    lib().orc_tables_of(L, H, D, n, np.ascontiguousarray(sym), freq)
    return freq


def encode_chunk(kv: np.ndarray, token_start: int, C: int, level: int,
                 adjacent: bool = False):
    """Returns (status, container bytes as uint8 array); adjacent=True writes
    format 2 (header version 2)."""
    L, _, T, H, D = kv.shape
    cap = encoded_bound(L, H, D, C)
    out = np.zeros(cap, dtype=np.uint8)
    size = _c.c_uint64(0)
    rc = lib().orc_encode_chunk_v(L, H, D, np.ascontiguousarray(kv, dtype=np.uint16), T,
                                  token_start, C, level, int(adjacent), out, cap,
                                  _c.byref(size))
    return rc, out[: size.value].copy()


def decode_chunk(container, L: int, H: int, D: int, C: int, level: int,
                 adjacent: bool = False):
    """Returns (status, values uint16 [L,2,n,H,D], n, token_start).  The
    container's format must be the one asked for (else MISMATCH)."""
    buf = np.ascontiguousarray(container, dtype=np.uint8)
    out = np.zeros(L * 2 * C * H * D, dtype=np.uint16)
    n, start = _c.c_int64(0), _c.c_int64(0)
    rc = lib().orc_decode_chunk_v(buf, buf.size, L, H, D, C, level, int(adjacent), out,
                                  out.size, _c.byref(n), _c.byref(start))
    vals = out[: L * 2 * n.value * H * D].reshape(L, 2, n.value, H, D) if rc == OK else out[:0]
    return rc, vals, n.value, start.value
