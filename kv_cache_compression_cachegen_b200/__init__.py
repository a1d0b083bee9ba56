"""kv_cache_compression_cachegen_b200 -- Python binding of libcachegen.

libcachegen is a CUDA (sm_100a) implementation of the CacheGen KV-cache codec;
its C ABI and the exact format are documented in include/cachegen.h.  This
module only marshals arguments: every function here has the C name, takes
device tensors (or raw integer pointers) and a CUDA stream, and returns the
library's status code.  All device work runs in the library's kernels; there
is no Python or CPU implementation of the codec in this package, and calling
any function without the built library raises immediately.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

__all__ = [
    "CG_OK", "CG_ERR_INVALID_ARG", "CG_ERR_CAPACITY", "CG_ERR_CORRUPT", "CG_ERR_MISMATCH",
    "CG_ERR_NONFINITE", "CG_ERR_CUDA", "CG_ERR_UNSUPPORTED", "LEVELS", "CacheGenError",
    "Shape", "library", "library_path", "check", "cg_status_string", "cg_section_offsets",
    "cg_encoded_bound", "cg_tables_bytes", "cg_encode_workspace_bytes", "cg_build_tables",
    "cg_encode", "cg_encode_static", "cg_encode_levels", "cg_encode_levels_workspace_bytes",
    "cg_encode_adjacent", "cg_decode_adjacent", "cg_decode_adjacent_into", "cg_decode_adjacent_into_paged", "cg_decode", "cg_decode_into", "cg_decode_into_paged",
]

CG_OK, CG_ERR_INVALID_ARG, CG_ERR_CAPACITY, CG_ERR_CORRUPT = 0, 1, 2, 3
CG_ERR_MISMATCH, CG_ERR_NONFINITE, CG_ERR_CUDA, CG_ERR_UNSUPPORTED = 4, 5, 6, 7
LEVELS = {"high": 0, "balanced": 1, "fast": 2}

_PKG = Path(__file__).resolve().parent


def library_path() -> Path:
    return _PKG / "libcachegen.so"


class CacheGenError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {cg_status_string(status)} ({status})" if what
                         else f"{cg_status_string(status)} ({status})")


class Shape(ctypes.Structure):
    """cg_shape: (num_layers, num_kv_heads, head_dim)."""
    _fields_ = [("num_layers", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32)]

    def __init__(self, L: int, H: int, D: int):
        super().__init__(L, H, D)

    def __repr__(self) -> str:
        return f"Shape(L={self.num_layers}, H={self.num_kv_heads}, D={self.head_dim})"


_P = ctypes.c_void_p
_SIGNATURES = {
    "cg_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "cg_section_offsets": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_uint64)]),
    "cg_encoded_bound": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.c_int32,
                                        ctypes.POINTER(ctypes.c_uint64)]),
    "cg_tables_bytes": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_uint64)]),
    "cg_encode_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.c_int32,
                                                 ctypes.c_int32,
                                                 ctypes.POINTER(ctypes.c_uint64)]),
    "cg_build_tables": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int, _P, _P, _P, ctypes.c_uint64, _P]),
    "cg_encode": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_int32, ctypes.c_int32, ctypes.c_int, _P, _P,
                                 ctypes.c_uint64, _P, _P, _P, ctypes.c_uint64, _P]),
    "cg_encode_static": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int, _P, _P, ctypes.c_uint64, _P, _P, _P]),
    "cg_encode_levels_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.c_int32,
                                                        ctypes.c_int32,
                                                        ctypes.POINTER(ctypes.c_uint64)]),
    "cg_encode_levels": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P,
                                        ctypes.c_uint64, _P, _P, _P, ctypes.c_uint64, _P]),
    "cg_encode_adjacent": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int, _P, ctypes.c_uint64, _P, _P, _P,
                                          ctypes.c_uint64, _P]),
    "cg_decode_adjacent": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int, _P,
                                          ctypes.c_uint64, _P, _P]),
    "cg_decode_adjacent_into": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64,
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_int, _P,
                                               ctypes.c_int64, _P, _P]),
    "cg_decode": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64, ctypes.c_int32,
                                 ctypes.c_int32, ctypes.c_int, _P, ctypes.c_uint64, _P, _P]),
    "cg_decode_into": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int, _P,
                                      ctypes.c_int64, _P, _P]),
    "cg_decode_into_paged": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_int, _P,
                                            ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int64,
                                            _P, _P]),
    "cg_decode_adjacent_into_paged": (ctypes.c_int, [ctypes.POINTER(Shape), _P, ctypes.c_uint64,
                                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_int,
                                                     _P, ctypes.c_int32, ctypes.c_int32, _P,
                                                     ctypes.c_int64, _P, _P]),
}

_lib = None


def library() -> ctypes.CDLL:
    """Load libcachegen.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not path.exists():
            raise RuntimeError(f"{path} is not built; run "
                               "`python -m kv_cache_compression_cachegen_b200.build`")
        lib = ctypes.CDLL(str(path))
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x) -> ctypes.c_void_p:
    if x is None:
        return ctypes.c_void_p(0)
    if isinstance(x, int):
        return ctypes.c_void_p(x)
    return ctypes.c_void_p(x.data_ptr())


def _stream(s) -> ctypes.c_void_p:
    if s is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return ctypes.c_void_p(s)
    return ctypes.c_void_p(s.cuda_stream)


def _shape(shape) -> Shape:
    return shape if isinstance(shape, Shape) else Shape(*shape)


def check(status: int, what: str = "") -> None:
    """Raise CacheGenError unless status == CG_OK."""
    if status != CG_OK:
        raise CacheGenError(status, what)


def cg_status_string(status: int) -> str:
    return library().cg_status_string(int(status)).decode()


def cg_section_offsets(shape, n_tokens: int) -> list[int]:
    arr = (ctypes.c_uint64 * 5)()
    check(library().cg_section_offsets(ctypes.byref(_shape(shape)), n_tokens, arr),
          "cg_section_offsets")
    return list(arr)


def _size_query(name: str, *args) -> int:
    out = ctypes.c_uint64(0)
    check(getattr(library(), name)(*args, ctypes.byref(out)), name)
    return out.value


def cg_encoded_bound(shape, chunk_tokens: int) -> int:
    return _size_query("cg_encoded_bound", ctypes.byref(_shape(shape)), chunk_tokens)


def cg_tables_bytes(shape) -> int:
    return _size_query("cg_tables_bytes", ctypes.byref(_shape(shape)))


def cg_encode_workspace_bytes(shape, chunk_tokens: int, num_chunks: int) -> int:
    return _size_query("cg_encode_workspace_bytes", ctypes.byref(_shape(shape)), chunk_tokens,
                       num_chunks)


def cg_build_tables(shape, kv, total_tokens: int, token_start: int, num_chunks: int,
                    chunk_tokens: int, level: int, tables, status, workspace=None,
                    workspace_bytes: int = 0, stream=None) -> int:
    return library().cg_build_tables(ctypes.byref(_shape(shape)), _ptr(kv), total_tokens,
                                     token_start, num_chunks, chunk_tokens, int(level),
                                     _ptr(tables), _ptr(status), _ptr(workspace),
                                     workspace_bytes, _stream(stream))


def cg_encode(shape, kv, total_tokens: int, token_start: int, num_chunks: int,
              chunk_tokens: int, level: int, tables, out, out_stride: int, out_sizes, status,
              workspace, workspace_bytes: int, stream=None) -> int:
    return library().cg_encode(ctypes.byref(_shape(shape)), _ptr(kv), total_tokens, token_start,
                               num_chunks, chunk_tokens, int(level), _ptr(tables), _ptr(out),
                               out_stride, _ptr(out_sizes), _ptr(status), _ptr(workspace),
                               workspace_bytes, _stream(stream))


def cg_encode_static(shape, kv, total_tokens: int, token_start: int, num_chunks: int,
                     chunk_tokens: int, level: int, tables, out, out_stride: int, out_sizes,
                     status, stream=None) -> int:
    """cg_encode with the library's own fixed scratch block (for callers that
    cannot allocate device memory; see include/cachegen.h)."""
    return library().cg_encode_static(ctypes.byref(_shape(shape)), _ptr(kv), total_tokens,
                                      token_start, num_chunks, chunk_tokens, int(level),
                                      _ptr(tables), _ptr(out), out_stride, _ptr(out_sizes),
                                      _ptr(status), _stream(stream))


def cg_encode_levels_workspace_bytes(shape, chunk_tokens: int, num_chunks: int) -> int:
    return _size_query("cg_encode_levels_workspace_bytes", ctypes.byref(_shape(shape)),
                       chunk_tokens, num_chunks)


def cg_encode_levels(shape, kv, total_tokens: int, token_start: int, num_chunks: int,
                     chunk_tokens: int, out, out_stride: int, out_sizes, status, workspace,
                     workspace_bytes: int, stream=None) -> int:
    """All three levels from one quantiser pass; container (level j, chunk k)
    at out + (j * num_chunks + k) * out_stride."""
    return library().cg_encode_levels(ctypes.byref(_shape(shape)), _ptr(kv), total_tokens,
                                      token_start, num_chunks, chunk_tokens, _ptr(out),
                                      out_stride, _ptr(out_sizes), _ptr(status),
                                      _ptr(workspace), workspace_bytes, _stream(stream))


def cg_encode_adjacent(shape, kv, total_tokens: int, token_start: int, num_chunks: int,
                       chunk_tokens: int, level: int, out, out_stride: int, out_sizes, status,
                       workspace, workspace_bytes: int, stream=None) -> int:
    """cg_encode writing format 2 (deltas between adjacent tokens)."""
    return library().cg_encode_adjacent(ctypes.byref(_shape(shape)), _ptr(kv), total_tokens,
                                        token_start, num_chunks, chunk_tokens, int(level),
                                        _ptr(out), out_stride, _ptr(out_sizes), _ptr(status),
                                        _ptr(workspace), workspace_bytes, _stream(stream))


def cg_decode_adjacent(shape, inp, in_stride: int, num_chunks: int, chunk_tokens: int,
                       level: int, out, out_elems: int, status, stream=None) -> int:
    return library().cg_decode_adjacent(ctypes.byref(_shape(shape)), _ptr(inp), in_stride,
                                        num_chunks, chunk_tokens, int(level), _ptr(out),
                                        out_elems, _ptr(status), _stream(stream))


def cg_decode_adjacent_into(shape, inp, in_stride: int, num_chunks: int, chunk_tokens: int,
                            level: int, kv, total_tokens: int, status, stream=None) -> int:
    return library().cg_decode_adjacent_into(ctypes.byref(_shape(shape)), _ptr(inp), in_stride,
                                             num_chunks, chunk_tokens, int(level), _ptr(kv),
                                             total_tokens, _ptr(status), _stream(stream))


def cg_decode(shape, inp, in_stride: int, num_chunks: int, chunk_tokens: int, level: int, out,
              out_elems: int, status, stream=None) -> int:
    return library().cg_decode(ctypes.byref(_shape(shape)), _ptr(inp), in_stride, num_chunks,
                               chunk_tokens, int(level), _ptr(out), out_elems, _ptr(status),
                               _stream(stream))


def cg_decode_into(shape, inp, in_stride: int, num_chunks: int, chunk_tokens: int, level: int,
                   kv, total_tokens: int, status, stream=None) -> int:
    return library().cg_decode_into(ctypes.byref(_shape(shape)), _ptr(inp), in_stride,
                                    num_chunks, chunk_tokens, int(level), _ptr(kv), total_tokens,
                                    _ptr(status), _stream(stream))


def cg_decode_into_paged(shape, inp, in_stride: int, num_chunks: int, chunk_tokens: int,
                         level: int, pool, num_pages: int, page_tokens: int, block_table,
                         total_tokens: int, status, stream=None) -> int:
    return library().cg_decode_into_paged(ctypes.byref(_shape(shape)), _ptr(inp), in_stride,
                                          num_chunks, chunk_tokens, int(level), _ptr(pool),
                                          num_pages, page_tokens, _ptr(block_table),
                                          total_tokens, _ptr(status), _stream(stream))


def cg_decode_adjacent_into_paged(shape, inp, in_stride: int, num_chunks: int,
                                  chunk_tokens: int, level: int, pool, num_pages: int,
                                  page_tokens: int, block_table, total_tokens: int, status,
                                  stream=None) -> int:
    return library().cg_decode_adjacent_into_paged(
        ctypes.byref(_shape(shape)), _ptr(inp), in_stride, num_chunks, chunk_tokens, int(level),
        _ptr(pool), num_pages, page_tokens, _ptr(block_table), total_tokens, _ptr(status),
        _stream(stream))
