"""Convenience wrappers over the libcachegen binding for torch CUDA tensors.

These helpers only allocate device buffers with torch and call the C ABI; the
codec itself runs entirely in the library's kernels.  KV tensors hold fp16
bits in a 16-bit dtype (torch.float16 or torch.int16), shaped [L, 2, T, H, D].
Nothing here synchronises: results are device tensors plus a device status
word, which the caller checks after synchronising (``status_of``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (CG_OK, CacheGenError, Shape, cg_build_tables, cg_decode, cg_decode_adjacent,
               cg_decode_adjacent_into, cg_decode_adjacent_into_paged, cg_decode_into,
               cg_decode_into_paged, cg_encode, cg_encode_adjacent, cg_encode_levels,
               cg_encode_levels_workspace_bytes, cg_encode_workspace_bytes, cg_encoded_bound,
               cg_tables_bytes, check)


def _shape_of(kv: torch.Tensor) -> tuple[Shape, int]:
    if kv.dim() != 5 or kv.shape[1] != 2 or kv.element_size() != 2:
        raise ValueError("kv must be a 16-bit tensor shaped [L, 2, T, H, D]")
    if not kv.is_cuda or not kv.is_contiguous():
        raise ValueError("kv must be a contiguous CUDA tensor")
    L, _, T, H, D = kv.shape
    return Shape(L, H, D), T


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def status_of(status: torch.Tensor) -> int:
    return int(status.item())


@dataclass
class Encoded:
    """Containers of consecutive chunks at a fixed stride, with their sizes."""
    data: torch.Tensor      # uint8 [num_chunks * stride]
    sizes: torch.Tensor     # int64 [num_chunks] (device; u64 values)
    stride: int
    num_chunks: int
    chunk_tokens: int
    level: int
    shape: Shape
    status: torch.Tensor
    adjacent: bool = False  # format 2 (deltas between adjacent tokens)

    def chunk(self, k: int) -> torch.Tensor:
        """Container k as a device view (synchronises to read its size)."""
        n = int(self.sizes[k].item())
        return self.data[k * self.stride:k * self.stride + n]


class Encoder:
    """Reusable encoder state: workspace and output slots for a fixed geometry."""

    def __init__(self, shape: Shape, chunk_tokens: int, num_chunks: int, device,
                 out_stride: int | None = None):
        self.shape, self.C, self.num_chunks = shape, chunk_tokens, num_chunks
        self.ws_bytes = cg_encode_workspace_bytes(shape, chunk_tokens, num_chunks)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.stride = out_stride or cg_encoded_bound(shape, chunk_tokens)
        self.out = torch.empty(self.stride * num_chunks, dtype=torch.uint8, device=device)
        self.sizes = torch.zeros(num_chunks, dtype=torch.int64, device=device)
        self.status = new_status(device)

    def encode(self, kv: torch.Tensor, level: int, token_start: int = 0,
               tables: torch.Tensor | None = None, stream=None,
               adjacent: bool = False) -> Encoded:
        """adjacent=True writes format 2 (cg_encode_adjacent; no supplied tables)."""
        shape, T = _shape_of(kv)
        if adjacent:
            if tables is not None:
                raise ValueError("format 2 builds its own tables")
            check(cg_encode_adjacent(shape, kv, T, token_start, self.num_chunks, self.C, level,
                                     self.out, self.stride, self.sizes, self.status,
                                     self.workspace, self.ws_bytes, stream),
                  "cg_encode_adjacent")
        else:
            check(cg_encode(shape, kv, T, token_start, self.num_chunks, self.C, level, tables,
                            self.out, self.stride, self.sizes, self.status, self.workspace,
                            self.ws_bytes, stream), "cg_encode")
        return Encoded(self.out, self.sizes, self.stride, self.num_chunks, self.C, level, shape,
                       self.status, adjacent)


class LevelsEncoder:
    """Workspace and output slots of cg_encode_levels for a fixed geometry:
    the three levels' containers of num_chunks chunks, level-major."""

    def __init__(self, shape: Shape, chunk_tokens: int, num_chunks: int, device,
                 out_stride: int | None = None):
        self.shape, self.C, self.num_chunks = shape, chunk_tokens, num_chunks
        self.ws_bytes = cg_encode_levels_workspace_bytes(shape, chunk_tokens, num_chunks)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.stride = out_stride or cg_encoded_bound(shape, chunk_tokens)
        self.out = torch.empty(3 * self.stride * num_chunks, dtype=torch.uint8, device=device)
        self.sizes = torch.zeros(3 * num_chunks, dtype=torch.int64, device=device)
        self.status = new_status(device)

    def encode(self, kv: torch.Tensor, token_start: int = 0, stream=None) -> list[Encoded]:
        """One Encoded view per level (HIGH, BALANCED, FAST)."""
        shape, T = _shape_of(kv)
        check(cg_encode_levels(shape, kv, T, token_start, self.num_chunks, self.C, self.out,
                               self.stride, self.sizes, self.status, self.workspace,
                               self.ws_bytes, stream), "cg_encode_levels")
        per = self.stride * self.num_chunks
        return [Encoded(self.out[j * per:(j + 1) * per],
                        self.sizes[j * self.num_chunks:(j + 1) * self.num_chunks], self.stride,
                        self.num_chunks, self.C, j, shape, self.status) for j in range(3)]


def encode_levels(kv: torch.Tensor, chunk_tokens: int, token_start: int = 0,
                  num_chunks: int | None = None, out_stride: int | None = None,
                  stream=None) -> list[Encoded]:
    shape, T = _shape_of(kv)
    if num_chunks is None:
        num_chunks = -(-(T - token_start) // chunk_tokens)
    enc = LevelsEncoder(shape, chunk_tokens, num_chunks, kv.device, out_stride)
    return enc.encode(kv, token_start, stream)


def encode(kv: torch.Tensor, chunk_tokens: int, level: int, token_start: int = 0,
           num_chunks: int | None = None, tables: torch.Tensor | None = None,
           out_stride: int | None = None, stream=None, adjacent: bool = False) -> Encoded:
    shape, T = _shape_of(kv)
    if num_chunks is None:
        num_chunks = -(-(T - token_start) // chunk_tokens)
    enc = Encoder(shape, chunk_tokens, num_chunks, kv.device, out_stride)
    return enc.encode(kv, level, token_start, tables, stream, adjacent)


def build_tables(kv: torch.Tensor, chunk_tokens: int, level: int, token_start: int = 0,
                 num_chunks: int | None = None, stream=None):
    shape, T = _shape_of(kv)
    if num_chunks is None:
        num_chunks = -(-(T - token_start) // chunk_tokens)
    tb = cg_tables_bytes(shape)
    tables = torch.empty(tb * num_chunks, dtype=torch.uint8, device=kv.device)
    status = new_status(kv.device)
    check(cg_build_tables(shape, kv, T, token_start, num_chunks, chunk_tokens, level, tables,
                          status, None, 0, stream), "cg_build_tables")
    return tables, tb, status


def decode(data: torch.Tensor, stride: int, shape: Shape, chunk_tokens: int, level: int,
           num_chunks: int, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
           stream=None, adjacent: bool = False):
    """Decode into chunk slots [num_chunks][L][2][C][H][D] (chunk k packed by its n_k).
    adjacent=True decodes format-2 containers."""
    L, H, D = shape.num_layers, shape.num_kv_heads, shape.head_dim
    slot = L * 2 * chunk_tokens * H * D
    if out is None:
        out = torch.empty(slot * num_chunks, dtype=torch.int16, device=data.device)
    if status is None:
        status = new_status(data.device)
    fn = cg_decode_adjacent if adjacent else cg_decode
    check(fn(shape, data, stride, num_chunks, chunk_tokens, level, out, out.numel(), status,
             stream), fn.__name__)
    return out, status


def decode_into(data: torch.Tensor, stride: int, shape: Shape, chunk_tokens: int, level: int,
                num_chunks: int, kv: torch.Tensor, status: torch.Tensor | None = None,
                stream=None, adjacent: bool = False):
    _, T = _shape_of(kv)
    if status is None:
        status = new_status(data.device)
    fn = cg_decode_adjacent_into if adjacent else cg_decode_into
    check(fn(shape, data, stride, num_chunks, chunk_tokens, level, kv, T, status, stream),
          fn.__name__)
    return status


def decode_into_paged(data: torch.Tensor, stride: int, shape: Shape, chunk_tokens: int,
                      level: int, num_chunks: int, pool: torch.Tensor, page_tokens: int,
                      block_table: torch.Tensor, total_tokens: int,
                      status: torch.Tensor | None = None, stream=None, adjacent: bool = False):
    """Decode into a paged pool [L][2][num_pages][page_tokens][H][D] through an
    int32 block table (logical page -> physical page).  adjacent=True decodes
    format-2 containers."""
    L, H, D = shape.num_layers, shape.num_kv_heads, shape.head_dim
    num_pages = pool.numel() // (L * 2 * page_tokens * H * D)
    if status is None:
        status = new_status(data.device)
    fn = cg_decode_adjacent_into_paged if adjacent else cg_decode_into_paged
    check(fn(shape, data, stride, num_chunks, chunk_tokens, level, pool, num_pages, page_tokens,
             block_table, total_tokens, status, stream), fn.__name__)
    return status


def raise_on_status(status: torch.Tensor, what: str = "") -> None:
    s = status_of(status)
    if s != CG_OK:
        raise CacheGenError(s, what)
