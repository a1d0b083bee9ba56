"""Measurement helpers that are not part of the codec's path.

clamp_rate: how often the [-127, 127] clamp of the delta codes broke the
quantiser's error bound.  For a delta value whose code was not clamped, the
reconstruction error is at most step/2 (the quantiser picks the nearest
multiple of the step) plus half an fp16 spacing of the stored value (the final
rounding).  A clamped code leaves the value more than step/2 away.  So,
counting from the input and the decoded output alone, a delta value is counted
as clamped when
    |x - x^| > step/2 + ulp16(x^)/2 + 2^-20 |x|,
the last term absorbing the float32 roundings of the reconstruction.  Anchor
tokens (local index 0 mod 10 of each chunk) are not deltas and never clamp
(their code range spans the chunk's anchors), so they are left out.
These are torch tensor operations on the side of a measurement; the codec's
own arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import LEVELS

GROUP = 10
STEPS = {  # [Practice] 3.1: first / middle / last third of the layers
    LEVELS["high"]: (0.3, 0.8, 1.2),
    LEVELS["balanced"]: (0.5, 1.0, 1.5),
    LEVELS["fast"]: (0.8, 1.5, 2.0),
}


def _half_ulp16(v: torch.Tensor) -> torch.Tensor:
    """Half the fp16 spacing at |v| (subnormal spacing 2^-24 below 2^-14)."""
    a = v.abs().clamp_min(2.0 ** -14)
    _, e = torch.frexp(a)  # a = m * 2^e, m in [0.5, 1)
    return torch.ldexp(torch.ones_like(a), (e - 12).to(torch.int32))


def clamp_counts(kv: torch.Tensor, decoded: torch.Tensor, chunk_tokens: int, level: int,
                 token_start: int = 0, n_tokens: int | None = None) -> tuple[int, int]:
    """(clamped delta values, delta values) over tokens [token_start,
    token_start + n_tokens) of two [L, 2, T, H, D] 16-bit tensors holding fp16
    bits (the input and its decode), chunks of chunk_tokens starting at
    token_start.  Works layer by layer to bound temporary memory."""
    L, _, T, H, D = kv.shape
    n_tokens = T - token_start if n_tokens is None else n_tokens
    local = torch.arange(n_tokens, device=kv.device) % chunk_tokens
    is_delta = (local % GROUP) != 0
    clamped = 0
    for l in range(L):
        step = STEPS[int(level)][(3 * l) // L]
        sl = slice(token_start, token_start + n_tokens)
        x = kv[l, :, sl].view(torch.float16).float()
        y = decoded[l, :, sl].view(torch.float16).float()
        bound = step / 2 + _half_ulp16(y) + x.abs() * 2.0 ** -20
        bad = ((x - y).abs() > bound) & is_delta.view(1, -1, 1, 1)
        clamped += int(bad.sum().item())
    deltas = int(is_delta.sum().item()) * L * 2 * H * D
    return clamped, deltas


def clamp_rate(kv: torch.Tensor, decoded: torch.Tensor, chunk_tokens: int, level: int,
               token_start: int = 0, n_tokens: int | None = None) -> float:
    c, n = clamp_counts(kv, decoded, chunk_tokens, level, token_start, n_tokens)
    return c / n if n else 0.0
