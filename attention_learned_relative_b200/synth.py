"""Seeded synthetic inputs: a counter-based normal generator.

This module holds none of the attention arithmetic.  The tests, the benchmark and
the oracle's callers draw every input from it, so the CUDA path and the oracle see
the same numbers.

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
as easy as 1, 2, 3", SC'11), keyed by (seed, tensor id) with the element group
index as the counter, followed by the Box-Muller transform in float64.  Each
Philox call yields four normals.  Element e of a tensor is therefore a pure
function of (seed, tensor id, e): any slice can be regenerated on its own, on
any device.  The integer arithmetic is exact in torch int64 on CPU and CUDA
(32x32-bit products are split into 16-bit halves so nothing overflows).
"""
from __future__ import annotations

import math

import torch

_M0 = 0xD2511F53
_M1 = 0xCD9E8D57
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK = 0xFFFFFFFF

# Tensor ids: one key per input of the attention call.
TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "r": 4, "w": 5, "bank": 6, "rs": 7, "proj": 8}


def _mulhilo(a: torch.Tensor, m: int):
    """High and low 32-bit words of a * m for uint32 values held in int64."""
    x = a * (m & 0xFFFF)            # < 2^48
    y = a * (m >> 16)               # < 2^48
    lo = (((y & 0xFFFF) << 16) + x) & _MASK
    hi = (y + (x >> 16)) >> 16
    return hi, lo


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Ten Philox4x32 rounds on int64 tensors holding uint32 words."""
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        hi0, lo0 = _mulhilo(c0, _M0)
        hi1, lo1 = _mulhilo(c2, _M1)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def _normals_range(seed: int, tid: int, start: int, count: int, device) -> torch.Tensor:
    """Normals number start .. start+count-1 of stream (seed, tid), float64."""
    g0 = start // 4
    g1 = (start + count + 3) // 4
    n = torch.arange(g0, g1, dtype=torch.int64, device=device)
    z = torch.zeros_like(n)
    x0, x1, x2, x3 = philox4x32_10(n & _MASK, n >> 32, z, z, seed & _MASK, tid & _MASK)
    inv = 1.0 / 4294967296.0
    out = torch.empty((g1 - g0, 4), dtype=torch.float64, device=device)
    for (a, b), col in (((x0, x1), 0), ((x2, x3), 2)):
        u1 = (a.to(torch.float64) + 1.0) * inv          # (0, 1]
        u2 = b.to(torch.float64) * inv                  # [0, 1)
        rad = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * math.pi) * u2
        out[:, col] = rad * torch.cos(ang)
        out[:, col + 1] = rad * torch.sin(ang)
    flat = out.reshape(-1)
    off = start - 4 * g0
    return flat[off:off + count]


def normal(shape, seed: int, tensor: str, std: float = 1.0, dtype=torch.float32,
           device="cpu", chunk: int = 1 << 26) -> torch.Tensor:
    """A tensor of N(0, std^2) draws, rounded once to `dtype` (round to nearest even).

    The value is computed in float64, multiplied by std, then cast, so
    std = 0.5 scales exactly before the single rounding.
    """
    tid = TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)
    numel = 1
    for s in shape:
        numel *= int(s)
    out = torch.empty(numel, dtype=dtype, device=device)
    for s0 in range(0, numel, chunk):
        cnt = min(chunk, numel - s0)
        vals = _normals_range(seed, tid, s0, cnt, device)
        if std != 1.0:
            vals = vals * std
        out[s0:s0 + cnt] = vals.to(dtype)
    return out.reshape(tuple(int(s) for s in shape))


def normal_slice(shape, seed: int, tensor: str, index, std: float = 1.0,
                 dtype=torch.float32) -> torch.Tensor:
    """Regenerate chosen elements of normal(shape, seed, tensor) on the CPU.

    `index` is a LongTensor of flat element indices into a tensor of `shape`.
    """
    tid = TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)
    index = torch.as_tensor(index, dtype=torch.int64).reshape(-1)
    out = torch.empty(index.numel(), dtype=torch.float64)
    # Elements are generated four at a time; draw each needed group once.
    groups = torch.unique(index // 4)
    z = torch.zeros_like(groups)
    x = philox4x32_10(groups & _MASK, groups >> 32, z, z, seed & _MASK, tid & _MASK)
    inv = 1.0 / 4294967296.0
    vals = torch.empty((groups.numel(), 4), dtype=torch.float64)
    for (a, b), col in (((x[0], x[1]), 0), ((x[2], x[3]), 2)):
        u1 = (a.to(torch.float64) + 1.0) * inv
        u2 = b.to(torch.float64) * inv
        rad = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * math.pi) * u2
        vals[:, col] = rad * torch.cos(ang)
        vals[:, col + 1] = rad * torch.sin(ang)
    pos = torch.searchsorted(groups, index // 4)
    out = vals[pos, index % 4]
    if std != 1.0:
        out = out * std
    return out.to(dtype)
