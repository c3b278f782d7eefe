"""Seeded synthetic inputs for the sparse-MoE layer workloads.

Every element is a pure function of (seed, tensor id, attempt, flat index), so the
same tensor comes out on any device and in any chunking:

* bits    - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
            generators", OOPSLA 2014): state_n = key + n * 0x9E3779B97F4A7C15,
            output = mix(state_n) with the published two-multiply finaliser;
* normals - Box-Muller (1958): two uniforms u1 in (0, 1], u2 in [0, 1) give
            sqrt(-2 ln u1) * cos(2 pi u2);
* storage - the fp64 value times the requested standard deviation, rounded to the
            nearest bf16 (ties to even) by torch's own conversion.

This module draws numbers only. It holds none of the layer's arithmetic: no router,
no softmax, no expert math. Rows that have to be redrawn (for instance to keep a
routing margin) are redrawn by calling ``normal`` again with the next ``attempt``;
deciding which rows need it is the caller's business.
"""
from __future__ import annotations

import math

import torch

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB


def _s64(v: int) -> int:
    """Two's-complement int64 with the bit pattern of the unsigned 64-bit ``v``."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def splitmix64_scalar(state: int) -> int:
    """SplitMix64 finaliser on one unsigned 64-bit integer (pure Python, exact)."""
    z = state & _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 tensors holding unsigned 64-bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    """SplitMix64 finaliser on an int64 tensor; multiplication wraps modulo 2**64."""
    z = (z ^ _srl(z, 30)) * _s64(_MIX1)
    z = (z ^ _srl(z, 27)) * _s64(_MIX2)
    return z ^ _srl(z, 31)


def stream_key(seed: int, tensor_id: int, attempt: int = 0) -> int:
    """Key of one independent stream: three chained SplitMix64 steps over the ids."""
    k = splitmix64_scalar(seed * _GOLDEN + 1)
    k = splitmix64_scalar(k + (tensor_id + 1) * _GOLDEN)
    return splitmix64_scalar(k + (attempt + 1) * _GOLDEN)


def uniform_bits(key: int, index: torch.Tensor) -> torch.Tensor:
    """SplitMix64 output number ``index + 1`` of the stream ``key`` (int64 bit patterns)."""
    return _mix(index * _s64(_GOLDEN) + _s64(key))


def normals_at(key: int, i: torch.Tensor) -> torch.Tensor:
    """Normal number ``i`` (an int64 tensor of flat indices) of stream ``key``, in fp64.

    Normal i consumes SplitMix64 outputs 2i+1 and 2i+2 (u1 and u2 of Box-Muller).
    """
    b1 = uniform_bits(key, 2 * i + 1)
    b2 = uniform_bits(key, 2 * i + 2)
    scale = 2.0 ** -53
    u1 = (_srl(b1, 11).to(torch.float64) + 1.0) * scale      # (0, 1]
    u2 = _srl(b2, 11).to(torch.float64) * scale              # [0, 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def standard_normal_f64(key: int, start: int, count: int, device) -> torch.Tensor:
    """Normals number start .. start+count-1 of stream ``key``, in fp64."""
    return normals_at(key, torch.arange(start, start + count, dtype=torch.int64, device=device))


_CHUNK = 1 << 25


def normal(shape, std: float, seed: int, tensor_id: int, attempt: int = 0,
           device="cpu", dtype=torch.bfloat16, first_row: int = 0) -> torch.Tensor:
    """Tensor of N(0, std^2) values stored in ``dtype`` (bf16 by default).

    ``first_row`` offsets the flat index by ``first_row * prod(shape[1:])`` so that a
    slice of rows of a larger tensor can be drawn on its own and still match.
    """
    shape = tuple(int(s) for s in shape)
    n = 1
    for s in shape:
        n *= s
    row = 1
    for s in shape[1:]:
        row *= s
    key = stream_key(seed, tensor_id, attempt)
    out = torch.empty(n, dtype=dtype, device=device)
    base = first_row * row
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = (standard_normal_f64(key, base + s, c, device) * std).to(dtype)
    return out.view(shape)


def normal_rows_unit_rms(num_rows: int, width: int, seed: int, tensor_id: int,
                         attempt: int = 0, device="cpu", first_row: int = 0) -> torch.Tensor:
    """[num_rows, width] bf16 rows of N(0,1) draws, each scaled to RMS 1 in fp64 first."""
    key = stream_key(seed, tensor_id, attempt)
    out = torch.empty((num_rows, width), dtype=torch.bfloat16, device=device)
    rows_per = max(1, _CHUNK // width)
    for r in range(0, num_rows, rows_per):
        c = min(rows_per, num_rows - r)
        z = standard_normal_f64(key, (first_row + r) * width, c * width, device).view(c, width)
        rms = torch.sqrt((z * z).mean(dim=1, keepdim=True))
        out[r:r + c] = (z / rms).to(torch.bfloat16)
    return out


def rows_at(rows: torch.Tensor, width: int, std: float, seed: int, tensor_id: int,
            attempt: int, unit_rms: bool) -> torch.Tensor:
    """bf16 rows ``rows`` (int64 tensor of row numbers) of a [*, width] tensor, as drawn
    by ``normal`` (``unit_rms`` False) or ``normal_rows_unit_rms`` (True) for ``attempt``."""
    key = stream_key(seed, tensor_id, attempt)
    idx = rows.to(torch.int64).view(-1, 1) * width + torch.arange(width, dtype=torch.int64,
                                                                  device=rows.device)
    z = normals_at(key, idx)
    if unit_rms:
        z = z / torch.sqrt((z * z).mean(dim=1, keepdim=True))
    else:
        z = z * std
    return z.to(torch.bfloat16)
