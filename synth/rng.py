"""Counter-based random draws for the synthetic workloads.

Every value is a pure function of (seed, stream key, element index), so any slice of
any tensor can be regenerated on its own, on the CPU or on a GPU, with the same torch
code.  The mixing function is the 32-bit finaliser of MurmurHash3 (Austin Appleby,
public domain): three xor-shifts and two multiplications modulo 2**32.  All integer
arithmetic is done in int64 with every intermediate kept below 2**63, so no step
relies on signed overflow.

Normals come from the cosine branch of the Box-Muller transform over two
independent uniforms in (0, 1) with 32-bit resolution (largest |z| is about 6.8).

This module draws numbers only; it holds none of the indexer's arithmetic.
"""
from __future__ import annotations

import math

import torch

MASK32 = 0xFFFFFFFF
_TWO32 = float(2 ** 32)


def _mul32(a: torch.Tensor, c: int) -> torch.Tensor:
    """(a * c) mod 2**32 for int64 tensors a in [0, 2**32) and a constant c < 2**32."""
    lo = c & 0xFFFF
    hi = c >> 16
    return (a * lo + (((a * hi) & 0xFFFF) << 16)) & MASK32


def fmix32(h: torch.Tensor) -> torch.Tensor:
    """MurmurHash3's 32-bit finaliser, a bijection on [0, 2**32)."""
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32(h, 0xC2B2AE35)
    h = h ^ (h >> 16)
    return h


def _fmix32_int(x: int) -> int:
    x &= MASK32
    x ^= x >> 16
    x = (x * 0x85EBCA6B) & MASK32
    x ^= x >> 13
    x = (x * 0xC2B2AE35) & MASK32
    x ^= x >> 16
    return x


def stream_key(seed: int, *labels: int) -> tuple[int, int]:
    """Two 32-bit keys for one named stream (seed plus a tuple of small integers)."""
    k = _fmix32_int(seed * 0x9E3779B1 + 0x7F4A7C15)
    for lab in labels:
        k = _fmix32_int(k ^ _fmix32_int(lab + 0x632BE5AB))
    k2 = _fmix32_int(k ^ 0xA5A5A5A5)
    return k, k2


def u32(key: tuple[int, int], idx: torch.Tensor) -> torch.Tensor:
    """32-bit draws (int64 tensor in [0, 2**32)) for element indices idx (int64, < 2**62)."""
    k1, k2 = key
    lo = idx & MASK32
    hi = idx >> 32
    h = fmix32(lo ^ k1)
    h = fmix32((h ^ hi ^ k2) & MASK32)
    return h


def uniform(key, idx: torch.Tensor) -> torch.Tensor:
    """float64 uniforms in (0, 1): (u32 + 0.5) / 2**32."""
    return (u32(key, idx).to(torch.float64) + 0.5) / _TWO32


def normal(key, idx: torch.Tensor) -> torch.Tensor:
    """float64 standard normals, one per index (Box-Muller, cosine branch)."""
    i2 = idx * 2
    u1 = uniform(key, i2)
    u2 = uniform(key, i2 + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def arange(n: int, start: int = 0, device="cpu") -> torch.Tensor:
    return torch.arange(start, start + n, dtype=torch.int64, device=device)
