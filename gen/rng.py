"""Counter-based random numbers for the synthetic workloads.

Every tensor is identified by (seed, name). Element ``i`` of a tensor draws the two
64-bit words ``splitmix64(key, 2i)`` and ``splitmix64(key, 2i + 1)`` where
``key = seed XOR fnv1a64(name)``, turns them into uniforms in double precision and
maps them to one standard normal with the Box–Muller transform. SplitMix64 is the
mixer published by Steele, Lea and Flood (OOPSLA 2014); FNV-1a is the public
Fowler–Noll–Vo hash. Both are written out here from their definitions.

The same torch code runs on the CPU and on a CUDA device, so a large tensor can be
drawn where it will live. Integer arithmetic wraps modulo 2**64 in torch's int64
kernels on both devices; the transcendental functions of the Box–Muller step may
differ by one unit in the last place of a double between devices, which after
rounding to fp32/bf16 almost never shows. Within one run both sides of a parity
check always receive the very same bytes, so this never affects a comparison.
"""

from __future__ import annotations

import math

import torch

_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _to_i64(u: int) -> int:
    """Reinterpret an unsigned 64-bit integer as a signed one (two's complement)."""
    u &= _MASK64
    return u - (1 << 64) if u >= (1 << 63) else u


def fnv1a64(name: str) -> int:
    """64-bit FNV-1a hash of the UTF-8 bytes of ``name`` (unsigned result)."""
    h = 0xCBF29CE484222325
    for byte in name.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & _MASK64
    return h


def splitmix64_scalar(key: int, counter: int) -> int:
    """Pure-Python SplitMix64 output for state ``key + (counter + 1) * golden``."""
    z = (key + (counter + 1) * _GOLDEN) & _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 data (torch's >> is arithmetic)."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def splitmix64(key: int, counters: torch.Tensor) -> torch.Tensor:
    """Vectorised SplitMix64; ``counters`` is int64, result holds the raw 64-bit words."""
    z = counters + 1
    z = z * _to_i64(_GOLDEN) + _to_i64(key)
    z = (z ^ _lsr(z, 30)) * _to_i64(_MIX1)
    z = (z ^ _lsr(z, 27)) * _to_i64(_MIX2)
    return z ^ _lsr(z, 31)


def _uniform53(words: torch.Tensor, open_zero: bool) -> torch.Tensor:
    """Top 53 bits of each word as a double in [0, 1), or in (0, 1] if ``open_zero``."""
    top = _lsr(words, 11).to(torch.float64)
    if open_zero:
        top = top + 1.0
    return top * (2.0 ** -53)


_BLOCK = 1 << 23


def normal(name: str, shape, seed: int, device="cpu") -> torch.Tensor:
    """Standard normal float64 tensor of ``shape`` for tensor ``name`` under ``seed``."""
    key = (seed ^ fnv1a64(name)) & _MASK64
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.float64, device=device)
    for start in range(0, n, _BLOCK):
        stop = min(n, start + _BLOCK)
        idx = torch.arange(start, stop, dtype=torch.int64, device=device)
        u1 = _uniform53(splitmix64(key, 2 * idx), open_zero=True)
        u2 = _uniform53(splitmix64(key, 2 * idx + 1), open_zero=False)
        out[start:stop] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return out.reshape(tuple(int(s) for s in shape))


def uniform(name: str, n: int, seed: int, device="cpu") -> torch.Tensor:
    """``n`` float64 uniforms in [0, 1) for tensor ``name`` under ``seed``."""
    key = (seed ^ fnv1a64(name)) & _MASK64
    idx = torch.arange(n, dtype=torch.int64, device=device)
    return _uniform53(splitmix64(key, idx), open_zero=False)


def distinct_positions(name: str, count: int, length: int, seed: int) -> list[int]:
    """``count`` distinct indices in [0, length) by a seeded partial Fisher–Yates shuffle."""
    if not 0 <= count <= length:
        raise ValueError("count must lie in [0, length]")
    u = uniform(name, count, seed).tolist()
    perm = list(range(length))
    for k in range(count):
        j = k + int(math.floor(u[k] * (length - k)))
        perm[k], perm[j] = perm[j], perm[k]
    return sorted(perm[:count])
