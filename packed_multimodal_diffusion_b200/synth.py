"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: only a counter-based normal
generator and the recipe that says which tensor gets which seed, mean and
standard deviation.  Both the CUDA path and the CPU oracle consume what it
produces.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014; the constants of Vigna's reference C code)
feeding Box-Muller in fp64, pairwise, as the image pipeline of
"cortiq-engine 0.8.83 src/h3imagegen.rs" does in its ``gauss``.  Output j of
a stream seeded with s is mix(s + (j + 1) * gamma), so any element can be
computed on its own; this file evaluates the whole stream at once with
wrapping int64 tensor arithmetic (the bits equal the uint64 ones).
"""

from __future__ import annotations

import math

import torch

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_CHUNK = 1 << 22


def _i64(v: int) -> int:
    """The int64 with the same bits as the uint64 ``v``."""
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 lanes (arithmetic shift, then mask)."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def splitmix64(seed: int, count: int, start: int = 0,
               device: str | torch.device = "cpu") -> torch.Tensor:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream seeded
    with ``seed``, as int64 tensors carrying the uint64 bits."""
    j = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = j * _i64(_GAMMA) + _i64(seed)
    z = (z ^ _lsr(z, 30)) * _i64(_M1)
    z = (z ^ _lsr(z, 27)) * _i64(_M2)
    return z ^ _lsr(z, 31)


def splitmix64_scalar(seed: int, count: int) -> list[int]:
    """The same stream, one value at a time in plain Python integers (the
    published sequential definition); used to pin the tensor version."""
    x = seed & ((1 << 64) - 1)
    out = []
    mask = (1 << 64) - 1
    for _ in range(count):
        x = (x + _GAMMA) & mask
        z = x
        z = ((z ^ (z >> 30)) * _M1) & mask
        z = ((z ^ (z >> 27)) * _M2) & mask
        out.append(z ^ (z >> 31))
    return out


def gauss(n: int, seed: int, device: str | torch.device = "cpu") -> torch.Tensor:
    """``n`` standard normals (fp64) from the SplitMix64 stream ``seed``:
    uniforms u = (z >> 11) / 2^53; each pair (a, b) gives
    r = sqrt(-2 ln max(a, 1e-300)), outputs r cos(2 pi b) then r sin(2 pi b)."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, _CHUNK):
        p1 = min(npairs, p0 + _CHUNK)
        z = splitmix64(seed, 2 * (p1 - p0), start=2 * p0, device=device)
        u = _lsr(z, 11).to(torch.float64) / float(1 << 53)
        a = u[0::2].clamp_min(1e-300)
        b = u[1::2]
        r = torch.sqrt(-2.0 * torch.log(a))
        ang = (2.0 * math.pi) * b
        pair = torch.stack((r * torch.cos(ang), r * torch.sin(ang)), dim=1).reshape(-1)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = pair[: hi - lo]
    return out


def normal(shape, seed: int, std: float = 1.0, mean: float = 0.0,
           dtype: torch.dtype = torch.float32,
           device: str | torch.device = "cpu") -> torch.Tensor:
    """A tensor of N(mean, std^2) values: fp64 normals scaled, then cast to
    fp32 and from there to ``dtype`` (so a bf16 tensor is the bf16 rounding
    of the fp32 value)."""
    n = 1
    for s in shape:
        n *= int(s)
    g = gauss(n, seed, device=device)
    v = (g * std + mean).to(torch.float32)
    return v.to(dtype).reshape(tuple(shape))


def tensor_seed(cfg_seed: int, index: int) -> int:
    """Per-tensor seed: ``cfg_seed * 1000 + index``."""
    return cfg_seed * 1000 + index
