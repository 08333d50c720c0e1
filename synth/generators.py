"""Counter-based random numbers, identical on numpy (host) and torch (any device).

Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; output function as published by
S. Vigna).  Element ``i`` of a stream with seed ``s`` is

    z  = s + (i + 1) * 0x9E3779B97F4A7C15          (mod 2^64)
    z  = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
    z  = (z ^ (z >> 27)) * 0x94D049BB133111EB
    out = z ^ (z >> 31)

Normals use Box-Muller on the counter pair (2i, 2i+1), cosine branch only, so
any slice of a stream can be regenerated on its own (random access).  The
numpy and torch versions run the same integer steps; the transcendental step
runs in float64 on both sides and the value is then rounded to fp32 and bf16,
so a host slice matches the device tensor bit for bit except when libm
results differ in the last float64 bit right at a rounding boundary.
"""
from __future__ import annotations

import math

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB
_M64 = (1 << 64) - 1


def _signed(v: int) -> int:
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


# ----------------------------------------------------------------------------- numpy


def splitmix64_np(seed: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 output for the given uint64 counters (vectorised, wraps mod 2^64)."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & _M64) + (c + np.uint64(1)) * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MUL1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MUL2)
        z = z ^ (z >> np.uint64(31))
    return z


def uniform_np(seed: int, start: int, n: int) -> np.ndarray:
    """Uniform [0, 1) float64 for stream elements start .. start+n-1."""
    c = np.arange(start, start + n, dtype=np.uint64)
    z = splitmix64_np(seed, c)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_np(seed: int, start: int, n: int) -> np.ndarray:
    """Standard normal float64 for stream elements start .. start+n-1."""
    i = np.arange(start, start + n, dtype=np.uint64)
    z1 = splitmix64_np(seed, i * np.uint64(2))
    z2 = splitmix64_np(seed, i * np.uint64(2) + np.uint64(1))
    u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    u2 = (z2 >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos((2.0 * math.pi) * u2)


def bf16_bits_np(x: np.ndarray) -> np.ndarray:
    """Round float64 -> fp32 (nearest) -> bf16 (nearest-even); return uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32_np(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (used to build derived inputs)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def e4m3_codes_np(x: np.ndarray) -> np.ndarray:
    """Encode values to OCP e4m3fn codes with the library conversion (clipped to +-448)."""
    import torch
    t = torch.from_numpy(np.clip(np.asarray(x, dtype=np.float32), -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def sub_seed(base: int, layer: int, tensor_id: int) -> int:
    """Independent stream seed for (base seed, layer, tensor) via one SplitMix64 step."""
    key = (base * 0x100000001B3 + layer * 0x9E37 + tensor_id * 0x85EBCA6B) & _M64
    return int(splitmix64_np(key, np.array([0], dtype=np.uint64))[0])


def ar1_keys_np(seed: int, length: int, dim: int, rho: float) -> np.ndarray:
    """Per-dimension AR(1) drift along positions: k_0 = e_0, k_s = rho k_{s-1} + sqrt(1-rho^2) e_s."""
    eps = normal_np(seed, 0, length * dim).reshape(length, dim)
    out = np.empty_like(eps)
    c = math.sqrt(1.0 - rho * rho)
    out[0] = eps[0]
    for s in range(1, length):
        out[s] = rho * out[s - 1] + c * eps[s]
    return out


# ----------------------------------------------------------------------------- torch


def _lsr(z, s: int):
    """Logical right shift of an int64 tensor holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _splitmix64_torch(seed: int, c):
    z = c.add(1).mul_(_signed(GAMMA)).add_(_signed(seed))
    z = (z ^ _lsr(z, 30)).mul_(_signed(MUL1))
    z = (z ^ _lsr(z, 27)).mul_(_signed(MUL2))
    return z ^ _lsr(z, 31)


def normal_torch(seed: int, start: int, n: int, device="cpu", chunk: int = 1 << 25):
    """Same values as :func:`normal_np`, as a float64 torch tensor on ``device``."""
    import torch
    out = torch.empty(n, dtype=torch.float64, device=device)
    inv = 1.0 / 9007199254740992.0
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        i = torch.arange(start + a, start + b, dtype=torch.int64, device=device)
        z1 = _splitmix64_torch(seed, i * 2)
        z2 = _splitmix64_torch(seed, i * 2 + 1)
        u1 = (_lsr(z1, 11).to(torch.float64) + 1.0) * inv
        u2 = _lsr(z2, 11).to(torch.float64) * inv
        out[a:b] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return out


def normal_bf16_torch(seed: int, n: int, device, scale: float = 1.0, chunk: int = 1 << 25):
    """bf16 tensor equal to bf16_bits_torch(normal_torch(seed, 0, n) * scale), built chunk
    by chunk so that no float64 copy of the whole tensor is held."""
    import torch
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        x = normal_torch(seed, a, b - a, device=device, chunk=chunk)
        if scale != 1.0:
            x = x * scale
        out[a:b] = bf16_bits_torch(x)
    return out


def bf16_bits_torch(x):
    """float64 tensor -> bf16 tensor with the same rounding as :func:`bf16_bits_np`."""
    import torch
    f = x.to(torch.float32).contiguous()
    u = f.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    r = torch.where(r >= 0x8000, r - 0x10000, r).to(torch.int16)
    return r.view(torch.bfloat16)


def e4m3_codes_torch(x):
    """Encode a float tensor to e4m3fn codes (uint8) with the library conversion, clipped to +-448."""
    import torch
    return x.to(torch.float32).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
