"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws numbers and nothing else: it holds no step of the attention
method (no pooling, scoring, selection, quantisation or softmax).  Both sides
of every parity check take their inputs from here, so the only code they share
is the random-number definition below.

Generator (counter based, so any slice of any tensor can be drawn on its own):

* splitmix64 finaliser (Steele, Lea and Flood, "Fast splittable pseudorandom
  number generators", OOPSLA 2014; constants as published by Vigna):
      z ^= z >> 30; z *= 0xBF58476D1CE4E5B9
      z ^= z >> 27; z *= 0x94D049BB133111EB
      z ^= z >> 31
* stream key  K = mix(fnv1a64(name) ^ mix(seed + GOLDEN))
* word i      h(i) = mix(K + (i + 1) * GOLDEN),  GOLDEN = 0x9E3779B97F4A7C15
* uniforms    u1 = ((h(2p) >> 11) + 1) * 2^-53 in (0, 1]
              u2 = (h(2p+1) >> 11) * 2^-53      in [0, 1)
* Box-Muller  element 2p   = sqrt(-2 ln u1) * cos(2 pi u2)
              element 2p+1 = sqrt(-2 ln u1) * sin(2 pi u2)
  computed in float64, multiplied by the requested standard deviation and
  then rounded once to the storage type (fp32, or bf16 by round-to-nearest-
  even from the fp32 value).

Two implementations of the same definition are provided: numpy (host) and
torch (any device, used to fill multi-GB device tensors quickly).  Their
uint64 words agree bit for bit; the float64 transcendental functions may
differ in the last ulp between libraries, which the tests measure.
"""
from __future__ import annotations

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1


def _mix_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for b in name.encode("utf-8"):
        h ^= b
        h = (h * 0x100000001B3) & MASK64
    return h


def stream_key(seed: int, name: str) -> int:
    """64-bit key of the stream that draws tensor `name` under `seed`."""
    return _mix_int(fnv1a64(name) ^ _mix_int((seed + GOLDEN) & MASK64))


# ----------------------------------------------------------------- numpy side
def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def words_np(key: int, start: int, count: int) -> np.ndarray:
    """h(i) for i in [start, start+count) as uint64."""
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (i + np.uint64(1)) * np.uint64(GOLDEN)
        return _mix_np(z)


def normal_np(seed: int, name: str, start: int, count: int, std: float = 1.0) -> np.ndarray:
    """Elements [start, start+count) of the N(0, std^2) stream, float64."""
    key = stream_key(seed, name)
    p0 = start // 2
    p1 = (start + count + 1) // 2
    w = words_np(key, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    u1 = ((w[:, 0] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (w[:, 1] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * np.pi * u2
    z = np.empty(2 * (p1 - p0), dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    off = start - 2 * p0
    return z[off:off + count] * std


def f32_to_bf16_bits_np(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32_np(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def tensor_np(seed: int, name: str, shape, std: float = 1.0, dtype: str = "f32",
              start: int = 0) -> np.ndarray:
    """A whole tensor (or the slice starting at flat index `start`) drawn on the host.

    dtype "f32" -> float32 array, "bf16" -> uint16 array of bf16 bits,
    "f64" -> float64 array (no rounding).
    """
    n = int(np.prod(shape)) if len(shape) else 1
    z = normal_np(seed, name, start, n, std)
    if dtype == "f64":
        return z.reshape(shape)
    f = z.astype(np.float32)
    if dtype == "f32":
        return f.reshape(shape)
    if dtype == "bf16":
        return f32_to_bf16_bits_np(f).reshape(shape)
    raise ValueError(dtype)


# ----------------------------------------------------------------- torch side
def _as_i64(u: int) -> int:
    return u - (1 << 64) if u >= (1 << 63) else u


def _lsr_t(z, k: int):
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_t(z):
    z = (z ^ _lsr_t(z, 30)) * _as_i64(M1)
    z = (z ^ _lsr_t(z, 27)) * _as_i64(M2)
    return z ^ _lsr_t(z, 31)


def words_torch(key: int, start: int, count: int, device="cpu"):
    import torch
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    z = (i + 1) * _as_i64(GOLDEN) + _as_i64(key)
    return _mix_t(z)


def tensor_torch(seed: int, name: str, shape, std: float = 1.0, dtype: str = "f32",
                 device="cuda", start: int = 0, chunk: int = 1 << 26):
    """Same stream as tensor_np, drawn with torch ops on `device`.

    dtype "f32" -> torch.float32, "bf16" -> torch.bfloat16 (RNE from the fp32
    value, as torch's own conversion does).  Drawn in chunks to bound the
    float64 temporaries.
    """
    import torch
    n = 1
    for s in shape:
        n *= int(s)
    key = stream_key(seed, name)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    out = torch.empty(n, dtype=tdt, device=device)
    pos = 0
    while pos < n:
        cnt = min(chunk, n - pos)
        s0 = start + pos
        p0 = s0 // 2
        p1 = (s0 + cnt + 1) // 2
        w = words_torch(key, 2 * p0, 2 * (p1 - p0), device).view(-1, 2)
        u1 = (_lsr_t(w[:, 0], 11).to(torch.float64) + 1.0) * 2.0 ** -53
        u2 = _lsr_t(w[:, 1], 11).to(torch.float64) * 2.0 ** -53
        del w
        r = torch.sqrt(-2.0 * torch.log(u1))
        th = 2.0 * np.pi * u2
        z = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).view(-1)
        off = s0 - 2 * p0
        z = z[off:off + cnt] * std
        out[pos:pos + cnt] = z.to(torch.float32).to(tdt)
        pos += cnt
    return out.view(*shape)
