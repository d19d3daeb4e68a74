"""Seeded synthetic inputs for the packed g128 linear layers (a module of its own).

This module is the one piece of code that both the CUDA path's tests/benchmark and
the CPU oracle's tests use: it only draws random numbers. It holds none of the
method's arithmetic (no packing, no dequantisation, no products).

Generator
---------
A counter-based 32-bit generator. For a (seed, tensor id) pair a 32-bit key is
derived, and element ``i`` of the stream is ``h(h(i) ^ key)`` where ``h`` is the
``lowbias32`` integer hash published by C. Wellons ("Hash Prospector", 2018):

    x ^= x >> 16; x *= 0x7feb352d; x ^= x >> 15; x *= 0x846ca68b; x ^= x >> 16

(all modulo 2**32).  Everything is computed with int64 torch ops whose
intermediate values stay below 2**63, so the same code gives the same bits on the
CPU and on a CUDA device.

Distributions (the recipe of the workloads):

* sign bits ~ Bernoulli(0.5): the raw stream bits. ``random_words`` returns 32 of
  them per uint32 word, ``random_signs`` one per element (top bit -> +1/-1).
* ternary values uniform over {-1, 0, +1}: ``floor(3 * u32 / 2**32) - 1``.
* N(0, 1): Box-Muller from two stream elements (fp64 on the host).
* scales: ``fp16(|N(0, 0.02)| + 1e-3)``; activations: ``N(0, 1)`` rounded to
  bf16 or fp16 (round-to-nearest-even by torch's conversion).
* token ids uniform in [0, V): ``floor(V * u32 / 2**32)``.
"""

from __future__ import annotations

import math

import torch

_M32 = 0xFFFFFFFF

# Tensor ids: each role in a workload draws from its own stream.
TID_X = 1
TID_WORDS = 2
TID_SCALES = 3
TID_TERNARY = 4
TID_IDS = 5
TID_SIGNS = 6


def _mul32(a: torch.Tensor, c: int) -> torch.Tensor:
    """(a * c) mod 2**32 for 0 <= a < 2**32 without int64 overflow."""
    c_lo = c & 0xFFFF
    c_hi = (c >> 16) & 0xFFFF
    lo = a * c_lo                      # < 2**48
    hi = ((a * c_hi) & 0xFFFF) << 16   # < 2**32
    return (lo + hi) & _M32


def _hash32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _key(seed: int, tid: int) -> int:
    t = torch.tensor([((seed & _M32) * 0x9E3779B9 + tid * 0x85EBCA6B) & _M32], dtype=torch.int64)
    return int(_hash32(_hash32(t) ^ (tid & _M32))[0])


def u32_stream(seed: int, tid: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Elements [start, start+count) of the stream (seed, tid), as int64 in [0, 2**32)."""
    if start < 0 or start + count > 2**32:
        raise ValueError("stream index out of range")
    key = _key(seed, tid)
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return _hash32(_hash32(i) ^ key)


def _as_int32_bits(u: torch.Tensor) -> torch.Tensor:
    """Reinterpret values in [0, 2**32) as int32 with the same 32 bits."""
    return torch.where(u >= 2**31, u - 2**32, u).to(torch.int32)


def random_words(seed: int, tid: int, count: int, device="cpu", start: int = 0) -> torch.Tensor:
    """``count`` uint32 words of i.i.d. Bernoulli(0.5) bits, returned as int32 bits."""
    return _as_int32_bits(u32_stream(seed, tid, start, count, device))


def random_signs(seed: int, tid: int, shape, device="cpu") -> torch.Tensor:
    """int8 values in {-1, +1}, each with probability 1/2."""
    n = math.prod(shape)
    u = u32_stream(seed, tid, 0, n, device)
    return ((u >> 31) * 2 - 1).to(torch.int8).reshape(shape)


def random_ternary(seed: int, tid: int, shape, device="cpu", row0: int = 0) -> torch.Tensor:
    """int8 values in {-1, 0, +1}, each with probability 1/3 (Lemire multiply-shift); with row0,
    rows [row0, row0 + shape[0]) of a matrix whose rows have shape[1] elements."""
    n = math.prod(shape)
    start = row0 * (n // shape[0]) if row0 else 0
    u = u32_stream(seed, tid, start, n, device)
    return (((u * 3) >> 32) - 1).to(torch.int8).reshape(shape)


def random_ids(seed: int, tid: int, count: int, vocab: int) -> torch.Tensor:
    """int32 token ids uniform in [0, vocab)."""
    if not 0 < vocab < 2**31:
        raise ValueError("vocab out of range")
    u = u32_stream(seed, tid, 0, count)
    return ((u * vocab) >> 32).to(torch.int32)


def normal(seed: int, tid: int, count: int, start: int = 0, device="cpu") -> torch.Tensor:
    """``count`` N(0,1) samples in fp64 (Box-Muller, cosine branch), on the host unless a
    device is given (device values may differ from host ones in the last bits of log/cos)."""
    u = u32_stream(seed, tid, 2 * start, 2 * count, device).to(torch.float64)
    u1 = (u[0::2] + 0.5) / 2.0**32
    u2 = u[1::2] / 2.0**32
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)


def activations(seed: int, M: int, K: int, dtype=torch.bfloat16, tid: int = TID_X) -> torch.Tensor:
    """x[M, K] ~ N(0, 1), rounded to ``dtype`` (bf16 or fp16), on the host."""
    return normal(seed, tid, M * K).reshape(M, K).to(dtype)


def scales(seed: int, N: int, G: int, tid: int = TID_SCALES, row0: int = 0,
           chunk: int = 1 << 24, device="cpu") -> torch.Tensor:
    """Group scales fp16[N, G] = fp16(|N(0, 0.02)| + 1e-3), rows [row0, row0 + N) of the stream."""
    out = torch.empty(N * G, dtype=torch.float16, device=device)
    for a in range(0, N * G, chunk):
        b = min(N * G, a + chunk)
        z = normal(seed, tid, b - a, start=row0 * G + a, device=device)
        out[a:b] = (z.abs() * 0.02 + 1e-3).to(torch.float16)
    return out.reshape(N, G)


def binary_words(seed: int, N: int, K: int, tid: int = TID_WORDS, row0: int = 0,
                 device="cpu") -> torch.Tensor:
    """Random packed sign words int32[N, K/32] (Bernoulli(0.5) bits), rows [row0, row0+N)."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    wpr = K // 32
    return random_words(seed, tid, N * wpr, device=device, start=row0 * wpr).reshape(N, wpr)
