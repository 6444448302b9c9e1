"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds random-number generation only: none of the method's
arithmetic lives here.  One counter-based generator serves every device so
that a tensor drawn on the GPU is bit-identical to the same tensor drawn on
the host:

* counter  c = 3*i + r  (element index i, lane r in 0..2), 32-bit;
* word     h = mix32(mix32(c ^ k1) ^ k2), with k1, k2 derived from the seed,
  where mix32 is the 32-bit integer finaliser x ^= x>>16; x *= 0x45d9f3b
  (twice), x ^= x>>16;
* the twelve bytes of the three words of element i are twelve uniforms
  u = (b + 0.5)/256 on (0, 1), and the element is  sum(u) - 6, the classic
  Irwin-Hall approximation to N(0, 1): mean 0, variance 1 - 2^-16, support
  (-6, 6).  The value equals (sum(b) - 1530)/256, which float32 holds exactly.

bf16 tensors are that float32 value rounded to nearest-even.  All steps are
int64 torch ops with products below 2^59, so CPU and CUDA agree bit for bit.
"""
from __future__ import annotations

import torch

_MASK32 = 0xFFFFFFFF
_MUL = 0x45D9F3B


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = (((x >> 16) ^ x) * _MUL) & _MASK32
    x = (((x >> 16) ^ x) * _MUL) & _MASK32
    return (x >> 16) ^ x


def _mix32_int(x: int) -> int:
    x &= _MASK32
    x = (((x >> 16) ^ x) * _MUL) & _MASK32
    x = (((x >> 16) ^ x) * _MUL) & _MASK32
    return (x >> 16) ^ x


def seed_of(*fields: int) -> int:
    """Fold integer fields (role, stream, chunk, step, layer, ...) into one 32-bit seed."""
    s = 0x2545F491
    for f in fields:
        s = _mix32_int(s ^ _mix32_int(int(f) + 0x9E3779B9))
    return s


def normal_f32(seed: int, shape, device="cpu") -> torch.Tensor:
    """Approximately N(0,1) float32 tensor of `shape` (exact Irwin-Hall(12) values)."""
    n = 1
    for d in shape:
        n *= int(d)
    if 3 * n >= (1 << 32):
        raise ValueError("counter space exhausted: at most 1.43e9 elements per tensor")
    k1 = _mix32_int(seed ^ 0x68E31DA4)
    k2 = _mix32_int(seed ^ 0xB5297A4D)
    i = torch.arange(n, dtype=torch.int64, device=device)
    acc = torch.zeros(n, dtype=torch.int64, device=device)
    for r in range(3):
        h = _mix32(_mix32((3 * i + r) ^ k1) ^ k2)
        acc += (h & 0xFF) + ((h >> 8) & 0xFF) + ((h >> 16) & 0xFF) + (h >> 24)
    x = (acc - 1530).to(torch.float32) / 256.0
    return x.reshape(tuple(int(d) for d in shape))


def normal_bf16(seed: int, shape, device="cpu") -> torch.Tensor:
    """The float32 draw of `normal_f32` rounded to bf16 (round to nearest even)."""
    return normal_f32(seed, shape, device).to(torch.bfloat16)


# Roles keep the streams of different tensors apart.
ROLE_Q, ROLE_K, ROLE_V, ROLE_X, ROLE_VEL, ROLE_STORE_K, ROLE_STORE_V = range(7)


def chunk_qkv(stream: int, chunk: int, step: int, layer: int, n_tokens: int,
              heads: int, head_dim: int, device="cpu"):
    """q, k, v of one chunk at one (step, layer): bf16 [n_tokens][heads][head_dim] each."""
    shape = (n_tokens, heads, head_dim)
    return tuple(normal_bf16(seed_of(role, stream, chunk, step, layer), shape, device)
                 for role in (ROLE_Q, ROLE_K, ROLE_V))


def latent(stream: int, frames: int, channels: int, height: int, width: int,
           device="cpu") -> torch.Tensor:
    """Initial latent x (the noise end of the flow) for one stream, float32."""
    return normal_f32(seed_of(ROLE_X, stream, frames), (frames, channels, height, width), device)


def velocity(stream: int, chunk: int, step: int, n: int, device="cpu") -> torch.Tensor:
    """A stand-in velocity v for one (chunk, step): float32 of n elements."""
    return normal_f32(seed_of(ROLE_VEL, stream, chunk, step), (n,), device)


def store_fill(stream: int, layer: int, step: int, heads: int, n_keys: int, head_dim: int,
               device="cpu"):
    """Pre-recorded K (already rotated) and V rows for a history that earlier chunks wrote.

    Returns bf16 [heads][n_keys][head_dim] K and V.
    """
    shape = (heads, n_keys, head_dim)
    return (normal_bf16(seed_of(ROLE_STORE_K, stream, layer, step), shape, device),
            normal_bf16(seed_of(ROLE_STORE_V, stream, layer, step), shape, device))


def ragged_fills(n_streams: int, ring_slots: int, seed: int = 0) -> list[int]:
    """Seeded ring fills in 0..ring_slots, one per stream, uniform."""
    out = []
    for i in range(n_streams):
        out.append(_mix32_int(seed_of(0x7F11, seed, i)) % (ring_slots + 1))
    return out


def text_lengths(n_prompts: int, max_len: int = 512, seed: int = 0) -> list[int]:
    """Seeded prompt lengths in 1..max_len, uniform: the real token counts of
    the text contexts that cross-attention reads (padding trimmed)."""
    return [1 + _mix32_int(seed_of(0x7E47, seed, i)) % max_len for i in range(n_prompts)]
