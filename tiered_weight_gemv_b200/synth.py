"""Seeded synthetic inputs: the only code the CUDA path and the CPU oracle both consume.

This module holds none of the method's arithmetic (no tier rule, quantiser or product); it only
draws numbers. Every tensor is a pure function of (seed, tensor_id, shape) and is bit-identical
however it is chunked; on one device it is bit-identical across runs.

Generator (written from its published definition): element i of stream (seed, tensor_id) is the
i-th output of SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014) started from key = mix64(seed * 2^32 + tensor_id):
    z = key + (i + 1) * 0x9E3779B97F4A7C15  (mod 2^64)
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
    z = (z ^ (z >> 27)) * 0x94D049BB133111EB
    out = z ^ (z >> 31)
Uniforms are u = (out >> 11 + 1/2) * 2^-53, in (0, 1), never 0 or 1/2 exactly.
    normal:  Box-Muller on the uniforms of outputs 2i and 2i+1 (fp64), then the target dtype.
    Laplace(0, b): inverse CDF, x = -b * sign(u - 1/2) * ln(1 - 2|u - 1/2|) (fp64 -> fp32).
The pages' workloads are Llama-class weights and activations; the stand-ins are
    weights      bf16(N(0, 0.02))
    activations  fp32 Laplace(0, 1)  (heavy-tailed, like decoder activations)
and shapes follow the decoder blocks named in the design notes.
"""
from __future__ import annotations

import math

import torch

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _s64(v: int) -> int:
    """Unsigned 64-bit constant as the signed int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix64_int(((seed & 0xFFFFFFFF) << 32) | (tensor_id & 0xFFFFFFFF))


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns (torch's >> is arithmetic)."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _splitmix_at(key: int, idx: torch.Tensor) -> torch.Tensor:
    """The idx-th SplitMix64 output (int64 bit pattern) of the stream started at key."""
    z = (idx + 1) * _s64(_GAMMA) + _s64(key)  # int64 arithmetic wraps mod 2^64
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def _uniform_at(key: int, idx: torch.Tensor) -> torch.Tensor:
    out = _splitmix_at(key, idx)
    return (_lsr(out, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


_CHUNK = 1 << 24


def _fill(n: int, device, fn, dtype) -> torch.Tensor:
    out = torch.empty(n, dtype=dtype, device=device)
    for start in range(0, n, _CHUNK):
        stop = min(n, start + _CHUNK)
        idx = torch.arange(start, stop, dtype=torch.int64, device=device)
        out[start:stop] = fn(idx).to(dtype)
    return out


def uniform(shape, seed: int, tensor_id: int, device="cpu") -> torch.Tensor:
    """fp64 uniforms in (0, 1)."""
    n = math.prod(shape)
    key = stream_key(seed, tensor_id)
    return _fill(n, device, lambda i: _uniform_at(key, i), torch.float64).reshape(shape)


def normal(shape, seed: int, tensor_id: int, std: float = 1.0, dtype=torch.float32,
           device="cpu") -> torch.Tensor:
    """N(0, std^2) by Box-Muller, computed in fp64, stored as `dtype` (bf16 rounds to nearest)."""
    n = math.prod(shape)
    key = stream_key(seed, tensor_id)

    def fn(i):
        u1 = _uniform_at(key, 2 * i)
        u2 = _uniform_at(key, 2 * i + 1)
        return std * torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)

    return _fill(n, device, fn, dtype).reshape(shape)


def laplace(shape, seed: int, tensor_id: int, scale: float = 1.0, device="cpu") -> torch.Tensor:
    """fp32 Laplace(0, scale) by inverse CDF in fp64."""
    n = math.prod(shape)
    key = stream_key(seed, tensor_id)

    def fn(i):
        v = _uniform_at(key, i) - 0.5
        return -scale * torch.sign(v) * torch.log1p(-2.0 * v.abs())

    return _fill(n, device, fn, torch.float32).reshape(shape)


def weight(d_out: int, d_in: int, seed: int, tensor_id: int, std: float = 0.02,
           device="cpu") -> torch.Tensor:
    """Row-major [d_out, d_in] bf16 weight, bf16(N(0, std^2)) (the nn.Linear layout)."""
    return normal((d_out, d_in), seed, tensor_id, std=std, dtype=torch.bfloat16, device=device)


def log_uniform(shape, seed: int, tensor_id: int, lo: float, hi: float, device="cpu"):
    """fp64 values with log uniform on [ln lo, ln hi] (per-token activation scales)."""
    u = uniform(shape, seed, tensor_id, device=device)
    return torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))


def silu_gated(gate: torch.Tensor, up: torch.Tensor) -> torch.Tensor:
    """SiLU(gate) * up in fp64: the input of a Llama down projection, built from the block's
    own gate/up outputs. This is input preparation (the nonlinearity between projections), not
    part of the tiered product."""
    g = gate.to(torch.float64)
    return (g / (1.0 + torch.exp(-g)) * up.to(torch.float64)).to(torch.float32)
