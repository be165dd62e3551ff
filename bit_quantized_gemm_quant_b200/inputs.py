"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the
quantization or matmul arithmetic, so the CPU oracle and the CUDA path can both
be fed from it without sharing any of the method.

Recipe (after the micro-benchmark on the MLX issue page, Repro): weights are
W ~ N(0, 1) * 0.02 in fp32, activations x ~ N(0, 1) cast to bf16; one
``torch.Generator`` seeded per workload draws W first, then x, so every token
count of one workload sees the same W.  For the affine formats W is cast to
bf16 first (the page quantizes a bf16 weight).
"""
from __future__ import annotations

import torch

W_STD = 0.02


def generator(seed: int = 0, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weights_fp32(N: int, K: int, g: torch.Generator, device: str = "cpu") -> torch.Tensor:
    """W[N][K] ~ N(0, 0.02^2), fp32."""
    return torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * W_STD


def weights_bf16_valued(N: int, K: int, g: torch.Generator, device: str = "cpu") -> torch.Tensor:
    """W[N][K] ~ N(0, 0.02^2) cast to bf16 and held as fp32 (input to affine quantization)."""
    return weights_fp32(N, K, g, device).to(torch.bfloat16).to(torch.float32)


def activations_bf16(M: int, K: int, g: torch.Generator, device: str = "cpu") -> torch.Tensor:
    """x[M][K] ~ N(0, 1), bf16."""
    return torch.randn(M, K, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def random_bytes(shape, g: torch.Generator) -> torch.Tensor:
    """Uniform random bytes (arbitrary packed nibbles / codes)."""
    return torch.randint(0, 256, shape, generator=g, dtype=torch.int32).to(torch.uint8)


def random_u32(shape, g: torch.Generator) -> torch.Tensor:
    """Uniform random 32-bit words, returned as int32 with the same bits."""
    lo = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    hi = torch.randint(0, 1 << 16, shape, generator=g, dtype=torch.int64)
    v = (hi << 16) | lo
    return torch.where(v >= (1 << 31), v - (1 << 32), v).to(torch.int32)


def random_f16_bits(shape, g: torch.Generator) -> torch.Tensor:
    """Random finite fp16 bit patterns (normals, subnormals, +-0; no inf/NaN), as int16."""
    sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int64)
    e = torch.randint(0, 31, shape, generator=g, dtype=torch.int64)      # field 31 = inf/NaN
    m = torch.randint(0, 1 << 10, shape, generator=g, dtype=torch.int64)
    v = (sign << 15) | (e << 10) | m
    return torch.where(v >= (1 << 15), v - (1 << 16), v).to(torch.int16)


def random_bf16_bits(shape, g: torch.Generator, exp_lo: int = 0, exp_hi: int = 254) -> torch.Tensor:
    """Random finite bf16 bit patterns with exponent field in [exp_lo, exp_hi]."""
    sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int64)
    e = torch.randint(exp_lo, exp_hi + 1, shape, generator=g, dtype=torch.int64)
    m = torch.randint(0, 128, shape, generator=g, dtype=torch.int64)
    v = (sign << 15) | (e << 7) | m
    return torch.where(v >= (1 << 15), v - (1 << 16), v).to(torch.int16)
