"""Named synthetic workloads (shapes only).

Shapes follow the pages' workloads: the 12288 x 4096 MLP up-projection at
1..8192 tokens of the MLX issue ("quantized_matmul takes 14-41% longer than
dequantize + bf16 matmul at prefill sizes (> 512 tokens)", Repro), and the
Llama-3.2-1B prefill / decode of "et-backend: Q4_0 matrix-engine GEMM rewrite
for prefill" (Overview), taken as its projection stack.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str                 # "q4_0" | "affine4" | "affine8"
    N: int
    K: int
    Ms: tuple
    seed: int = 0
    group_size: int = 32
    bits: int = 4


Q4_0_SMALL = Workload("q4_0_small_m16_n256_k512", "q4_0", 256, 512, (16,), group_size=32, bits=4)
Q4_0_DECODE = Workload("q4_0_decode_n12288_k4096", "q4_0", 12288, 4096, (1, 8, 32), group_size=32, bits=4)
AFFINE4_PREFILL = Workload("affine4_g64_n12288_k4096", "affine4", 12288, 4096, (512, 2048, 8192),
                           group_size=64, bits=4)
AFFINE8_SWEEP = Workload("affine8_g64_n12288_k4096", "affine8", 12288, 4096, (1, 32, 512, 2048, 8192),
                         group_size=64, bits=8)

# Llama-3.2-1B projection shapes (N, K) per layer: q, k, v, o, gate, up, down.
LLAMA_1B_LAYER = ((2048, 2048), (512, 2048), (512, 2048), (2048, 2048),
                  (8192, 2048), (8192, 2048), (2048, 8192))
LLAMA_1B_LAYERS = 16


@dataclass(frozen=True)
class StackWorkload:
    name: str
    shapes: tuple = field(default=LLAMA_1B_LAYER)
    layers: int = LLAMA_1B_LAYERS
    Ms: tuple = (512, 1)
    seed: int = 0


LLAMA_1B_STACK = StackWorkload("llama3.2_1b_q4_0_projection_stack")

ALL = {w.name: w for w in (Q4_0_SMALL, Q4_0_DECODE, AFFINE4_PREFILL, AFFINE8_SWEEP)}


def packed_weight_bytes(fmt: str, N: int, K: int, group_size: int) -> int:
    """Bytes of packed codes + scales (+ biases) that one pass over W must read."""
    if fmt == "q4_0":
        return N * K // 2 + N * (K // 32) * 2
    bits = 4 if fmt == "affine4" else 8
    return N * K * bits // 8 + 2 * N * (K // group_size) * 2
