"""Shared helpers for the GPU parity tests: seeded problems quantized by the CPU
oracle, uploaded to the device, and the oracle's float64 reference."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_quantized_gemm_quant_b200 import inputs

FMT = {"q4_0": (32, 4), "affine4": (64, 4), "affine8": (64, 8),
       "affine4_g32": (32, 4), "affine4_g128": (128, 4), "affine8_g32": (32, 8), "affine8_g128": (128, 8),
       "affine2": (64, 2), "affine3": (64, 3), "affine6": (64, 6),
       "affine2_g32": (32, 2), "affine3_g32": (32, 3), "affine3_g128": (128, 3), "affine6_g32": (32, 6)}


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Problem:
    """Quantized weight W[N][K] of one format, its oracle dequantization, and x[M][K]."""

    def __init__(self, fmt: str, N: int, K: int, seed: int = 0, w: np.ndarray | None = None):
        self.fmt, self.N, self.K = fmt, N, K
        self.group_size, self.bits = FMT[fmt]
        self.g = inputs.generator(seed)
        if w is None:
            wt = inputs.weights_fp32(N, K, self.g) if fmt == "q4_0" else inputs.weights_bf16_valued(N, K, self.g)
            w = wt.numpy()
        self.w = np.ascontiguousarray(w, np.float32)
        if fmt == "q4_0":
            self.wq, self.scales = oracle.q4_0_quantize(self.w)
            self.biases = None
            self.wb = oracle.q4_0_dequantize(self.wq, self.scales)
        else:
            self.wq, self.scales, self.biases = oracle.affine_quantize(self.w, self.group_size, self.bits)
            self.wb = oracle.affine_dequantize(self.wq, self.scales, self.biases, self.group_size, self.bits)

    def device(self, dev="cuda"):
        wq = torch.from_numpy(self.wq.view(np.int32) if self.fmt != "q4_0" else self.wq).to(dev)
        sdt = torch.float16 if self.fmt == "q4_0" else torch.bfloat16
        s = torch.from_numpy(self.scales.view(np.int16)).to(dev).view(sdt)
        b = None if self.biases is None else torch.from_numpy(self.biases.view(np.int16)).to(dev).view(torch.bfloat16)
        return wq, s, b

    def x(self, M: int) -> torch.Tensor:
        return inputs.activations_bf16(M, self.K, self.g)


def reference(x_bf16: torch.Tensor, wb: np.ndarray, rows=None):
    y, a, _ = oracle.matmul_ref(u16(x_bf16), wb, rows=rows)
    return y, a


def assert_within_tolerance(y_gpu: torch.Tensor, y_ref: np.ndarray, a_ref: np.ndarray, what: str = ""):
    got = y_gpu.float().cpu().numpy().astype(np.float64)
    assert got.shape == y_ref.shape, (got.shape, y_ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - y_ref)
    tol = oracle.tolerance(a_ref, y_ref)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outputs out of tolerance; worst at {i}: "
                             f"gpu {got[i]!r} ref {y_ref[i]!r} tol {tol[i]!r}")
