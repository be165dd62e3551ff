"""CPU oracle for weight-only block-quantized matmul.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the smoke check and by the
CPU-baseline leg of ``bench.py``, never by the library's product path.  The
arithmetic lives in ``bq_oracle.c`` (plain C, float64 accumulation, no FMA
contraction); this module only marshals numpy arrays into it.

Parity status of each function (what pins it, see ``tests/test_oracle_pins.py``):
  f32/f16/bf16 conversions  -- numpy / torch conversions, exhaustive or 1M+ values
  q4_0_quantize             -- closed forms: exact round trip, all-zero block,
                               max-abs element -> q = 0, q range, error bound;
                               exact w/d = k - 1/2 ties and the first-max rule
                               (planted variants of the source fail them)
  q4_0_dequantize           -- closed form over every code value with both signs
                               of d, exact round trip of quantize
  q4_0_import_aos           -- blocks assembled byte by byte with numpy from
                               random codes and scales
  affine_quantize           -- closed forms: exact round trip, constant group,
                               min -> 0 / max -> L, error bound (2, 3, 4, 6, 8 bits);
                               exact half-way ties go to even (roundf fails)
  affine_dequantize         -- closed form over every code value, codes laid out
                               by an independent numpy bit-stream packer and a
                               hand-derived 3-bit word; exact round trip of quantize
  q8_1_quantize             -- closed forms: power-of-two scales with exact codes,
                               half-away-from-zero ties, all-zero block, |q| <= 127,
                               qsum, reconstruction error <= d/2
  q4_0_q8_matmul            -- unit scales give numpy's exact integer dot product;
                               within the x-quantization error bound of matmul_ref
  matmul_ref                -- exact rational (fractions.Fraction) brute force
                               on tiny non-square shapes, one-hot identities
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build
        _build.build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    lib.oracle_f32_to_bf16_array.argtypes = [P, P, I64]
    lib.oracle_bf16_to_f32_array.argtypes = [P, P, I64]
    lib.oracle_f32_to_f16_array.argtypes = [P, P, I64]
    lib.oracle_f16_to_f32_array.argtypes = [P, P, I64]
    lib.oracle_q4_0_quantize.argtypes = [P, I64, I64, P, P]
    lib.oracle_q4_0_dequantize.argtypes = [P, P, I64, I64, P]
    lib.oracle_q4_0_import_aos.argtypes = [P, I64, I64, P, P]
    lib.oracle_q8_1_quantize.argtypes = [P, I64, I64, P, P, P]
    lib.oracle_q4_0_q8_matmul.argtypes = [P, P, P, P, I64, I64, I64, P, P]
    lib.oracle_affine_quantize.argtypes = [P, I64, I64, I, I, P, P, P]
    lib.oracle_affine_dequantize.argtypes = [P, P, P, I64, I64, I, I, P]
    lib.oracle_matmul_ref.argtypes = [P, P, I64, I64, I64, P, I64, P, P, I]
    lib.oracle_matmul_ref.restype = I
    for name in ("oracle_f32_to_bf16_array", "oracle_bf16_to_f32_array", "oracle_f32_to_f16_array",
                 "oracle_f16_to_f32_array", "oracle_q4_0_quantize", "oracle_q4_0_dequantize",
                 "oracle_affine_quantize", "oracle_affine_dequantize"):
        getattr(lib, name).restype = None
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# ---------------------------------------------------------------- conversions
def f32_to_bf16(a) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().oracle_f32_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def bf16_to_f32(a) -> np.ndarray:
    a = _c(a, np.uint16)
    out = np.empty(a.shape, np.float32)
    _load().oracle_bf16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


def f32_to_f16(a) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().oracle_f32_to_f16_array(_ptr(a), _ptr(out), a.size)
    return out


def f16_to_f32(a) -> np.ndarray:
    a = _c(a, np.uint16)
    out = np.empty(a.shape, np.float32)
    _load().oracle_f16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


# ---------------------------------------------------------------------- Q4_0
def q4_0_quantize(w) -> tuple[np.ndarray, np.ndarray]:
    """fp32 w[N][K] -> (wq u8 [N][K/2], d fp16 bits u16 [N][K/32])."""
    w = _c(w, np.float32)
    N, K = w.shape
    assert K % 32 == 0
    wq = np.empty((N, K // 2), np.uint8)
    d = np.empty((N, K // 32), np.uint16)
    _load().oracle_q4_0_quantize(_ptr(w), N, K, _ptr(wq), _ptr(d))
    return wq, d


def q4_0_dequantize(wq, d) -> np.ndarray:
    """(wq u8 [N][K/2], d fp16 bits [N][K/32]) -> bf16 bits u16 [N][K]."""
    wq = _c(wq, np.uint8)
    d = _c(d, np.uint16)
    N, K = wq.shape[0], wq.shape[1] * 2
    assert d.shape == (N, K // 32)
    out = np.empty((N, K), np.uint16)
    _load().oracle_q4_0_dequantize(_ptr(wq), _ptr(d), N, K, _ptr(out))
    return out


def q4_0_import_aos(blocks) -> tuple[np.ndarray, np.ndarray]:
    """Array-of-structs Q4_0 blocks u8 [N][K/32 * 18] (fp16 d, then 16 code bytes)
    -> (wq u8 [N][K/2], d fp16 bits u16 [N][K/32])."""
    blocks = _c(blocks, np.uint8)
    N, K = blocks.shape[0], blocks.shape[1] // 18 * 32
    assert blocks.shape[1] == K // 32 * 18
    wq = np.empty((N, K // 2), np.uint8)
    d = np.empty((N, K // 32), np.uint16)
    _load().oracle_q4_0_import_aos(_ptr(blocks), N, K, _ptr(wq), _ptr(d))
    return wq, d


# ------------------------------------------------------- quantized activations
def q8_1_quantize(x_bf16_bits) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """bf16 bits u16 [M][K] -> (xq int8 [M][K], dx f32 [M][K/32], qsum int32 [M][K/32])."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    assert K % 32 == 0
    xq = np.empty((M, K), np.int8)
    dx = np.empty((M, K // 32), np.float32)
    qs = np.empty((M, K // 32), np.int32)
    _load().oracle_q8_1_quantize(_ptr(x), M, K, _ptr(xq), _ptr(dx), _ptr(qs))
    return xq, dx, qs


def q4_0_q8_matmul(xq, dx, wq, d) -> tuple[np.ndarray, np.ndarray]:
    """Q4_0 weights times Q8_1-style activations, float64 from the integer codes:
    -> (y f64 [M][N], a f64 [M][N] = sum of |block terms|)."""
    xq = _c(xq, np.int8)
    dx = _c(dx, np.float32)
    wq = _c(wq, np.uint8)
    d = _c(d, np.uint16)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape == (N, K // 2) and d.shape == (N, K // 32) and dx.shape == (M, K // 32)
    y = np.empty((M, N), np.float64)
    a = np.empty((M, N), np.float64)
    _load().oracle_q4_0_q8_matmul(_ptr(xq), _ptr(dx), _ptr(wq), _ptr(d), M, N, K, _ptr(y), _ptr(a))
    return y, a


# -------------------------------------------------------------------- affine
AFFINE_BITS = (2, 3, 4, 6, 8)


def affine_quantize(w, group_size: int = 64, bits: int = 4):
    """fp32 w[N][K] -> (wq u32 [N][K*bits/32], scales bf16 bits, biases bf16 bits [N][K/group]).
    Codes are a little-endian bit stream per row (code k at stream bits bits*k ..)."""
    assert bits in AFFINE_BITS
    w = _c(w, np.float32)
    N, K = w.shape
    assert K % group_size == 0 and (K * bits) % 32 == 0
    wq = np.empty((N, K * bits // 32), np.uint32)
    s = np.empty((N, K // group_size), np.uint16)
    b = np.empty((N, K // group_size), np.uint16)
    _load().oracle_affine_quantize(_ptr(w), N, K, group_size, bits, _ptr(wq), _ptr(s), _ptr(b))
    return wq, s, b


def affine_dequantize(wq, scales, biases, group_size: int = 64, bits: int = 4) -> np.ndarray:
    assert bits in AFFINE_BITS
    wq = _c(wq, np.uint32)
    scales = _c(scales, np.uint16)
    biases = _c(biases, np.uint16)
    N = wq.shape[0]
    K = wq.shape[1] * 32 // bits
    assert scales.shape == (N, K // group_size) and biases.shape == scales.shape
    out = np.empty((N, K), np.uint16)
    _load().oracle_affine_dequantize(_ptr(wq), _ptr(scales), _ptr(biases), N, K, group_size, bits,
                                     _ptr(out))
    return out


# -------------------------------------------------------------------- matmul
def matmul_ref(x_bf16, w_bf16, rows=None, nthreads: int | None = None):
    """float64 y[r][n] = sum_k x[rows[r]][k] * w[n][k] and a[r][n] = sum_k |x w|.

    x_bf16: u16 [M][K]; w_bf16: u16 [N][K]; rows: optional 1-D int array of
    selected rows of x.  Returns (y, a, threads_used).
    """
    x = _c(x_bf16, np.uint16)
    w = _c(w_bf16, np.uint16)
    M, K = x.shape
    N, K2 = w.shape
    assert K == K2
    if rows is None:
        r = None
        R = M
    else:
        r = _c(rows, np.int64)
        assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < M))
        R = r.size
    y = np.empty((R, N), np.float64)
    a = np.empty((R, N), np.float64)
    nt = nthreads or os.cpu_count() or 1
    used = _load().oracle_matmul_ref(_ptr(x), _ptr(w), M, N, K,
                                     _ptr(r) if r is not None else None, R,
                                     _ptr(y), _ptr(a), nt)
    return y, a, used


def bf16_half_ulp(y: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place of |y| (float64): the largest error the
    output's own round-to-nearest to bf16 (8 significant bits) can add."""
    ay = np.abs(np.asarray(y, np.float64))
    e = np.floor(np.log2(np.where(ay > 0, ay, 1.0)))
    e = np.maximum(e, -126.0)                       # bf16 subnormal spacing below 2^-126
    return np.where(ay > 0, np.exp2(e - 8.0), 0.0)


def tolerance(a: np.ndarray, y_ref: np.ndarray | None = None) -> np.ndarray:
    """Allowed |y_gpu - y_ref| for outputs with absolute-product sums ``a``:
    2e-3 * a + 1e-5 for the accumulation, plus half a bf16 ulp of y_ref for the
    rounding of the bf16 output itself (which alone can reach 2^-8 |y|, above
    2e-3 * a whenever |y| is close to a)."""
    tol = 2e-3 * a + 1e-5
    if y_ref is not None:
        tol = tol + bf16_half_ulp(y_ref)
    return tol
