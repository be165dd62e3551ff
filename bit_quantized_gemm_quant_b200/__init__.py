"""Thin Python binding of libbqgemm (include/bqgemm.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; PyTorch
provides device memory and the current stream.  There is no CPU fallback: the
first call raises if libbqgemm.so is missing or the device is not sm_100.

Names follow the C ABI: q4_0_dequantize, affine_dequantize, quant_matmul,
quant_matmul_ex, bf16_matmul, q4_0_quantize, affine_quantize,
quant_matmul_select_path, quant_matmul_workspace_size, bq_device_status.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbqgemm.so")

BQ_OK = 0
STATUS = {0: "BQ_OK", 1: "BQ_ERR_NULL", 2: "BQ_ERR_SHAPE", 3: "BQ_ERR_UNSUPPORTED", 4: "BQ_ERR_ALIGN",
          5: "BQ_ERR_CUDA", 6: "BQ_ERR_TIMEOUT", 7: "BQ_ERR_WORKSPACE", 8: "BQ_ERR_DEVICE"}
PATH_AUTO, PATH_GEMV, PATH_TC_FUSED, PATH_DEQUANT_GEMM, PATH_GEMV_STREAM = 0, 1, 2, 3, 4
PATHS = {"auto": PATH_AUTO, "gemv": PATH_GEMV, "tc_fused": PATH_TC_FUSED, "dequant_gemm": PATH_DEQUANT_GEMM,
         "gemv_stream": PATH_GEMV_STREAM}

_lib = None


class BqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded libbqgemm.so (loaded on first use; raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbqgemm.so not found at {LIB_PATH}; build it with "
                           "`python -c 'import __graft_entry__ as g; g.build()'` (no CPU fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sigs = {
        "q4_0_dequantize": [P, P, P, I64, I64, P],
        "q4_0_import_aos": [P, P, P, I64, I64, P],
        "q8_1_quantize": [P, P, P, P, I64, I64, P],
        "quant_matmul_q8": [P, P, P, P, P, P, I64, I64, I64, P],
        "affine_dequantize": [P, P, P, P, I64, I64, I, I, P],
        "quant_matmul": [P, P, P, P, P, I64, I64, I64, I, I, I, P],
        "quant_matmul_ex": [P, P, P, P, P, I64, I64, I64, I, I, I, I, P, SZ, P],
        "quant_matmul_noalloc": [P, P, P, P, P, I64, I64, I64, I, I, I, P],
        "quant_matmul_multi": [P, I, P, P, P, P, P, I64, I64, I, I, I, P],
        "quant_matmul_workspace_size": [I64, I64, I64, I, I, I],
        "quant_matmul_gemv_kernel": [I64, I64, I64, I, I, I],
        "quant_matmul_select_path": [I64, I64, I64, I, I],
        "bf16_matmul": [P, P, P, I64, I64, I64, P],
        "q4_0_quantize": [P, P, P, I64, I64, P],
        "affine_quantize": [P, P, P, P, I64, I64, I, I, P],
        "bq_device_status": [],
        "bq_selftest_wait_timeout": [ctypes.c_longlong, P],
        "bq_status_string": [I],
        "bq_version": [],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = I
    L.quant_matmul_workspace_size.restype = SZ
    L.bq_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != BQ_OK:
        raise BqError(status, where)


_EMPTY_TAG = ctypes.c_void_p(16)   # non-NULL, 16-byte aligned, never dereferenced (empty tensor)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if t.numel() == 0:
        # an empty tensor has no storage; a NULL biases pointer would select Q4_0
        return _EMPTY_TAG
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _bits16(t: torch.Tensor) -> torch.Tensor:
    """bf16 / fp16 / int16 tensors are passed by their 16-bit patterns."""
    if t.dtype not in (torch.bfloat16, torch.float16, torch.int16, torch.uint16):
        raise TypeError(f"expected a 16-bit tensor, got {t.dtype}")
    return t


BF16 = (torch.bfloat16, torch.int16, torch.uint16)      # bf16 values or their bit patterns
BITS16 = (torch.bfloat16, torch.float16, torch.int16, torch.uint16)
U8 = (torch.uint8, torch.int8)
U32 = (torch.int32, torch.uint32)


def _arg(t: torch.Tensor | None, dtypes, elems: int, name: str):
    """The pointer of `t` after checking its type and that it holds at least `elems`
    elements: the library reads and writes by the sizes it is given, so a tensor of
    the wrong type or too small would be read or written out of bounds."""
    if t is None:
        return None
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: expected one of {[str(d) for d in dtypes]}, got {t.dtype}")
    if t.numel() < elems:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {elems}")
    return _ptr(t)


def _weights_args(wq, scales, biases, N: int, K: int, group_size: int, bits: int, transpose: bool, i=""):
    """Checked pointers of one quantized matrix: Q4_0 (biases None) u8 codes [N][K/2]
    with 16-bit scales [N][K/32]; affine u32 codes with bf16 scales and biases,
    [N][K bits/32] and [N][K/group] (transpose), else [K][N bits/32] and [K][N/group]."""
    if biases is None:
        return (_arg(wq, U8, N * (K // 2), f"wq{i}"), _arg(scales, BITS16, N * (K // 32), f"scales{i}"), None)
    g = max(group_size, 1)
    ng = N * (K // g) if transpose else K * (N // g)
    return (_arg(wq, U32, N * K * bits // 32, f"wq{i}"), _arg(scales, BITS16, ng, f"scales{i}"),
            _arg(biases, BITS16, ng, f"biases{i}"))


# ----------------------------------------------------------------- dequantize
def q4_0_dequantize(wq: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """wq u8 [N][K/2], scales fp16 [N][K/32] -> bf16 [N][K]."""
    N, K = wq.shape[0], wq.shape[1] * 2
    if out is None:
        out = torch.empty(N, K, dtype=torch.bfloat16, device=wq.device)
    _check(lib().q4_0_dequantize(_arg(wq, U8, N * K // 2, "wq"), _arg(scales, BITS16, N * (K // 32), "scales"),
                                 _arg(out, BF16, N * K, "out"), N, K, _stream(stream)),
           "q4_0_dequantize")
    return out


def q4_0_import_aos(blocks: torch.Tensor, stream=None):
    """Array-of-structs Q4_0 blocks u8 [N][K/32 * 18] (fp16 d, then 16 code bytes)
    -> (wq u8 [N][K/2], scales fp16 [N][K/32])."""
    N, K = blocks.shape[0], blocks.shape[1] // 18 * 32
    if blocks.dtype != torch.uint8 or blocks.shape[1] != K // 32 * 18:
        raise ValueError("blocks must be u8 [N][K/32 * 18]")
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=blocks.device)
    scales = torch.empty(N, K // 32, dtype=torch.float16, device=blocks.device)
    _check(lib().q4_0_import_aos(_ptr(blocks), _ptr(wq), _ptr(scales), N, K, _stream(stream)), "q4_0_import_aos")
    return wq, scales


def affine_dequantize(wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, group_size: int = 64,
                      bits: int = 4, out: torch.Tensor | None = None, stream=None):
    """wq u32 (int32) [N][K*bits/32], scales/biases bf16 [N][K/group_size] -> bf16 [N][K]."""
    N, K = wq.shape[0], wq.shape[1] * 32 // bits
    if out is None:
        out = torch.empty(N, K, dtype=torch.bfloat16, device=wq.device)
    ng = N * (K // max(group_size, 1))
    _check(lib().affine_dequantize(_arg(wq, U32, N * K * bits // 32, "wq"), _arg(scales, BITS16, ng, "scales"),
                                   _arg(biases, BITS16, ng, "biases"), _arg(out, BF16, N * K, "out"), N, K,
                                   group_size, bits, _stream(stream)), "affine_dequantize")
    return out


# --------------------------------------------------------------------- matmul
def _k_of(wq: torch.Tensor, biases, bits: int) -> int:
    if biases is None:
        return wq.shape[1] * 2
    return wq.shape[1] * 32 // bits


def _nk_of(wq: torch.Tensor, biases, bits: int, transpose: bool) -> tuple[int, int]:
    """(N, K) of the weights: [N][K] packed along K (transpose), else [K][N] packed along N."""
    if transpose:
        return wq.shape[0], _k_of(wq, biases, bits)
    return _k_of(wq, biases, bits), wq.shape[0]


def quant_matmul(x: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor | None = None,
                 group_size: int = 32, bits: int = 4, transpose: bool = True, out: torch.Tensor | None = None,
                 stream=None):
    """y[M][N] = x[M][K] . dequant(W)[N][K]^T (biases None: Q4_0); transpose=False:
    y = x . dequant(W) with affine W [K][N] packed and grouped along N."""
    return quant_matmul_ex(x, wq, scales, biases, group_size, bits, transpose, "auto", out=out, stream=stream)


def quant_matmul_ex(x: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor | None = None,
                    group_size: int = 32, bits: int = 4, transpose: bool = True, path="auto",
                    workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None):
    M, K = x.shape
    N, Kw = _nk_of(wq, biases, bits, transpose)
    if K != Kw:
        raise ValueError(f"K mismatch: x has {K}, weights hold {Kw}")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    p = PATHS[path] if isinstance(path, str) else int(path)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    fn = lib().quant_matmul_ex if (p != PATH_AUTO or workspace is not None) else None
    xp, yp = _arg(x, BF16, M * K, "x"), _arg(out, BF16, M * N, "out")
    wp, sp, bp = _weights_args(wq, scales, biases, N, K, group_size, bits, transpose)
    if fn is None:
        st = lib().quant_matmul(xp, wp, sp, bp, yp, M, N, K, group_size, bits, 1 if transpose else 0,
                                _stream(stream))
    else:
        st = fn(xp, wp, sp, bp, yp, M, N, K, group_size, bits, 1 if transpose else 0, p, _ptr(workspace), ws_bytes,
                _stream(stream))
    _check(st, "quant_matmul")
    return out


def quant_matmul_multi(x: torch.Tensor, weights, group_size: int = 32, bits: int = 4, transpose: bool = True,
                       outs=None, stream=None):
    """Several quantized matmuls sharing x: weights = [(wq, scales, biases|None), ...]
    (at most 8, one format); returns [y_i bf16 [M][N_i]].  Decode sizes run as one launch."""
    M, K = x.shape
    count = len(weights)
    q4 = weights[0][2] is None
    if any((b is None) != q4 for _, _, b in weights):
        raise ValueError("all matrices must be Q4_0 (biases None) or all affine")
    Ns = [wq.shape[0] for wq, _, _ in weights]
    for wq, _, b in weights:
        if K != _k_of(wq, b, bits):
            raise ValueError("K mismatch between x and a weight matrix")
    if outs is None:
        outs = [torch.empty(M, n, dtype=torch.bfloat16, device=x.device) for n in Ns]
    VP = ctypes.c_void_p * max(count, 1)
    args = [_weights_args(wq, sc, b, n, K, group_size, bits, True, f"[{i}]")
            for i, ((wq, sc, b), n) in enumerate(zip(weights, Ns))]
    wq_a = VP(*[a[0] for a in args])
    s_a = VP(*[a[1] for a in args])
    b_a = None if q4 else VP(*[a[2] for a in args])
    y_a = VP(*[_arg(y, BF16, M * n, f"outs[{i}]") for i, (y, n) in enumerate(zip(outs, Ns))])
    n_a = (ctypes.c_int64 * max(count, 1))(*Ns)
    _check(lib().quant_matmul_multi(_arg(x, BF16, M * K, "x"), count, wq_a, s_a, b_a, y_a, n_a, M, K, group_size, bits,
                                    1 if transpose else 0, _stream(stream)), "quant_matmul_multi")
    return outs


def q8_1_quantize(x: torch.Tensor, stream=None):
    """bf16 x [M][K] -> (xq int8 [M][K], dx f32 [M][K/32], qsum int32 [M][K/32])."""
    M, K = x.shape
    xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
    dx = torch.empty(M, K // 32, dtype=torch.float32, device=x.device)
    qs = torch.empty(M, K // 32, dtype=torch.int32, device=x.device)
    _check(lib().q8_1_quantize(_arg(x, BF16, M * K, "x"), _ptr(xq), _ptr(dx), _ptr(qs), M, K, _stream(stream)), "q8_1_quantize")
    return xq, dx, qs


def quant_matmul_q8(xq: torch.Tensor, dx: torch.Tensor, qsum: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor,
                    out: torch.Tensor | None = None, stream=None):
    """Q4_0 weights times quantized activations -> bf16 y [M][N]."""
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] * 2 != K:
        raise ValueError("K mismatch between activations and weights")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=xq.device)
    _check(lib().quant_matmul_q8(_arg(xq, (torch.int8,), M * K, "xq"), _arg(dx, (torch.float32,), M * (K // 32), "dx"),
                                 _arg(qsum, (torch.int32,), M * (K // 32), "qsum"), _arg(wq, U8, N * K // 2, "wq"),
                                 _arg(scales, BITS16, N * (K // 32), "scales"), _arg(out, BF16, M * N, "out"), M, N,
                                 K, _stream(stream)), "quant_matmul_q8")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def quant_matmul_noalloc(x: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor | None,
                         out: torch.Tensor, group_size: int = 32, bits: int = 4, transpose: bool = True, stream=None):
    """quant_matmul for callers that must not allocate: the library uses its fixed
    32 MiB device scratch (N * K <= 16 Mi weights) and allocates nothing.  `out`
    (bf16 [M][N]) is required, since creating it here would allocate."""
    M, K = x.shape
    N, Kw = _nk_of(wq, biases, bits, transpose)
    if K != Kw:
        raise ValueError(f"K mismatch: x has {K}, weights hold {Kw}")
    if tuple(out.shape) != (M, N) or out.dtype != torch.bfloat16:
        raise ValueError("out must be a bf16 tensor of shape [M][N]")
    wp, sp, bp = _weights_args(wq, scales, biases, N, K, group_size, bits, transpose)
    _check(lib().quant_matmul_noalloc(_arg(x, BF16, M * K, "x"), wp, sp, bp, _arg(out, BF16, M * N, "out"), M, N, K,
                                      group_size, bits, 1 if transpose else 0, _stream(stream)),
           "quant_matmul_noalloc")
    return out


def quant_matmul_select_path(M: int, N: int, K: int, group_size: int, bits: int) -> int:
    return lib().quant_matmul_select_path(M, N, K, group_size, bits)


GEMV_KERNELS = {0: "gemv_kernel", 1: "gemv_tma_kernel", 2: "gemv_int_prep_kernel + gemv_stream_kernel",
                3: "gemv_affine_kernel"}


def quant_matmul_gemv_kernel(M: int, N: int, K: int, group_size: int, bits: int, path="auto") -> int:
    """Which decode kernel runs (GEMV_KERNELS), -1 off the decode path (host only)."""
    p = PATHS[path] if isinstance(path, str) else int(path)
    return lib().quant_matmul_gemv_kernel(M, N, K, group_size, bits, p)


def quant_matmul_workspace_size(M: int, N: int, K: int, group_size: int, bits: int, path="auto") -> int:
    p = PATHS[path] if isinstance(path, str) else int(path)
    return lib().quant_matmul_workspace_size(M, N, K, group_size, bits, p)


def bf16_matmul(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """y[M][N] = x[M][K] . w[N][K]^T, bf16 in/out, fp32 accumulation (tcgen05)."""
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _check(lib().bf16_matmul(_arg(x, BF16, M * K, "x"), _arg(w, BF16, N * K, "w"), _arg(out, BF16, M * N, "out"),
                             M, N, K, _stream(stream)), "bf16_matmul")
    return out


# ------------------------------------------------------------------- quantize
def q4_0_quantize(w: torch.Tensor, stream=None):
    """fp32 w [N][K] -> (wq u8 [N][K/2], scales fp16 [N][K/32])."""
    N, K = w.shape
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device)
    d = torch.empty(N, K // 32, dtype=torch.float16, device=w.device)
    _check(lib().q4_0_quantize(_arg(w, (torch.float32,), N * K, "w"), _ptr(wq), _ptr(d), N, K, _stream(stream)),
           "q4_0_quantize")
    return wq, d


def affine_quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4, stream=None):
    """fp32 w [N][K] -> (wq int32 [N][K*bits/32], scales bf16, biases bf16 [N][K/group_size])."""
    N, K = w.shape
    wq = torch.empty(N, K * bits // 32, dtype=torch.int32, device=w.device)
    s = torch.empty(N, K // group_size, dtype=torch.bfloat16, device=w.device)
    b = torch.empty(N, K // group_size, dtype=torch.bfloat16, device=w.device)
    _check(lib().affine_quantize(_arg(w, (torch.float32,), N * K, "w"), _ptr(wq), _ptr(s), _ptr(b), N, K, group_size,
                                 bits, _stream(stream)),
           "affine_quantize")
    return wq, s, b


def bq_device_status() -> int:
    """Synchronize the device and return (and clear) the library's device error status."""
    return lib().bq_device_status()
