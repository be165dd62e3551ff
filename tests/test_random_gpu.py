"""Randomized parity sweep: seeded random formats, group sizes, shapes (ragged in every
dimension) and every path valid for them, against the CPU oracle within the GEMM
tolerance.  Sizes are kept small enough for the float64 reference to stay fast."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
import oracle
from bit_quantized_gemm_quant_b200 import inputs
from _helpers import assert_within_tolerance, reference

pytestmark = pytest.mark.gpu

LAYOUTS = [("q4_0", 32, 4), ("affine", 32, 4), ("affine", 64, 4), ("affine", 128, 4), ("affine", 64, 8),
           ("affine", 32, 8), ("affine", 64, 2), ("affine", 64, 3), ("affine", 128, 6), ("affine", 32, 3)]


def _cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        kind, G, bits = LAYOUTS[rng.integers(len(LAYOUTS))]
        K = int(G * rng.integers(1, max(2, 1536 // G)))
        M = int(rng.choice([rng.integers(1, 33), rng.integers(33, 400)]))
        N = int(rng.integers(1, 400))
        out.append((i, kind, G, bits, M, N, K))
    return out


@pytest.mark.parametrize("case", _cases(40, 2024), ids=lambda c: f"{c[1]}{c[3]}g{c[2]}-{c[4]}x{c[5]}x{c[6]}")
def test_random_transpose1(case):
    i, kind, G, bits, M, N, K = case
    g = inputs.generator(1000 + i)
    if kind == "q4_0":
        w = inputs.weights_fp32(N, K, g).numpy()
        wq, s = oracle.q4_0_quantize(w)
        wb = oracle.q4_0_dequantize(wq, s)
        dev = (torch.from_numpy(wq).cuda(), torch.from_numpy(s.view(np.int16)).cuda().view(torch.float16), None)
    else:
        w = inputs.weights_bf16_valued(N, K, g).numpy()
        wq, s, b = oracle.affine_quantize(w, G, bits)
        wb = oracle.affine_dequantize(wq, s, b, G, bits)
        dev = (torch.from_numpy(wq.view(np.int32)).cuda(), torch.from_numpy(s.view(np.int16)).cuda().view(torch.bfloat16),
               torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16))
    x = inputs.activations_bf16(M, K, g)
    y_ref, a_ref = reference(x, wb)
    fast = kind == "q4_0" or bits in (4, 8)
    paths = ["auto", "dequant_gemm"]
    if (fast and M <= 32) or (not fast and M <= 8):
        paths.append("gemv")
    if fast and K % 64 == 0:
        paths.append("tc_fused")
    for path in paths:
        y = bq.quant_matmul_ex(x.cuda(), *dev, G, bits, True, path)
        torch.cuda.synchronize()
        assert_within_tolerance(y, y_ref, a_ref, f"{case} {path}")
    assert bq.bq_device_status() == 0


@pytest.mark.parametrize("case", _cases(12, 77), ids=lambda c: f"t0-{c[1]}{c[3]}g{c[2]}-{c[4]}x{c[5]}x{c[6]}")
def test_random_transpose0(case):
    i, kind, G, bits, M, N, K = case
    if kind == "q4_0":
        bits = 4
    N = G * max(1, N // G)                     # groups run along N
    K = max(8, K // 8 * 8) if K % 8 else K     # activation rows: 16-byte multiples
    g = inputs.generator(2000 + i)
    w = inputs.weights_bf16_valued(K, N, g).numpy()
    wq, s, b = oracle.affine_quantize(w, G, bits)
    w_ref = np.ascontiguousarray(oracle.affine_dequantize(wq, s, b, G, bits).T)
    x = inputs.activations_bf16(M, K, g)
    y = bq.quant_matmul(x.cuda(), torch.from_numpy(wq.view(np.int32)).cuda(),
                        torch.from_numpy(s.view(np.int16)).cuda().view(torch.bfloat16),
                        torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16), G, bits, transpose=False)
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, w_ref)
    assert_within_tolerance(y, y_ref, a_ref, f"transpose=0 {case}")
