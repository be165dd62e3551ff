"""Quantized-activation decode path (Q4_0 weights x Q8_1-style int8 activations):
the activation codes bit-exact with the oracle, the matmul within a bound derived
from fp32 scaling and summation of exact integer block dot products, and end to
end within the activation-quantization bound of the exact bf16 product."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
import oracle
from bit_quantized_gemm_quant_b200 import inputs
from _helpers import Problem, u16, reference

pytestmark = pytest.mark.gpu


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,K", [(1, 32), (3, 1024), (8, 4096), (37, 512)])
def test_q8_1_quantize_bit_exact(M, K):
    g = inputs.generator(M * 7 + K)
    x = inputs.activations_bf16(M, K, g)
    x[0, :32] = 0.0                                    # all-zero block: d = 0
    if K >= 64:
        x[-1, 32:64] = torch.arange(-16, 16, dtype=torch.float32).to(torch.bfloat16) * 0.25   # exact ties at .5
    xq_r, dx_r, qs_r = oracle.q8_1_quantize(_bits(x))
    xq, dx, qs = bq.q8_1_quantize(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), xq_r)
    assert np.array_equal(dx.cpu().numpy().view(np.uint32), dx_r.view(np.uint32))
    assert np.array_equal(qs.cpu().numpy(), qs_r)


def test_q8_1_quantize_random_bits():
    """Random normal bf16 bit patterns, both signs, exponents over the whole range (a
    block whose largest magnitude is below 127 * 2^-128 would overflow 1/d; not tested)."""
    g = inputs.generator(31)
    bits = inputs.random_bf16_bits((6, 2048), g, 1, 254).numpy().view(np.uint16)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    xq_r, dx_r, qs_r = oracle.q8_1_quantize(bits)
    xq, dx, qs = bq.q8_1_quantize(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), xq_r)
    assert np.array_equal(dx.cpu().numpy().view(np.uint32), dx_r.view(np.uint32))
    assert np.array_equal(qs.cpu().numpy(), qs_r)


def _q8_tolerance(a: np.ndarray, y_ref: np.ndarray, K: int) -> np.ndarray:
    # each block term: two fp32 roundings (scale product, product with the exact
    # integer); the sum over K/32 blocks and the quad's two shuffle additions add
    # one rounding each of at most the running |sum| <= a
    nb = K // 32
    return (nb + 8) * 2.0 ** -24 * a + oracle.bf16_half_ulp(y_ref) + 1e-30


@pytest.mark.parametrize("M,N,K", [(1, 300, 1024), (3, 250, 4096), (13, 40, 512), (8, 12288, 4096)])
def test_quant_matmul_q8_vs_oracle(M, N, K):
    p = Problem("q4_0", N, K, seed=M + N + K)
    wq, s, _ = p.device()
    x = p.x(M)
    xq_r, dx_r, _ = oracle.q8_1_quantize(_bits(x))
    xq, dx, qs = bq.q8_1_quantize(x.cuda())
    y = bq.quant_matmul_q8(xq, dx, qs, wq, s)
    torch.cuda.synchronize()
    rows = slice(None) if N <= 1000 else np.r_[0:64, N - 64:N]
    y_ref, a = oracle.q4_0_q8_matmul(xq_r, dx_r, p.wq[rows], p.scales[rows])
    got = y.float().cpu().numpy().astype(np.float64)[:, rows]
    assert np.all(np.abs(got - y_ref) <= _q8_tolerance(a, y_ref, K))


def test_quant_matmul_q8_within_activation_bound_of_exact_product():
    """End to end against the exact bf16 product of quant_matmul's definition:
    at most dx/2 * |w| per term plus the bf16 rounding of the weights."""
    M, N, K = 4, 500, 2048
    p = Problem("q4_0", N, K, seed=77)
    wq, s, _ = p.device()
    x = p.x(M)
    xq, dx, qs = bq.q8_1_quantize(x.cuda())
    y = bq.quant_matmul_q8(xq, dx, qs, wq, s)
    torch.cuda.synchronize()
    y_exact, a_exact = reference(x, p.wb)
    wabs = np.abs((p.wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    dxn = dx.cpu().numpy().astype(np.float64)
    bound = (np.repeat(dxn, 32, axis=1) / 2) @ wabs.T + 2.0 ** -9 * a_exact * 1.01 \
        + oracle.bf16_half_ulp(y_exact) + 1e-5 * a_exact
    assert np.all(np.abs(y.float().cpu().numpy().astype(np.float64) - y_exact) <= bound)


def test_quant_matmul_q8_deterministic_and_empty():
    p = Problem("q4_0", 300, 1024, seed=5)
    wq, s, _ = p.device()
    xq, dx, qs = bq.q8_1_quantize(p.x(3).cuda())
    ys = [u16(bq.quant_matmul_q8(xq, dx, qs, wq, s)) for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    assert bq.lib().quant_matmul_q8(None, None, None, None, None, None, 0, 300, 1024, None) == 0
