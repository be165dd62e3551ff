"""GPU dequantize and quantize kernels vs the CPU oracle: bit-exact (integer
codes, fp16/bf16 scale bits and bf16 outputs compared as bit patterns, sign of
zero included)."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
import oracle
from bit_quantized_gemm_quant_b200 import inputs
from _helpers import Problem, u16
import _ties

pytestmark = pytest.mark.gpu

SHAPES = [(1, 64), (3, 128), (250, 192), (256, 512), (64, 4096)]


def _gpu_dequant(p: Problem):
    wq, s, b = p.device()
    if p.fmt == "q4_0":
        out = bq.q4_0_dequantize(wq, s)
    else:
        out = bq.affine_dequantize(wq, s, b, p.group_size, p.bits)
    torch.cuda.synchronize()
    return u16(out)


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
@pytest.mark.parametrize("N,K", SHAPES)
def test_dequant_bit_exact(fmt, N, K):
    p = Problem(fmt, N, K, seed=N + K)
    assert np.array_equal(_gpu_dequant(p), p.wb)


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_dequant_bit_exact_full_size(fmt):
    p = Problem(fmt, 12288, 4096)
    assert np.array_equal(_gpu_dequant(p), p.wb)


def test_q4_0_dequant_random_codes_and_scale_bits():
    """Arbitrary bytes and arbitrary finite fp16 scales (subnormals, negatives, +-0)."""
    g = inputs.generator(21)
    N, K = 300, 1024
    wq = inputs.random_bytes((N, K // 2), g).numpy()
    d = inputs.random_f16_bits((N, K // 32), g).numpy().view(np.uint16)
    ref = oracle.q4_0_dequantize(wq, d)
    out = bq.q4_0_dequantize(torch.from_numpy(wq).cuda(), torch.from_numpy(d.view(np.int16)).cuda().view(torch.float16))
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_affine_dequant_random_codes_and_scale_bits(bits):
    g = inputs.generator(22 + bits)
    N, K = 300, 1024
    wq = inputs.random_u32((N, K * bits // 32), g).numpy()
    s = inputs.random_bf16_bits((N, K // 64), g, 100, 140).numpy().view(np.uint16)
    b = inputs.random_bf16_bits((N, K // 64), g, 100, 140).numpy().view(np.uint16)
    ref = oracle.affine_dequantize(wq.view(np.uint32), s, b, 64, bits)
    out = bq.affine_dequantize(torch.from_numpy(wq).cuda(), torch.from_numpy(s.view(np.int16)).cuda().view(torch.bfloat16),
                               torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16), 64, bits)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), ref)


def test_dequant_empty():
    wq = torch.zeros(0, 16, dtype=torch.uint8, device="cuda")
    d = torch.zeros(0, 1, dtype=torch.float16, device="cuda")
    out = bq.q4_0_dequantize(wq, d)
    assert out.shape == (0, 32)


# ------------------------------------------------------------------ quantize
@pytest.mark.parametrize("N,K", [(3, 64), (250, 512), (12288, 4096)])
def test_q4_0_quantize_bit_exact(N, K):
    g = inputs.generator(N)
    w = inputs.weights_fp32(N, K, g)
    w[0, :32] = 0.0                      # all-zero block
    w[min(1, N - 1), 32:64] = 0.01       # all-equal block (first index wins)
    w[min(2, N - 1), 0] = -w[min(2, N - 1), 1].abs() - 0.1
    w[min(2, N - 1), 1] = -w[min(2, N - 1), 0]   # max-abs tie with opposite signs
    wq_ref, d_ref = oracle.q4_0_quantize(w.numpy())
    wq, d = bq.q4_0_quantize(w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), wq_ref)
    assert np.array_equal(u16(d), d_ref)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(3, 64), (250, 512), (12288, 4096)])
def test_affine_quantize_bit_exact(bits, N, K):
    g = inputs.generator(N + bits)
    w = inputs.weights_bf16_valued(N, K, g)
    w[0, :64] = -0.375                   # constant group: scale 0
    wq_ref, s_ref, b_ref = oracle.affine_quantize(w.numpy(), 64, bits)
    wq, s, b = bq.affine_quantize(w.cuda(), 64, bits)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), wq_ref)
    assert np.array_equal(u16(s), s_ref)
    assert np.array_equal(u16(b), b_ref)


def test_q4_0_quantize_division_ties():
    """Blocks whose elements divide to k - 1/2 exactly (code k): the device
    quantizer divides by the fp32 d exactly as the pinned oracle does."""
    w, q = _ties.q4_0_tie_matrix()
    wq_ref, d_ref = oracle.q4_0_quantize(w)
    wq, d = bq.q4_0_quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), wq_ref)
    assert np.array_equal(u16(d), d_ref)
    got = wq.cpu().numpy()
    assert np.array_equal(np.concatenate([got & 15, got >> 4], axis=1), q)


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_affine_quantize_ties_to_even(bits):
    """(w - bias)/scale = j + 1/2 exactly: the device quantizer takes the even code."""
    w, _, q = _ties.affine_tie_matrix(bits)
    wq_ref, s_ref, b_ref = oracle.affine_quantize(w, 64, bits)
    wq, s, b = bq.affine_quantize(torch.from_numpy(w).cuda(), 64, bits)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), wq_ref)
    assert np.array_equal(u16(s), s_ref)
    assert np.array_equal(u16(b), b_ref)


@pytest.mark.parametrize("N,K", [(1, 32), (3, 96), (250, 1024), (37, 4096), (12288, 4096)])
def test_q4_0_import_aos_bit_exact(N, K):
    """Random 18-byte blocks (random fp16 scale bits and code bytes), split on the GPU
    and by the oracle: identical bytes.  Block counts cover whole 32-block warp
    chunks and ragged tails."""
    g = inputs.generator(N + K)
    blocks = inputs.random_bytes((N, K // 32 * 18), g)
    wq_ref, d_ref = oracle.q4_0_import_aos(blocks.numpy())
    wq, d = bq.q4_0_import_aos(blocks.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), wq_ref)
    assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16), d_ref)


def test_q4_0_import_aos_then_matmul():
    """Blocks assembled from an oracle quantization feed quant_matmul after import."""
    N, K, M = 300, 1024, 16
    g = inputs.generator(4)
    w = inputs.weights_fp32(N, K, g).numpy()
    wq, d = oracle.q4_0_quantize(w)
    blocks = np.empty((N, K // 32, 18), np.uint8)
    blocks[:, :, 0] = d & 0xFF
    blocks[:, :, 1] = d >> 8
    blocks[:, :, 2:] = wq.reshape(N, K // 32, 16)
    wq_d, d_d = bq.q4_0_import_aos(torch.from_numpy(blocks.reshape(N, -1)).cuda())
    x = inputs.activations_bf16(M, K, g)
    y = bq.quant_matmul(x.cuda(), wq_d, d_d, None, 32, 4)
    torch.cuda.synchronize()
    y_ref, a_ref, _ = oracle.matmul_ref(x.view(torch.int16).numpy().view(np.uint16), oracle.q4_0_dequantize(wq, d))
    tol = oracle.tolerance(a_ref, y_ref)
    assert np.all(np.abs(y.float().cpu().numpy().astype(np.float64) - y_ref) <= tol)


GROUP_FORMATS = ["affine4_g32", "affine4_g128", "affine8_g32", "affine8_g128"]


@pytest.mark.parametrize("fmt", GROUP_FORMATS)
@pytest.mark.parametrize("N,K", [(3, 128), (250, 512), (64, 4096)])
def test_dequant_bit_exact_group_sizes(fmt, N, K):
    p = Problem(fmt, N, K, seed=N + K + 3)
    assert np.array_equal(_gpu_dequant(p), p.wb)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G", [32, 128])
def test_affine_quantize_bit_exact_group_sizes(bits, G):
    N, K = 250, 1024
    g = inputs.generator(N + bits + G)
    w = inputs.weights_bf16_valued(N, K, g)
    w[0, :G] = -0.375                    # constant group: scale 0
    wq_ref, s_ref, b_ref = oracle.affine_quantize(w.numpy(), G, bits)
    wq, s, b = bq.affine_quantize(w.cuda(), G, bits)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), wq_ref)
    assert np.array_equal(u16(s), s_ref)
    assert np.array_equal(u16(b), b_ref)


NEW_WIDTHS = ["affine2", "affine3", "affine6", "affine2_g32", "affine3_g128", "affine6_g32"]


@pytest.mark.parametrize("fmt", NEW_WIDTHS)
@pytest.mark.parametrize("N,K", [(3, 128), (250, 512), (64, 4096)])
def test_dequant_bit_exact_2_3_6_bits(fmt, N, K):
    p = Problem(fmt, N, K, seed=N + K + 5)
    assert np.array_equal(_gpu_dequant(p), p.wb)


@pytest.mark.parametrize("bits", [2, 3, 6])
def test_affine_dequant_random_codes_2_3_6_bits(bits):
    """Arbitrary code words (3- and 6-bit codes crossing words) and scale bits."""
    g = inputs.generator(40 + bits)
    N, K, G = 300, 1024, 64
    wq = inputs.random_u32((N, K * bits // 32), g).numpy()
    s = inputs.random_bf16_bits((N, K // G), g, 100, 140).numpy().view(np.uint16)
    b = inputs.random_bf16_bits((N, K // G), g, 100, 140).numpy().view(np.uint16)
    ref = oracle.affine_dequantize(wq.view(np.uint32), s, b, G, bits)
    out = bq.affine_dequantize(torch.from_numpy(wq).cuda(), torch.from_numpy(s.view(np.int16)).cuda().view(torch.bfloat16),
                               torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16), G, bits)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), ref)


@pytest.mark.parametrize("bits", [2, 3, 6])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_affine_quantize_bit_exact_2_3_6_bits(bits, G):
    N, K = 250, 1024
    g = inputs.generator(N + bits + G + 1)
    w = inputs.weights_bf16_valued(N, K, g)
    w[0, :G] = -0.375                    # constant group: scale 0
    wq_ref, s_ref, b_ref = oracle.affine_quantize(w.numpy(), G, bits)
    wq, s, b = bq.affine_quantize(w.cuda(), G, bits)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), wq_ref)
    assert np.array_equal(u16(s), s_ref)
    assert np.array_equal(u16(b), b_ref)
