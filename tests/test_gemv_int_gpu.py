"""The streamed decode GEMV (one or two tokens, forced with path gemv_stream),
where x enters integer MMAs as signed byte slices per scale group: eight for one
token (exact within 2^54 of the group's largest activation), four for each of
two (2^22).  Activations here stress that split: magnitudes spread over many
binades inside each group, zero, tiny (subnormal) and huge groups, NaN, and
spreads wider than the slices (the launch then takes fp32 dot products).
Checked against the oracle's float64 product with the workload tolerance and,
where the slices hold x exactly, with a bound of fp32 rounding only."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
from _helpers import FMT, Problem, assert_within_tolerance, reference, u16

pytestmark = pytest.mark.gpu

FMTS = ["q4_0", "affine4", "affine8", "affine4_g32", "affine4_g128", "affine8_g32", "affine8_g128"]


def gemv(p: Problem, x: torch.Tensor) -> torch.Tensor:
    wq, s, b = p.device()
    y = bq.quant_matmul_ex(x.cuda(), wq, s, b, p.group_size, p.bits, True, "gemv_stream")
    torch.cuda.synchronize()
    return y


def signed_binades(M: int, K: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Random signs and mantissas, exponents uniform in [lo, hi]."""
    rng = np.random.default_rng(seed)
    e = rng.integers(lo, hi + 1, size=(M, K))
    m = rng.uniform(1.0, 2.0, size=(M, K))
    s = rng.choice([-1.0, 1.0], size=(M, K))
    return (s * m * np.exp2(e)).astype(np.float32)


def bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(a)) - 7)


def fp32_bound(p: Problem, xb: torch.Tensor, y_ref: np.ndarray, a_ref: np.ndarray) -> np.ndarray:
    """2^-16 of the magnitudes the fp32 arithmetic rounds, plus one bf16 ulp of y:
    sum |x w| for Q4_0; for affine also the two terms s sum q x and z sum x that
    cancel where a weight s q + z is small, bounded by (qmax |s| + |z|) sum_g |x|."""
    mag = a_ref
    if p.biases is not None:
        gs, qmax = p.group_size, (1 << p.bits) - 1
        f = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        xa = np.abs(xb.float().numpy().astype(np.float64))
        xg = xa.reshape(xa.shape[0], -1, gs).sum(axis=2)                   # [M][groups]
        mag = a_ref + xg @ (qmax * np.abs(f(p.scales)) + np.abs(f(p.biases))).T
    return 2.0 ** -16 * mag + ulp_bf16(y_ref)


def exact_weights(fmt: str, N: int, K: int, seed: int) -> np.ndarray:
    """Weights that every quantizer reproduces exactly and whose dequantization is
    exact in bf16: per group a power-of-two step s and codes q, w = s (q - half)
    with half = 8 (4-bit) or 128 (8-bit), the first two codes of each group 0 and
    the largest code (so max - min = (2^bits - 1) s, min = -half s, and for Q4_0
    the signed max-abs is -8 s, d = s)."""
    gs, bits = FMT[fmt]
    rng = np.random.default_rng(seed)
    qmax = (1 << bits) - 1
    half = 1 << (bits - 1)
    q = rng.integers(0, qmax + 1, size=(N, K))
    q[:, 0::gs] = 0
    q[:, 1::gs] = qmax
    step = np.exp2(rng.integers(-10, -4, size=(N, K // gs))).repeat(gs, axis=1)
    return (step * (q - half)).astype(np.float32)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
def test_wide_range_groups_fp32_bound(fmt, M):
    """Exponents -20..1 inside every group: the slices hold x exactly, so with
    weights that dequantize exactly the only error is fp32 rounding of the
    per-group products and their sum, then the bf16 output rounding."""
    p = Problem(fmt, 300, 2048, w=exact_weights(fmt, 300, 2048, seed=40 + M))
    w_exact = exact_weights(fmt, 300, 2048, seed=40 + M)
    assert np.array_equal((p.wb.astype(np.uint32) << 16).view(np.float32), w_exact), "inexact dequantization"
    xb = bf16(signed_binades(M, p.K, -20, 1, seed=7 * M))
    y = gemv(p, xb)
    y_ref, a_ref = reference(xb, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, f"{fmt} M={M}")
    got = y.float().cpu().numpy().astype(np.float64)
    tight = fp32_bound(p, xb, y_ref, a_ref)
    assert np.all(np.abs(got - y_ref) <= tight), float(np.max(np.abs(got - y_ref) / tight))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
def test_zero_tiny_and_huge_groups(fmt, M):
    """Whole groups of zeros, of subnormal bf16 (2^-130) and of 2^60, among
    N(0,1) ones; one group holding both 2^40 and 2^-40."""
    p = Problem(fmt, 130, 1024, seed=50 + M)
    gs = p.group_size
    x = p.x(M).float().numpy().copy()
    ng = p.K // gs
    for m in range(M):
        for gi in range(m, ng, 5):
            x[m, gi * gs:(gi + 1) * gs] = 0.0
        for gi in range(m + 1, ng, 7):
            x[m, gi * gs:(gi + 1) * gs] *= 2.0 ** -130
        x[m, (ng - 2) * gs:(ng - 1) * gs] *= 2.0 ** 60
        x[m, 3 * gs] = 2.0 ** 40
        x[m, 3 * gs + 1] = -(2.0 ** -40)
    xb = bf16(x)
    y = gemv(p, xb)
    y_ref, a_ref = reference(xb, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_two_tokens_match_one_token_bitwise(fmt):
    """Token 0 of a two-token call gives the same bits as the one-token call."""
    p = Problem(fmt, 250, 4096, seed=61)
    x = p.x(2)
    y2 = gemv(p, x)
    y1 = gemv(p, x[:1].contiguous())
    assert np.array_equal(u16(y2[:1]), u16(y1))
    y_ref, a_ref = reference(x, p.wb)
    assert_within_tolerance(y2, y_ref, a_ref, f"{fmt} M=2")


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_nan_activation_poisons_only_its_token(fmt):
    """A NaN in one group of token 1: every output of token 1 is NaN, token 0 is
    unaffected (same bits as alone)."""
    p = Problem(fmt, 200, 1024, seed=62)
    x = p.x(2).float().numpy().copy()
    x[1, 517] = np.nan
    xb = bf16(x)
    y = gemv(p, xb)
    assert torch.isnan(y[1].float()).all()
    y1 = gemv(p, xb[:1].contiguous())
    assert np.array_equal(u16(y[:1]), u16(y1))
    assert bq.bq_device_status() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
def test_group_leader_with_zero_weight(fmt, M):
    """Each group's largest activation (+-1.5) meets a zero weight, the others lie
    2^-14 .. 2^-22 below it: y comes from the low slices alone, and the fp32
    bound holds (a lost low slice would cost a quarter of each small term)."""
    N, K = 260, 1024
    w = exact_weights(fmt, N, K, seed=70 + M)
    gs = FMT[fmt][0]
    w[:, 2::gs] = 0.0                          # code `half`: exact, and keeps the group's min and max
    p = Problem(fmt, N, K, w=w)
    assert np.array_equal((p.wb.astype(np.uint32) << 16).view(np.float32), w)
    x = signed_binades(M, K, -22, -14, seed=71 + M)
    x[:, 2::gs] = np.where(np.arange(K // gs) % 2 == 0, 1.5, -1.5)
    xb = bf16(x)
    y = gemv(p, xb)
    y_ref, a_ref = reference(xb, p.wb)
    got = y.float().cpu().numpy().astype(np.float64)
    tight = fp32_bound(p, xb, y_ref, a_ref)
    assert np.all(np.abs(got - y_ref) <= tight), float(np.max(np.abs(got - y_ref) / tight))


@pytest.mark.parametrize("fmt", FMTS)
def test_one_token_spread_2_50_fp32_bound(fmt):
    """One token gets eight slices: exponents -10..40 inside a group are still
    held exactly, so the fp32 bound holds."""
    N, K = 200, 2048
    w = exact_weights(fmt, N, K, seed=80)
    p = Problem(fmt, N, K, w=w)
    x = signed_binades(1, K, -10, 40, seed=81)
    xb = bf16(x)
    y = gemv(p, xb)
    y_ref, a_ref = reference(xb, p.wb)
    got = y.float().cpu().numpy().astype(np.float64)
    tight = fp32_bound(p, xb, y_ref, a_ref)
    assert np.all(np.abs(got - y_ref) <= tight), float(np.max(np.abs(got - y_ref) / tight))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
def test_spread_beyond_slices_takes_exact_path(fmt, M):
    """Some groups hold one 2^60 activation that meets a zero weight among N(0, 1)
    ones: wider than the slices (2^54 for one token, 2^22 for two), so the
    launch computes fp32 dot products, and the small terms still count."""
    N, K = 180, 1024
    w = exact_weights(fmt, N, K, seed=90 + M)
    gs = FMT[fmt][0]
    w[:, 2::gs] = 0.0
    p = Problem(fmt, N, K, w=w)
    x = p.x(M).float().numpy().copy()
    x[:, 2 * gs + 2] = 2.0 ** 60
    x[M - 1, 5 * gs + 2] = -(2.0 ** 60)
    xb = bf16(x)
    y = gemv(p, xb)
    y_ref, a_ref = reference(xb, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, f"{fmt} M={M}")
    # quant_matmul_multi (two matrices sharing x) gives quant_matmul's bits
    wq, s, b = p.device()
    ys = bq.quant_matmul_multi(xb.cuda(), [(wq, s, b), (wq, s, b)], p.group_size, p.bits)
    y_auto = bq.quant_matmul(xb.cuda(), wq, s, b, p.group_size, p.bits)
    torch.cuda.synchronize()
    assert np.array_equal(u16(ys[0]), u16(y_auto)) and np.array_equal(u16(ys[1]), u16(y_auto))
    assert_within_tolerance(y_auto, y_ref, a_ref, f"{fmt} M={M} auto")


@pytest.mark.parametrize("fmt", ["affine8", "affine8_g32", "affine8_g128"])
@pytest.mark.parametrize("M", [1, 2])
def test_dispatcher_takes_streamed_kernel_for_affine8(fmt, M):
    """BQ_PATH_GEMV (and AUTO) run the streamed kernel for affine 8-bit at one or
    two tokens: the same bits as forcing it; quant_matmul_multi too."""
    p = Problem(fmt, 12288, 4096, seed=100 + M)
    wq, s, b = p.device()
    x = p.x(M).cuda()
    y_forced = bq.quant_matmul_ex(x, wq, s, b, p.group_size, p.bits, True, "gemv_stream")
    y_gemv = bq.quant_matmul_ex(x, wq, s, b, p.group_size, p.bits, True, "gemv")
    y_auto = bq.quant_matmul(x, wq, s, b, p.group_size, p.bits)
    ys = bq.quant_matmul_multi(x, [(wq, s, b)], p.group_size, p.bits)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y_gemv), u16(y_forced))
    assert np.array_equal(u16(y_auto), u16(y_forced))
    assert np.array_equal(u16(ys[0]), u16(y_forced))
    rows = list(range(0, 12288, 61)) + [12287]
    y_ref, a_ref = reference(x.cpu(), p.wb[rows])
    assert_within_tolerance(y_forced[:, torch.as_tensor(rows, device=y_forced.device)], y_ref, a_ref, fmt)


def test_forced_streamed_kernel_where_it_does_not_apply():
    """Three tokens, or K not a multiple of 8 groups: BQ_ERR_UNSUPPORTED; a caller
    workspace smaller than the tables: BQ_ERR_WORKSPACE."""
    p = Problem("q4_0", 64, 544, seed=3)
    wq, s, b = p.device()
    with pytest.raises(bq.BqError, match="UNSUPPORTED"):
        bq.quant_matmul_ex(p.x(1).cuda(), wq, s, b, 32, 4, True, "gemv_stream")
    p = Problem("q4_0", 64, 1024, seed=4)
    wq, s, b = p.device()
    with pytest.raises(bq.BqError, match="UNSUPPORTED"):
        bq.quant_matmul_ex(p.x(3).cuda(), wq, s, b, 32, 4, True, "gemv_stream")
    need = bq.quant_matmul_workspace_size(1, 64, 1024, 32, 4, "gemv_stream")
    assert need > 0
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(bq.BqError, match="WORKSPACE"):
        bq.quant_matmul_ex(p.x(1).cuda(), wq, s, b, 32, 4, True, "gemv_stream", workspace=ws)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    x = p.x(1)
    y = bq.quant_matmul_ex(x.cuda(), wq, s, b, 32, 4, True, "gemv_stream", workspace=ws)
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, "caller workspace")
    assert bq.bq_device_status() == 0
