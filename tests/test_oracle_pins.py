"""Pins for the CPU oracle: checks against facts fixed by the format definitions,
by IEEE-754 and by exact arithmetic -- never against the oracle itself.

The pages print no worked example, so each pin is a closed form (values that
are exact by construction), an invariant of the quantizers, a reduction to a
library routine (numpy / torch float conversions), or exact rational brute
force (fractions.Fraction).  The last test plants mistakes in the oracle's
outputs and checks that the pins notice them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_gemm_quant_b200 import inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --------------------------------------------------------------------------
# helpers written from the layout statements (independent of the oracle)
# --------------------------------------------------------------------------
def pack_q4_0(q: np.ndarray) -> np.ndarray:
    """q[N][K] codes in [0,15] -> bytes: byte j of a 32-block holds element j
    (low nibble) and element j+16 (high nibble)."""
    N, K = q.shape
    qb = q.reshape(N, K // 32, 32).astype(np.uint8)
    return (qb[:, :, :16] | (qb[:, :, 16:] << 4)).reshape(N, K // 2)


def pack_affine(q: np.ndarray, bits: int) -> np.ndarray:
    """q[N][K] -> u32 words of a little-endian bit stream per row: the bits of
    code k, lowest first, are stream bits bits*k ..; stream bit i is bit i%32 of
    word i//32 (numpy bit arrays, independent of the oracle's loops)."""
    N, K = q.shape
    code_bits = (q.astype(np.uint64)[..., None] >> np.arange(bits, dtype=np.uint64)) & 1   # [N][K][bits]
    stream = code_bits.reshape(N, K * bits).astype(np.uint8)
    return np.ascontiguousarray(np.packbits(stream, axis=1, bitorder="little")).view("<u4")


def unpack_affine(wq: np.ndarray, bits: int, K: int) -> np.ndarray:
    N = wq.shape[0]
    stream = np.unpackbits(np.ascontiguousarray(wq).astype("<u4").view(np.uint8), axis=1, bitorder="little")
    code_bits = stream[:, :K * bits].reshape(N, K, bits).astype(np.int64)
    return (code_bits << np.arange(bits)).sum(axis=2)


AFFINE_BITS = [2, 3, 4, 6, 8]


def f32_from_bf16_bits(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32)


def torch_bf16_bits(v32: np.ndarray) -> np.ndarray:
    """Library rounding fp32 -> bf16 (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(v32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def np_f16_bits(v32: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(v32, np.float32).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------------------
# conversions: reduce to numpy / torch
# --------------------------------------------------------------------------
def test_f16_to_f32_exhaustive_vs_numpy():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _interesting_f32_bits(n, seed):
    rng = np.random.default_rng(seed)
    u = rng.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
    # concentrate on the fp16 range and on exact ties
    e = rng.integers(90, 145, n // 2).astype(np.uint32)
    m = rng.integers(0, 1 << 23, n // 2).astype(np.uint32)
    s = rng.integers(0, 2, n // 2).astype(np.uint32)
    near = (s << 31) | (e << 23) | m
    tie16 = (near & ~np.uint32(0x1FFF)) | np.uint32(0x1000)      # fp16-normal ties
    tie_bf = (near & ~np.uint32(0xFFFF)) | np.uint32(0x8000)     # bf16 ties
    specials = np.array([0x00000000, 0x80000000, 0x7F800000, 0xFF800000, 0x477FE000, 0x477FF000,
                         0x477FEFFF, 0x477FF001, 0x33800000, 0x33000000, 0x33000001, 0x33C00000,
                         0x38800000, 0x387FFFFF, 0x00000001, 0x807FFFFF, 0x3F800000, 0x7F7FFFFF,
                         0x7F7F8000, 0x7F7F7FFF], dtype=np.uint32)
    return np.concatenate([u, near, tie16, tie_bf, specials])


def test_f32_to_f16_vs_numpy():
    bits = _interesting_f32_bits(400_000, 1)
    v = bits.view(np.float32)
    finite = np.isfinite(v) | np.isinf(v)
    v = v[finite]
    got = oracle.f32_to_f16(v)
    ref = np_f16_bits(v)
    assert np.array_equal(got, ref)


def test_f32_to_bf16_vs_torch():
    bits = _interesting_f32_bits(400_000, 2)
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]
    assert np.array_equal(oracle.f32_to_bf16(v), torch_bf16_bits(v))


def test_bf16_to_f32_exhaustive_vs_torch():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f32(h)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


# --------------------------------------------------------------------------
# Q4_0
# --------------------------------------------------------------------------
def test_q4_0_dequant_closed_form_layout():
    """Scales with few significant bits make every d*(q-8) exact in bf16, so the
    expected values need no rounding; the bytes are packed from the layout
    statement by hand, which pins nibble order, the -8 offset and the scale."""
    rng = np.random.default_rng(3)
    N, K = 5, 96
    q = rng.integers(0, 16, (N, K))
    d_vals = rng.choice([0.5, -1.5, 0.125, 3.0, -0.25, 1.0], size=(N, K // 32))
    wq = pack_q4_0(q)
    d16 = np_f16_bits(d_vals.astype(np.float32))
    got = f32_from_bf16_bits(oracle.q4_0_dequantize(wq, d16))
    expect = np.repeat(d_vals, 32, axis=1) * (q - 8)
    assert np.array_equal(got.astype(np.float64), expect)


def test_q4_0_dequant_specific_block():
    # byte j = j | (15 - j) << 4: elements 0..15 are q = 0..15, elements 16..31 are q = 15..0
    wq = np.array([[j | ((15 - j) << 4) for j in range(16)]], np.uint8)
    d16 = np.array([[0x3800]], np.uint16)                   # 0.5
    got = f32_from_bf16_bits(oracle.q4_0_dequantize(wq, d16))[0]
    assert list(got[:16]) == [0.5 * (j - 8) for j in range(16)]
    assert list(got[16:]) == [0.5 * (7 - j) for j in range(16)]


def test_q4_0_dequant_rounding_reduces_to_library():
    """Arbitrary finite fp16 scales (subnormals, signs) and codes: the fp32 product
    d*(q-8) is exact (11-bit x 4-bit), so the result is the library's bf16
    rounding of it, sign of zero included."""
    g = inputs.generator(4)
    N, K = 64, 256
    wq = inputs.random_bytes((N, K // 2), g).numpy()
    d16 = inputs.random_f16_bits((N, K // 32), g).numpy().view(np.uint16)
    got = oracle.q4_0_dequantize(wq, d16)
    d = np.repeat(d16.view(np.float16).astype(np.float32), 32, axis=1)
    qb = wq.reshape(N, K // 32, 16)
    q = np.concatenate([qb & 15, qb >> 4], axis=2).reshape(N, K).astype(np.float32)
    exact = d * (q - np.float32(8))          # exact in fp32
    assert np.array_equal(got, torch_bf16_bits(exact))


def _exact_q4_0_blocks(rng, N, K):
    """Blocks w = d*(q-8) with fp16 d whose products are exact in bf16, and at
    least one q = 0 in every block (so the max-abs element is -8d)."""
    q = rng.integers(1, 16, (N, K))
    q.reshape(N, K // 32, 32)[:, :, 0] = 0
    perm = rng.permuted(np.tile(np.arange(32), (N * K // 32, 1)), axis=1)
    q = np.take_along_axis(q.reshape(-1, 32), perm, axis=1).reshape(N, K)
    mant = rng.integers(0, 16, (N, K // 32))                 # 5-bit significands
    expo = rng.integers(-12, 4, (N, K // 32))
    sign = rng.choice([-1.0, 1.0], (N, K // 32))
    d = sign * (1 + mant / 16.0) * np.exp2(expo)
    w = np.repeat(d, 32, axis=1) * (q - 8)
    return q, d, w.astype(np.float32)


def test_q4_0_round_trip_exact():
    rng = np.random.default_rng(5)
    N, K = 16, 256
    q, d, w = _exact_q4_0_blocks(rng, N, K)
    wq, d16 = oracle.q4_0_quantize(w)
    assert np.array_equal(d16, np_f16_bits(d.astype(np.float32)))
    assert np.array_equal(wq, pack_q4_0(q))
    back = f32_from_bf16_bits(oracle.q4_0_dequantize(wq, d16))
    assert np.array_equal(back, w)


def test_q4_0_all_zero_block():
    w = np.zeros((2, 64), np.float32)
    wq, d16 = oracle.q4_0_quantize(w)
    assert np.all(wq == 0x88)
    assert np.all((d16 & 0x7FFF) == 0)
    out = oracle.q4_0_dequantize(wq, d16)
    assert np.all((out & 0x7FFF) == 0)


def test_q4_0_invariants_random():
    g = inputs.generator(6)
    w = inputs.weights_fp32(64, 1024, g).numpy()
    wq, d16 = oracle.q4_0_quantize(w)
    N, K = w.shape
    blk = w.reshape(N, K // 32, 32)
    qb = wq.reshape(N, K // 32, 16)
    q = np.concatenate([qb & 15, qb >> 4], axis=2)            # element order 0..31
    # the max-abs element (first on ties) maps to q = 0 and d = max / -8
    idx = np.abs(blk).argmax(axis=2)
    assert np.all(np.take_along_axis(q, idx[..., None], axis=2) == 0)
    mx = np.take_along_axis(blk, idx[..., None], axis=2)[..., 0]
    assert np.array_equal(d16, np_f16_bits(mx / np.float32(-8)))
    # error bound: nearest code (half |d|) plus fp16 scale and bf16 output rounding;
    # only an element equal to -max may clamp (error up to |d|)
    d = d16.view(np.float16).astype(np.float64)[..., None]
    deq = f32_from_bf16_bits(oracle.q4_0_dequantize(wq, d16)).reshape(N, K // 32, 32).astype(np.float64)
    err = np.abs(blk - deq)
    clamped = (q == 15) & (blk / (mx[..., None] / -8.0) > 7.5)
    bound = np.where(clamped, 1.0, 0.5) * np.abs(d) + 8 * np.abs(d) * 2.0 ** -11 + np.abs(deq) * 2.0 ** -8
    assert np.all(err <= bound * (1 + 1e-6))


# --------------------------------------------------------------------------
# affine
# --------------------------------------------------------------------------
def test_affine_packing_hand_derived():
    """Layout fixed by hand: eight 3-bit codes 0..7 are the octal number
    76543210 = 0xFAC688, bytes 88 C6 FA repeating; four 6-bit codes 1, 2, 3, 4 are
    1 + 2*64 + 3*4096 + 4*262144 = 0x103081, bytes 81 30 10 repeating; 4- and
    8-bit codes fill each word lowest bits first."""
    q3 = (np.arange(32) % 8)[None, :]
    assert pack_affine(q3, 3).tolist() == [[0x88FAC688, 0xC688FAC6, 0xFAC688FA]]
    q6 = np.tile([1, 2, 3, 4], 8)[None, :]
    assert pack_affine(q6, 6).tolist() == [[0x81103081, 0x30811030, 0x10308110] * 2]
    q4 = (np.arange(32) % 16)[None, :]
    assert pack_affine(q4, 4).tolist() == [[0x76543210, 0xFEDCBA98, 0x76543210, 0xFEDCBA98]]
    q2 = (np.arange(32) % 4)[None, :]
    assert pack_affine(q2, 2).tolist() == [[0xE4E4E4E4, 0xE4E4E4E4]]
    # the oracle reads codes from the same layout: unit scale, zero bias gives q itself
    for q, bits in ((q3, 3), (q6, 6), (q4, 4), (q2, 2)):
        one = torch_bf16_bits(np.ones((1, 1), np.float32))
        zero = np.zeros((1, 1), np.uint16)
        got = f32_from_bf16_bits(oracle.affine_dequantize(pack_affine(q, bits), one, zero, 32, bits))
        assert np.array_equal(got, q.astype(np.float32))


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_dequant_closed_form_layout(bits, G):
    rng = np.random.default_rng(7 + bits + G)
    N, K = 3, 256
    L = (1 << bits) - 1
    q = rng.integers(0, L + 1, (N, K))
    s = rng.choice([0.25, 0.5, 0.0625], size=(N, K // G))      # b/s integer, q + b/s in [-48, 255]
    b = rng.choice([-1.0, 0.0, -3.0, -0.5], size=(N, K // G))
    wq = pack_affine(q, bits)
    got = f32_from_bf16_bits(oracle.affine_dequantize(wq, torch_bf16_bits(s.astype(np.float32)),
                                                      torch_bf16_bits(b.astype(np.float32)), G, bits))
    expect = np.repeat(s, G, axis=1) * q + np.repeat(b, G, axis=1)
    assert np.array_equal(got.astype(np.float64), expect)


@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_dequant_rounding_reduces_to_library(bits):
    """Random bf16 scale/bias with exponents close enough that scale*q + bias is
    exact in fp32; the result is then the library's bf16 rounding of it."""
    g = inputs.generator(8 + bits)
    N, K, G = 32, 512, 64
    L = (1 << bits) - 1
    s16 = inputs.random_bf16_bits((N, K // G), g, 112, 116).numpy().view(np.uint16) & 0x7FFF
    b16 = inputs.random_bf16_bits((N, K // G), g, 112, 120).numpy().view(np.uint16)
    q = torch.randint(0, L + 1, (N, K), generator=g).numpy()
    got = oracle.affine_dequantize(pack_affine(q, bits), s16, b16, G, bits)
    s = np.repeat(f32_from_bf16_bits(s16), G, axis=1).astype(np.float64)
    b = np.repeat(f32_from_bf16_bits(b16), G, axis=1).astype(np.float64)
    exact = s * q + b
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)   # exact in fp32
    assert np.array_equal(got, torch_bf16_bits(exact.astype(np.float32)))


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_round_trip_exact(bits, G):
    rng = np.random.default_rng(9 + bits + G)
    N, K = 8, 256
    L = (1 << bits) - 1
    q = rng.integers(0, L + 1, (N, K))
    qg = q.reshape(N, K // G, G)
    qg[:, :, 0] = 0
    qg[:, :, 1] = L
    e = rng.integers(-9, -3, (N, K // G)).astype(np.float64)
    s = np.exp2(e)
    b = -16.0 * s * rng.integers(0, 4, (N, K // G))
    w = (np.repeat(s, G, axis=1) * q + np.repeat(b, G, axis=1)).astype(np.float32)
    assert np.array_equal(torch_bf16_bits(w), np.ascontiguousarray(w).view(np.uint32) >> 16)  # bf16-valued
    wq, s16, b16 = oracle.affine_quantize(w, G, bits)
    assert np.array_equal(f32_from_bf16_bits(s16).astype(np.float64), s)
    assert np.array_equal(f32_from_bf16_bits(b16).astype(np.float64), b)
    assert np.array_equal(wq, pack_affine(q, bits))
    back = f32_from_bf16_bits(oracle.affine_dequantize(wq, s16, b16, G, bits))
    assert np.array_equal(back, w)


@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_constant_group(bits):
    w = np.full((2, 128), -0.375, np.float32)
    w[1, 64:] = 0.0
    wq, s16, b16 = oracle.affine_quantize(w, 64, bits)
    assert np.all(s16 == 0) and np.all(wq == 0)
    assert np.array_equal(f32_from_bf16_bits(b16), np.array([[-0.375, -0.375], [-0.375, 0.0]], np.float32))
    back = f32_from_bf16_bits(oracle.affine_dequantize(wq, s16, b16, 64, bits))
    assert np.array_equal(back, w)


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_invariants_random(bits, G):
    g = inputs.generator(10 + bits + G)
    N, K = 48, 1024
    L = (1 << bits) - 1
    w = inputs.weights_bf16_valued(N, K, g).numpy()
    wq, s16, b16 = oracle.affine_quantize(w, G, bits)
    assert wq.shape == (N, K * bits // 32)
    q = unpack_affine(wq, bits, K)
    wg = w.reshape(N, K // G, G)
    qg = q.reshape(N, K // G, G)
    # min maps to 0, max to L; scale = (max-min)/L and bias = min
    assert np.all(np.take_along_axis(qg, wg.argmin(axis=2)[..., None], axis=2) == 0)
    assert np.array_equal(b16, torch_bf16_bits(wg.min(axis=2)))
    s_exact = (wg.max(axis=2) - wg.min(axis=2)) / np.float32(L)
    assert np.array_equal(s16, torch_bf16_bits(s_exact))
    # the max maps to L, except that a bf16 scale rounded above (max-min)/L may
    # bring it down by one code (possible only when L is large next to 2^8)
    q_max = np.take_along_axis(qg, wg.argmax(axis=2)[..., None], axis=2)[..., 0]
    s_stored = f32_from_bf16_bits(s16)
    assert np.all(q_max[s_stored <= s_exact] == L)
    assert np.all(q_max >= L - 1)
    if bits <= 6:                       # L * 2^-8 < 1/2: the rounded scale cannot move the max's code
        assert np.all(q_max == L)
    s = f32_from_bf16_bits(s16).astype(np.float64)[..., None]
    deq = f32_from_bf16_bits(oracle.affine_dequantize(wq, s16, b16, G, bits)).reshape(N, K // G, G)
    err = np.abs(wg.astype(np.float64) - deq)
    bound = s * (0.5 + L * 2.0 ** -8) + np.abs(deq) * 2.0 ** -8
    assert np.all(err <= bound * (1 + 1e-6))


# --------------------------------------------------------------------------
# matmul: exact rational brute force
# --------------------------------------------------------------------------
def _bf16_frac(h):
    return Fraction(float(f32_from_bf16_bits(np.array([h], np.uint16))[0]))


def test_matmul_ref_fraction_bruteforce():
    g = inputs.generator(11)
    M, N, K = 3, 5, 40
    x = inputs.activations_bf16(M, K, g).view(torch.int16).numpy().view(np.uint16)
    w = inputs.activations_bf16(N, K, g).view(torch.int16).numpy().view(np.uint16)
    y, a, _ = oracle.matmul_ref(x, w, nthreads=2)
    for m in range(M):
        for n in range(N):
            prods = [_bf16_frac(x[m, k]) * _bf16_frac(w[n, k]) for k in range(K)]
            exact = sum(prods, Fraction(0))
            exact_abs = sum((abs(p) for p in prods), Fraction(0))
            assert abs(Fraction(y[m, n]) - exact) <= exact_abs * K * Fraction(1, 2 ** 52)
            assert abs(Fraction(a[m, n]) - exact_abs) <= exact_abs * K * Fraction(1, 2 ** 52)


def test_matmul_ref_one_hot_and_rows():
    g = inputs.generator(12)
    N, K = 7, 64
    w = inputs.activations_bf16(N, K, g).view(torch.int16).numpy().view(np.uint16)
    x = np.zeros((K, K), np.uint16)
    x[np.arange(K), np.arange(K)] = 0x3F80                        # bf16 1.0
    y, a, _ = oracle.matmul_ref(x, w)
    assert np.array_equal(y, f32_from_bf16_bits(w).T.astype(np.float64))
    assert np.array_equal(a, np.abs(y))
    rows = np.array([5, 0, 63])
    y2, _, _ = oracle.matmul_ref(x, w, rows=rows, nthreads=3)
    assert np.array_equal(y2, y[rows])


def test_quantized_chain_fraction_bruteforce():
    """x . dequant(W)^T for a Q4_0 and an affine-8 weight, exact rationals."""
    rng = np.random.default_rng(13)
    M, N, K = 2, 3, 64
    q = rng.integers(0, 16, (N, K))
    d = np.array([[0.5, -0.25], [1.0, 0.125], [-2.0, 0.75]])
    wq = pack_q4_0(q)
    x = torch.randn(M, K, generator=inputs.generator(13)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = oracle.q4_0_dequantize(wq, np_f16_bits(d.astype(np.float32)))
    y, _, _ = oracle.matmul_ref(xb, wb)
    for m in range(M):
        for n in range(N):
            exact = sum((Fraction(float(x[m, k])) * Fraction(d[n, k // 32]) * (int(q[n, k]) - 8)
                         for k in range(K)), Fraction(0))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(1, 2 ** 40)
    q8 = rng.integers(0, 256, (N, K))
    s = np.array([[0.0078125], [0.25], [2.0 ** -10]])
    b = np.array([[-1.0], [0.5], [-0.125]])
    w8 = oracle.affine_dequantize(pack_affine(q8, 8), torch_bf16_bits(s.astype(np.float32)),
                                  torch_bf16_bits(b.astype(np.float32)), 64, 8)
    y8, _, _ = oracle.matmul_ref(xb, w8)
    for m in range(M):
        for n in range(N):
            exact = sum((Fraction(float(x[m, k])) * (Fraction(s[n, 0]) * int(q8[n, k]) + Fraction(b[n, 0]))
                         for k in range(K)), Fraction(0))
            assert abs(Fraction(y8[m, n]) - exact) <= Fraction(1, 2 ** 36)


# --------------------------------------------------------------------------
# planted mistakes: the pins above must notice each of these
# --------------------------------------------------------------------------
def test_pins_catch_planted_mistakes():
    rng = np.random.default_rng(14)
    N, K = 4, 64
    q = rng.integers(0, 16, (N, K))
    d = np.full((N, K // 32), 0.5)
    wq = pack_q4_0(q)
    d16 = np_f16_bits(d.astype(np.float32))
    expect = np.repeat(d, 32, axis=1) * (q - 8)

    def ok(deq_fn):
        return np.array_equal(f32_from_bf16_bits(deq_fn(wq, d16)).astype(np.float64), expect)

    assert ok(oracle.q4_0_dequantize)
    swapped = lambda a, s: oracle.q4_0_dequantize(((a & 15) << 4) | (a >> 4), s)            # nibble order
    plus8 = lambda a, s: oracle.f32_to_bf16(-f32_from_bf16_bits(oracle.q4_0_dequantize(a, s)))  # sign of offset
    interleaved = lambda a, s: oracle.q4_0_dequantize(a, s).reshape(N, -1, 2, 16).transpose(0, 1, 3, 2).reshape(N, K)
    for bad in (swapped, plus8, interleaved):
        assert not ok(bad)
    # matmul transposed operand / dropped term
    g = inputs.generator(15)
    x = inputs.activations_bf16(3, 32, g).view(torch.int16).numpy().view(np.uint16)
    w = inputs.activations_bf16(3, 32, g).view(torch.int16).numpy().view(np.uint16)
    y, _, _ = oracle.matmul_ref(x, w)
    yt, _, _ = oracle.matmul_ref(w, x)
    assert not np.allclose(y, yt)
    ydrop, _, _ = oracle.matmul_ref(x[:, :31], w[:, :31])
    assert not np.allclose(y, ydrop)


def test_q4_0_import_aos_matches_hand_assembled_blocks():
    """Array-of-structs blocks (fp16 d little-endian, then 16 code bytes) built
    with numpy from random codes and scales split back into exactly those arrays."""
    rng = np.random.default_rng(11)
    N, K = 7, 96
    wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    d = rng.integers(0, 65536, (N, K // 32), dtype=np.uint16)
    blocks = np.empty((N, K // 32, 18), np.uint8)
    blocks[:, :, 0] = d & 0xFF
    blocks[:, :, 1] = d >> 8
    blocks[:, :, 2:] = wq.reshape(N, K // 32, 16)
    got_wq, got_d = oracle.q4_0_import_aos(blocks.reshape(N, -1))
    assert np.array_equal(got_wq, wq)
    assert np.array_equal(got_d, d)
    # a planted byte swap of the scale is caught
    swapped = blocks.copy()
    swapped[:, :, [0, 1]] = swapped[:, :, [1, 0]]
    _, bad_d = oracle.q4_0_import_aos(swapped.reshape(N, -1))
    assert not np.array_equal(bad_d, d)


# --------------------------------------------------------------------------
# Q8_1-style activations for the quantized-activation decode path
# --------------------------------------------------------------------------
def _bf16_bits_of(v: np.ndarray) -> np.ndarray:
    return torch_bf16_bits(np.asarray(v, np.float32))


def test_q8_1_quantize_closed_forms():
    """Blocks of integer multiples of 2^e with one |value| = 127 * 2^e: d = 2^e exactly
    and every code is the integer itself; ties at .5 round away from zero; an all-zero
    block has d = 0 and zero codes."""
    rng = np.random.default_rng(21)
    e = np.array([-3, 0, -7], np.float64)
    ints = rng.integers(-127, 128, (3, 32))
    ints[:, 5] = 127
    ints[1, 9] = -127
    x = ints * np.exp2(e)[:, None]
    half = np.zeros((1, 32))
    half[0, 0] = 127.0
    half[0, 1:5] = [2.5, -2.5, 0.5, -0.5]          # exactly halfway after scaling by 1/d = 1
    zero = np.zeros((1, 32))
    xb = _bf16_bits_of(np.concatenate([x, half, zero]).reshape(1, -1))
    xq, dx, qs = oracle.q8_1_quantize(xb)
    q = xq.reshape(5, 32)
    assert np.array_equal(dx[0], np.array([2 ** -3, 1.0, 2 ** -7, 1.0, 0.0], np.float32))
    assert np.array_equal(q[:3], ints)
    assert list(q[3, 1:5]) == [3, -3, 1, -1]
    assert np.all(q[4] == 0)
    assert np.array_equal(qs[0], q.sum(axis=1))


def test_q8_1_quantize_invariants_random():
    g = inputs.generator(22)
    M, K = 5, 1024
    x = inputs.activations_bf16(M, K, g)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    xf = x.float().numpy().astype(np.float64)
    xq, dx, qs = oracle.q8_1_quantize(xb)
    assert np.abs(xq.astype(np.int32)).max() <= 127
    amax = np.abs(xf.reshape(M, K // 32, 32)).max(axis=2)
    assert np.array_equal(dx, (amax.astype(np.float32) / np.float32(127)))
    assert np.array_equal(qs, xq.reshape(M, K // 32, 32).astype(np.int32).sum(axis=2))
    err = np.abs(xf - xq.astype(np.float64) * np.repeat(dx.astype(np.float64), 32, axis=1))
    # half a step, plus the fp32 rounding of 1/d and of x * (1/d) near ties
    # (at most |x| * 2^-22 <= 127 d * 2^-22)
    assert np.all(err <= np.repeat(dx.astype(np.float64), 32, axis=1) * (0.5 + 127 * 2.0 ** -22))


def test_q4_0_q8_matmul_unit_scales_is_integer_dot_product():
    """Activations that are integers with block maximum 127 (dx = 1) and weight
    scales 1.0: the result is numpy's exact int64 dot product of x and (q - 8)."""
    rng = np.random.default_rng(23)
    M, N, K = 3, 5, 128
    xi = rng.integers(-127, 128, (M, K))
    xi[:, ::32] = 127
    wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    d = np.full((N, K // 32), 0x3C00, np.uint16)                 # fp16 1.0
    xq, dx, _ = oracle.q8_1_quantize(_bf16_bits_of(xi))
    assert np.all(dx == 1.0) and np.array_equal(xq, xi)
    blk = wq.reshape(N, K // 32, 16)
    q = np.concatenate([blk & 0x0F, blk >> 4], axis=2).reshape(N, K).astype(np.int64)   # element j, then j + 16
    expect = xi.astype(np.int64) @ (q - 8).T
    y, a = oracle.q4_0_q8_matmul(xq, dx, wq, d)
    assert np.array_equal(y, expect.astype(np.float64))


def test_q4_0_q8_matmul_within_activation_quantization_bound():
    """Against the plain bf16 matmul of the same weights: the difference is bounded by
    the activation quantization error (<= dx / 2 per element) times |w|, plus the bf16
    rounding of the weights (<= 2^-9 |w|) that the q8 path does not apply."""
    g = inputs.generator(24)
    M, N, K = 4, 40, 512
    w = inputs.weights_fp32(N, K, g).numpy()
    wq, d = oracle.q4_0_quantize(w)
    x = inputs.activations_bf16(M, K, g)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    xq, dx, _ = oracle.q8_1_quantize(xb)
    y, _ = oracle.q4_0_q8_matmul(xq, dx, wq, d)
    wb = oracle.q4_0_dequantize(wq, d)
    y_ref, a_ref, _ = oracle.matmul_ref(xb, wb)
    wabs = np.abs(f32_from_bf16_bits(wb).astype(np.float64))
    bound = (np.repeat(dx.astype(np.float64), 32, axis=1) / 2) @ wabs.T + 2.0 ** -9 * a_ref * 1.01 + 1e-12
    assert np.all(np.abs(y - y_ref) <= bound)
    # and the bound is not vacuous: a planted sign error on the weights breaks it
    y_bad, _ = oracle.q4_0_q8_matmul(xq, dx, wq ^ 0x88, d)
    assert not np.all(np.abs(y_bad - y_ref) <= bound)


# --------------------------------------------------------------------------
# quantizer rounding decisions: exact ties, and planted variants of the oracle
# --------------------------------------------------------------------------
import ctypes
import os
import subprocess

import _ties
from oracle import build as _oracle_build


def _q4_0_quantize_with(lib, w):
    w = np.ascontiguousarray(w, np.float32)
    N, K = w.shape
    wq = np.empty((N, K // 2), np.uint8)
    d = np.empty((N, K // 32), np.uint16)
    lib.oracle_q4_0_quantize(ctypes.c_void_p(w.ctypes.data), ctypes.c_int64(N), ctypes.c_int64(K),
                             ctypes.c_void_p(wq.ctypes.data), ctypes.c_void_p(d.ctypes.data))
    return wq, d


def _affine_quantize_with(lib, w, group, bits):
    w = np.ascontiguousarray(w, np.float32)
    N, K = w.shape
    wq = np.empty((N, K * bits // 32), np.uint32)
    s = np.empty((N, K // group), np.uint16)
    b = np.empty((N, K // group), np.uint16)
    lib.oracle_affine_quantize(ctypes.c_void_p(w.ctypes.data), ctypes.c_int64(N), ctypes.c_int64(K),
                               ctypes.c_int(group), ctypes.c_int(bits), ctypes.c_void_p(wq.ctypes.data),
                               ctypes.c_void_p(s.ctypes.data), ctypes.c_void_p(b.ctypes.data))
    return wq, s, b


class _Oracle:
    """The oracle's own library, or a copy of its source with one planted change."""

    def __init__(self, lib):
        self.lib = lib

    def q4_0(self, w):
        return _q4_0_quantize_with(self.lib, w)

    def affine(self, w, group, bits):
        return _affine_quantize_with(self.lib, w, group, bits)


def _planted(tmp_path, name, old, new):
    src = open(_oracle_build.SRC).read()
    assert src.count(old) >= 1, f"planted change {name!r} no longer applies"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", *_oracle_build.CFLAGS, str(path), "-o", str(lib), "-lm"])
    return _Oracle(ctypes.CDLL(str(lib)))


def _q4_0_ties_hold(orc: _Oracle) -> bool:
    w, q = _ties.q4_0_tie_matrix()
    wq, d16 = orc.q4_0(w)
    d = np.array([np.float32(d) for d, _ in _ties.Q4_0_TIE_BLOCKS], np.float32)
    return np.array_equal(wq, pack_q4_0(q)) and np.array_equal(d16[:, 0], np_f16_bits(d))


def _affine_ties_hold(orc: _Oracle, bits: int) -> bool:
    w, s, q = _ties.affine_tie_matrix(bits)
    wq, s16, b16 = orc.affine(w, 64, bits)
    return (np.array_equal(f32_from_bf16_bits(s16).astype(np.float64), np.repeat(s[:, None], 2, axis=1))
            and np.all(b16 == 0) and np.array_equal(wq, pack_affine(q, bits)))


def test_q4_0_quantize_exact_division_ties():
    """Elements with w/d = k - 1/2 exactly get code k (q = int(w/d + 8.5) with the
    fp32 d); both the reciprocal form w·(1/d) and a division by the stored fp16
    scale give k - 1 on these blocks."""
    assert _ties.q4_0_tie_exactness()
    assert _q4_0_ties_hold(_Oracle(oracle._load()))
    # the blocks discriminate the alternative readings (numpy fp32 arithmetic)
    w, q = _ties.q4_0_tie_matrix()
    for r, (d, ties) in enumerate(_ties.Q4_0_TIE_BLOCKS):
        d32 = np.float32(d)
        for i, k in ties:
            assert int(np.float32(w[r, i] * (np.float32(1) / d32)) + np.float32(8.5)) == k - 1
            assert int(np.float32(w[r, i] / np.float32(np.float16(d32))) + np.float32(8.5)) == k - 1


def test_q4_0_quantize_max_abs_tie_takes_first_element():
    """+a before -a with |a| the block maximum: d = a / -8 (negative), the +a
    element gets code 0 and the -a element clamps to 15."""
    w = np.full((1, 32), 0.125, np.float32)
    w[0, 2], w[0, 7] = 0.75, -0.75
    wq, d16 = oracle.q4_0_quantize(w)
    assert d16[0, 0] == np_f16_bits(np.array([-0.09375], np.float32))[0]
    lo, hi = wq[0] & 15, wq[0] >> 4
    assert lo[2] == 0 and lo[7] == 15
    assert np.all(np.delete(lo, [2, 7]) == 7) and np.all(hi == 7)     # 0.125 / -0.09375 + 8.5 = 7.17


@pytest.mark.parametrize("bits", AFFINE_BITS)
def test_affine_quantize_ties_to_even(bits):
    """(w - bias)/scale = j + 1/2 exactly: the code is the even neighbour."""
    assert _affine_ties_hold(_Oracle(oracle._load()), bits)


def test_quantizer_pins_catch_planted_oracle_variants(tmp_path):
    """Copies of the oracle source with one rounding rule changed fail the pins above."""
    variants = [
        ("roundf", "float r = nearbyintf(t);", "float r = roundf(t);", "affine"),
        ("trunc_half", "float r = nearbyintf(t);", "float r = floorf(t + 0.5f);", "affine"),
        ("reciprocal", "float t0 = (d != 0.0f) ? blk[j] / d : 0.0f;",
         "float t0 = (d != 0.0f) ? blk[j] * (1.0f / d) : 0.0f;", "q4_0"),
        ("fp16_scale", "float t0 = (d != 0.0f) ? blk[j] / d : 0.0f;",
         "float t0 = (d != 0.0f) ? blk[j] / oracle_f16_to_f32(oracle_f32_to_f16(d)) : 0.0f;", "q4_0"),
        ("last_max", "if (fabsf(v) > amax)", "if (fabsf(v) >= amax)", "q4_0_max"),
    ]
    for name, old, new, kind in variants:
        orc = _planted(tmp_path, name, old, new)
        if kind == "affine":
            assert not all(_affine_ties_hold(orc, b) for b in AFFINE_BITS), name
        elif kind == "q4_0":
            assert not _q4_0_ties_hold(orc), name
        else:
            w = np.full((1, 32), 0.125, np.float32)
            w[0, 2], w[0, 7] = 0.75, -0.75
            _, d16 = orc.q4_0(w)
            assert d16[0, 0] != np_f16_bits(np.array([-0.09375], np.float32))[0], name
