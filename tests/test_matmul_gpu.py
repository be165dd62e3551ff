"""quant_matmul on every kernel path vs the CPU oracle's float64 reference:
|y_gpu - y_ref| <= 2e-3 * sum_k |x_k w_k| + 1e-5 for every checked output,
where w is the oracle's bf16 dequantization (the equivalence
quantized_matmul == x @ dequantize(...).T of the MLX issue page, Repro)."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
import oracle
from bit_quantized_gemm_quant_b200 import inputs
from _helpers import Problem, assert_within_tolerance, reference, u16


def f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)

pytestmark = pytest.mark.gpu

GEMV_M = [1, 2, 8, 9, 16, 19, 32]
TC_M = [1, 16, 33, 100, 256, 300]


def run(p: Problem, x: torch.Tensor, path: str):
    wq, s, b = p.device()
    y = bq.quant_matmul_ex(x.cuda(), wq, s, b, p.group_size, p.bits, True, path)
    torch.cuda.synchronize()
    return y


def check(p: Problem, M: int, path: str, rows=None):
    x = p.x(M)
    y = run(p, x, path)
    y_ref, a_ref = reference(x, p.wb, rows)
    got = y if rows is None else y[torch.as_tensor(rows, device=y.device)]
    assert_within_tolerance(got, y_ref, a_ref, f"{p.fmt} {path} M={M} N={p.N} K={p.K}")


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
@pytest.mark.parametrize("N,K", [(256, 512), (300, 1024)])
def test_small_all_paths(fmt, N, K):
    p = Problem(fmt, N, K, seed=N * 7 + K)
    for M in GEMV_M:
        check(p, M, "gemv")
        check(p, M, "auto")
    for M in TC_M:
        check(p, M, "tc_fused")
        check(p, M, "dequant_gemm")
        check(p, M, "auto")


def test_q4_0_ragged_k_uses_pair():
    p = Problem("q4_0", 130, 544, seed=5)      # K % 64 == 32: no fused tile, the pair handles it
    assert bq.quant_matmul_select_path(200, 130, 544, 32, 4) == bq.PATH_DEQUANT_GEMM
    for M in (1, 7, 40, 200):
        check(p, M, "auto")
    for M in (3, 32):
        check(p, M, "gemv")


@pytest.mark.parametrize("M", [1, 8, 32])
def test_q4_0_decode_config_full(M):
    p = Problem("q4_0", 12288, 4096)
    check(p, M, "auto")


def _sample_rows(M, n=64, seed=0):
    rng = np.random.default_rng(seed + M)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, size=min(n, M), replace=False)]))
    return rows


@pytest.mark.parametrize("fmt,M", [("affine4", 512), ("affine4", 2048), ("affine4", 8192),
                                   ("q4_0", 512), ("q4_0", 2048), ("q4_0", 4096)])
def test_prefill_config_sampled(fmt, M):
    """The 12288 x 4096 projection at prefill sizes: the fused kernel's plans
    there (split tail tiles at 512 and 2048 tokens, whole tiles at 4096 and
    8192) and the pair."""
    p = Problem(fmt, 12288, 4096)
    rows = _sample_rows(M)
    check(p, M, "auto", rows)
    check(p, M, "tc_fused", rows)
    check(p, M, "dequant_gemm", rows)


@pytest.mark.parametrize("M", [1, 32, 512, 2048, 8192])
def test_affine8_sweep_config(M):
    p = Problem("affine8", 12288, 4096)
    rows = None if M <= 32 else _sample_rows(M)
    check(p, M, "auto", rows)
    if M >= 512:
        check(p, M, "dequant_gemm", rows)


@pytest.mark.parametrize("M", [1, 512])
def test_llama_1b_layer_shapes(M):
    for i, (N, K) in enumerate(((2048, 2048), (512, 2048), (8192, 2048), (2048, 8192))):
        p = Problem("q4_0", N, K, seed=100 + i)
        check(p, M, "auto", None if M == 1 else _sample_rows(M, 32))


# ---------------------------------------------------------------- edge cases
PATHS_FOR = {1: ["gemv", "tc_fused", "dequant_gemm"], 64: ["tc_fused", "dequant_gemm"]}


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_one_hot_rows_are_exact(fmt):
    """x = e_k gives y[:, n] = dequant(W)[n][k] exactly (one exact product, already bf16)."""
    p = Problem(fmt, 200, 512, seed=9)
    for M, paths in ((32, ["gemv", "tc_fused", "dequant_gemm"]), (64, ["tc_fused", "dequant_gemm"])):
        ks = np.random.default_rng(M).choice(512, M, replace=False)
        x = torch.zeros(M, 512, dtype=torch.bfloat16)
        x[torch.arange(M), torch.as_tensor(ks)] = 1.0
        expect = f32(p.wb[:, ks].T.copy())
        for path in paths:
            y = run(p, x, path)
            # compared as values: the sign of an exact-zero sum is not fixed by the method
            assert np.array_equal(y.float().cpu().numpy(), expect), (fmt, M, path)


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_all_equal_weights_tight_tolerance(fmt):
    """x = 1 and every dequantized weight equal: |y| = sum|x w|, so the output's
    own bf16 rounding uses almost all of the tolerance."""
    N, K = 130, 1024
    if fmt == "q4_0":
        w = np.full((N, K), -0.0123456, np.float32)     # every code 0, d = w / -8 with 11 significant bits
    else:
        w = np.full((N, K), 0.0123456, np.float32)
        w = torch.from_numpy(w).to(torch.bfloat16).float().numpy()
    p = Problem(fmt, N, K, w=w)
    for M, paths in ((8, ["gemv", "tc_fused", "dequant_gemm"]), (100, ["tc_fused", "dequant_gemm"])):
        x = torch.ones(M, K, dtype=torch.bfloat16)
        y_ref, a_ref = reference(x, p.wb)
        assert np.allclose(np.abs(y_ref), a_ref)
        for path in paths:
            assert_within_tolerance(run(p, x, path), y_ref, a_ref, f"{fmt} {path} M={M}")


def test_zero_weights_give_zero():
    p = Problem("q4_0", 64, 256, w=np.zeros((64, 256), np.float32))
    for M, path in ((4, "gemv"), (4, "tc_fused"), (80, "tc_fused"), (80, "dequant_gemm")):
        y = run(p, p.x(M), path)
        assert torch.all(y.float() == 0), path


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_deterministic(fmt):
    p = Problem(fmt, 300, 1024, seed=3)
    for M, path in ((5, "gemv"), (32, "gemv"), (100, "tc_fused"), (100, "dequant_gemm")):
        x = p.x(M)
        ys = [u16(run(p, x, path)) for _ in range(3)]
        assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2]), (fmt, path)


def test_empty_problems():
    p = Problem("affine4", 64, 128)
    wq, s, b = p.device()
    x0 = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    assert bq.quant_matmul(x0, wq, s, b, 64, 4).shape == (0, 64)
    x = p.x(4).cuda()
    y = torch.full((4, 0), 1.0, dtype=torch.bfloat16, device="cuda")
    wq0 = torch.zeros(0, 16, dtype=torch.int32, device="cuda")
    s0 = torch.zeros(0, 2, dtype=torch.bfloat16, device="cuda")
    assert bq.quant_matmul(x, wq0, s0, s0, 64, 4).shape == (4, 0)
    # K == 0: an empty sum, y = 0
    xk = torch.zeros(3, 0, dtype=torch.bfloat16, device="cuda")
    wk = torch.zeros(5, 0, dtype=torch.uint8, device="cuda")
    sk = torch.zeros(5, 0, dtype=torch.float16, device="cuda")
    out = torch.full((3, 5), 7.0, dtype=torch.bfloat16, device="cuda")
    bq.quant_matmul(xk, wk, sk, None, 32, 4, out=out)
    torch.cuda.synchronize()
    assert torch.all(out.float() == 0)


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (37, 200, 72), (300, 129, 640), (64, 256, 8)])
def test_bf16_matmul(M, N, K):
    g = inputs.generator(M + N + K)
    x = inputs.activations_bf16(M, K, g)
    w = inputs.activations_bf16(N, K, g)
    y = bq.bf16_matmul(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, u16(w))
    assert_within_tolerance(y, y_ref, a_ref, f"bf16_matmul {M}x{N}x{K}")


def test_device_status_clean():
    assert bq.bq_device_status() == 0


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
@pytest.mark.parametrize("N,K", [(250, 1024), (1000, 2048), (130, 4096), (520, 8192)])
def test_gemv_shapes(fmt, N, K):
    """Decode sizes over ragged row tiles (N % 32 != 0) and several K."""
    p = Problem(fmt, N, K, seed=N + K)
    for M in (1, 3, 8, 17, 32):
        check(p, M, "gemv")


def test_gemv_many_rows_sampled():
    p = Problem("q4_0", 12288, 1024, seed=21)
    rows = list(range(0, 12288, 97)) + [12287]
    for M in (1, 8, 32):
        x = p.x(M)
        y = run(p, x, "gemv")
        y_ref, a_ref = reference(x, p.wb[rows])
        assert_within_tolerance(y[:, torch.as_tensor(rows, device=y.device)], y_ref, a_ref, f"M={M}")


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
@pytest.mark.parametrize("M", [1, 8, 32, 100])
def test_multi_matches_separate_calls(fmt, M):
    """quant_matmul_multi (Q/K/V-like: three matrices sharing x, ragged N) gives the
    same bits as separate quant_matmul calls, and each is within the oracle's bound."""
    K = 1024
    probs = [Problem(fmt, n, K, seed=n) for n in (300, 64, 130)]
    x = probs[0].x(M)
    xd = x.cuda()
    ws = [p.device() for p in probs]
    ys = bq.quant_matmul_multi(xd, ws, probs[0].group_size, probs[0].bits)
    torch.cuda.synchronize()
    for p, (wq, s, b), y in zip(probs, ws, ys):
        y1 = bq.quant_matmul(xd, wq, s, b, p.group_size, p.bits)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), (fmt, M, p.N)
        y_ref, a_ref = reference(x, p.wb)
        assert_within_tolerance(y, y_ref, a_ref, f"multi {fmt} M={M} N={p.N}")


@pytest.mark.parametrize("fmt", ["affine4_g32", "affine4_g128", "affine8_g32", "affine8_g128"])
@pytest.mark.parametrize("N,K", [(300, 1024), (130, 4096)])
def test_group_sizes_all_paths(fmt, N, K):
    """Affine group sizes 32 and 128 (mx.quantize's other sizes) on every path,
    including K-split fused tiles (few tiles) and windows of 4 or 16 k-blocks."""
    p = Problem(fmt, N, K, seed=N * 3 + K)
    for M in (1, 8, 32):
        check(p, M, "gemv")
    for M in (33, 100, 300):
        check(p, M, "tc_fused")
        check(p, M, "dequant_gemm")
        check(p, M, "auto")


@pytest.mark.parametrize("fmt", ["q4_0", "affine4"])
def test_odd_n_tensor_core_paths(fmt):
    """N odd: the epilogue's paired row stores do not apply and single stores are used."""
    p = Problem(fmt, 77, 512, seed=13)
    for M in (40, 300):
        check(p, M, "tc_fused")
        check(p, M, "dequant_gemm")


@pytest.mark.parametrize("fmt", ["q4_0", "affine8"])
def test_split_k_with_caller_workspace(fmt):
    """Few tiles (N = 300, M = 48): the fused kernel splits K.  With a caller
    workspace of the reported size it splits, with one too small it runs unsplit;
    with none it uses the library's.  All three agree with the oracle."""
    p = Problem(fmt, 300, 2048, seed=17)
    wq, s, b = p.device()
    M = 48
    x = p.x(M)
    need = bq.quant_matmul_workspace_size(M, 300, 2048, p.group_size, p.bits, "tc_fused")
    assert need > 0, "this shape is expected to split K"
    y_ref, a_ref = reference(x, p.wb)
    xd = x.cuda()
    for ws in (torch.empty(need, dtype=torch.uint8, device="cuda"),
               torch.empty(64, dtype=torch.uint8, device="cuda"), None):
        y = bq.quant_matmul_ex(xd, wq, s, b, p.group_size, p.bits, True, "tc_fused", workspace=ws)
        torch.cuda.synchronize()
        assert_within_tolerance(y, y_ref, a_ref, f"{fmt} ws={None if ws is None else ws.numel()}")


@pytest.mark.parametrize("fmt,M,N,K,sampled", [
    ("q4_0", 64, 19160, 1024, False),      # 150 tiles of 64 tokens: 148 whole, 2 split 4 ways
    ("affine4", 100, 18950, 1024, False),  # 149 tiles of 112 tokens (ragged), N % 4 == 2
    ("affine8", 400, 9750, 1024, True),    # one accumulator, 256-token tiles: 6 split tiles, ragged M and N
    ("affine4", 400, 9750, 1024, True),
    ("q4_0", 200, 19750, 1024, False),     # one accumulator, a 208-token tile
])
def test_split_tail_tiles(fmt, M, N, K, sampled):
    """More tiles than SMs: whole tiles fill the whole rounds and only the last
    round's tiles are split over K, their fp32 partials reduced in split order.
    The reported workspace holds only the split tiles' partials (every-tile
    splitting needs at least 2 x M x N x 4 bytes); with it, with one too small
    (no split) and with the library's, the result agrees with the oracle, and
    repeated runs are bit-identical."""
    p = Problem(fmt, N, K, seed=M + N)
    need = bq.quant_matmul_workspace_size(M, N, K, p.group_size, p.bits, "tc_fused")
    assert 0 < need < 2 * M * N * 4, need
    wq, s, b = p.device()
    x = p.x(M)
    rows = _sample_rows(M) if sampled else None
    y_ref, a_ref = reference(x, p.wb, rows)
    xd = x.cuda()
    outs = []
    for ws in (torch.empty(need, dtype=torch.uint8, device="cuda"),
               torch.empty(64, dtype=torch.uint8, device="cuda"), None):
        y = bq.quant_matmul_ex(xd, wq, s, b, p.group_size, p.bits, True, "tc_fused", workspace=ws)
        torch.cuda.synchronize()
        got = y if rows is None else y[torch.as_tensor(rows, device=y.device)]
        assert_within_tolerance(got, y_ref, a_ref, f"{fmt} M={M} N={N} ws={None if ws is None else ws.numel()}")
        outs.append(y)
    assert torch.equal(outs[0], outs[2])
    assert torch.equal(outs[0], bq.quant_matmul_ex(xd, wq, s, b, p.group_size, p.bits, True, "tc_fused"))
    assert bq.bq_device_status() == 0


@pytest.mark.parametrize("fmt", ["q4_0", "affine4", "affine8"])
def test_minimal_shapes_every_path(fmt):
    """One weight row, the smallest K of the format, and M at the path limits."""
    gs = 32 if fmt == "q4_0" else 64
    for N, K in ((1, max(gs, 64)), (1, 128), (17, 64 if fmt == "q4_0" else 128)):
        p = Problem(fmt, N, K, seed=N + K)
        for M in (1, 32):
            check(p, M, "gemv")
        for M in (1, 33, 129):
            check(p, M, "tc_fused")
            check(p, M, "dequant_gemm")
        check(p, 7, "auto")


def test_q4_0_smallest_k_gemv_and_pair():
    """K = 32 (one Q4_0 block): no 64-wide tensor-core k-block exists, so the
    auto path takes the GEMV or the pair."""
    p = Problem("q4_0", 40, 32, seed=2)
    for M in (1, 5, 32):
        check(p, M, "gemv")
    for M in (33, 200):
        check(p, M, "auto")
        check(p, M, "dequant_gemm")


# ---------------------------------------------------------------- 2-, 3-, 6-bit affine
@pytest.mark.parametrize("fmt", ["affine2", "affine3", "affine6", "affine3_g128", "affine6_g32"])
@pytest.mark.parametrize("M", [1, 8, 9, 33, 300])
def test_2_3_6_bit_pair(fmt, M):
    """2/3/6-bit widths: the any-width decode GEMV up to 8 tokens, the unfused pair
    above (and at every M when forced)."""
    N, K = 300, 1024
    p = Problem(fmt, N, K, seed=M + 11)
    wq, s, b = p.device()
    x = p.x(M)
    assert bq.quant_matmul_select_path(M, N, K, p.group_size, p.bits) == (1 if M <= 8 else 3)
    y_ref, a_ref = reference(x, p.wb)
    for path in (["auto", "gemv", "dequant_gemm"] if M <= 8 else ["auto"]):
        y = bq.quant_matmul_ex(x.cuda(), wq, s, b, p.group_size, p.bits, True, path)
        torch.cuda.synchronize()
        assert_within_tolerance(y, y_ref, a_ref, f"{fmt} M={M} {path}")


@pytest.mark.parametrize("bits", [2, 3, 6])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,K", [(1, 32), (17, 96), (250, 2048)])
def test_affine_any_width_gemv(bits, M, N, K):
    """Every token-count template and ragged row groups of the any-width GEMV."""
    p = Problem(f"affine{bits}_g32", N, K, seed=bits * 100 + M + N)
    wq, s, b = p.device()
    x = p.x(M)
    y = bq.quant_matmul_ex(x.cuda(), wq, s, b, 32, bits, True, "gemv")
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, f"bits={bits} M={M} {N}x{K}")


@pytest.mark.parametrize("bits", [2, 3, 6])
@pytest.mark.parametrize("M", [9, 16, 17, 32])
@pytest.mark.parametrize("N,K", [(17, 96), (250, 2048)])
def test_affine_any_width_gemv_passes(bits, M, N, K):
    """Forced beyond 8 tokens, the any-width GEMV runs in passes of 8 tokens (the
    last one ragged); each is checked against the oracle, and 33 tokens are
    rejected."""
    p = Problem(f"affine{bits}_g32", N, K, seed=bits * 300 + M + N)
    wq, s, b = p.device()
    x = p.x(M)
    y = bq.quant_matmul_ex(x.cuda(), wq, s, b, 32, bits, True, "gemv")
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, f"bits={bits} M={M} {N}x{K}")
    assert bq.quant_matmul_gemv_kernel(M, N, K, 32, bits, "gemv") == 3
    with pytest.raises(bq.BqError, match="UNSUPPORTED"):
        bq.quant_matmul_ex(p.x(33).cuda(), wq, s, b, 32, bits, True, "gemv")


# ---------------------------------------------------------------- transpose = 0
def _transposed_problem(bits: int, G: int, N: int, K: int, seed: int):
    """Affine W stored [K][N] (codes and groups along N), quantized by the oracle."""
    g = inputs.generator(seed)
    w = inputs.weights_bf16_valued(K, N, g).numpy()
    wq, sc, bi = oracle.affine_quantize(w, G, bits)
    wd = oracle.affine_dequantize(wq, sc, bi, G, bits)          # [K][N] bf16 bits
    dev = (torch.from_numpy(wq.view(np.int32)).cuda(),
           torch.from_numpy(sc.view(np.int16)).cuda().view(torch.bfloat16),
           torch.from_numpy(bi.view(np.int16)).cuda().view(torch.bfloat16))
    return dev, np.ascontiguousarray(wd.T), g                      # reference weight [N][K]


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (17, 320, 200), (130, 128, 1032), (300, 192, 64)])
def test_transpose0(bits, M, N, K):
    """y = x . W for W stored [K][N]: the pair with a transposing dequantize; K is
    any multiple of 8 (ragged tiles in both directions)."""
    (wq, s, b), w_ref, g = _transposed_problem(bits, 64, N, K, seed=bits * 1000 + M + K)
    x = inputs.activations_bf16(M, K, g)
    y = bq.quant_matmul(x.cuda(), wq, s, b, 64, bits, transpose=False)
    torch.cuda.synchronize()
    assert tuple(y.shape) == (M, N)
    y_ref, a_ref = reference(x, w_ref)
    assert_within_tolerance(y, y_ref, a_ref, f"transpose=0 bits={bits} {M}x{N}x{K}")


def test_transpose0_group_sizes_and_noalloc():
    for G, bits in ((32, 4), (128, 8), (32, 3)):
        (wq, s, b), w_ref, g = _transposed_problem(bits, G, 256, 136, seed=G + bits)
        x = inputs.activations_bf16(40, 136, g)
        y = bq.quant_matmul(x.cuda(), wq, s, b, G, bits, transpose=False)
        out = torch.empty(40, 256, dtype=torch.bfloat16, device="cuda")
        bq.quant_matmul_noalloc(x.cuda(), wq, s, b, out, G, bits, transpose=False)
        torch.cuda.synchronize()
        y_ref, a_ref = reference(x, w_ref)
        assert_within_tolerance(y, y_ref, a_ref, f"transpose=0 G={G} bits={bits}")
        assert torch.equal(out.view(torch.int16), y.view(torch.int16))


def test_2_3_6_bit_and_transpose0_edges():
    """Empty and minimal problems for the pair-only layouts; multi falls back to
    per-matrix calls for 3-bit weights with the same bits as separate calls."""
    dev = "cuda"
    for bits in (2, 3, 6):
        p = Problem(f"affine{bits}_g32", 5, 32, seed=bits)
        wq, s, b = p.device()
        for M in (0, 1, 3):
            x = p.x(M)
            y = bq.quant_matmul(x.cuda(), wq, s, b, 32, bits)
            torch.cuda.synchronize()
            assert tuple(y.shape) == (M, 5)
            if M:
                y_ref, a_ref = reference(x, p.wb)
                assert_within_tolerance(y, y_ref, a_ref, f"bits={bits} M={M} K=32")
    # transpose=0: empty M, N, and K = 0 (zeros)
    (wq, s, b), w_ref, g = _transposed_problem(4, 64, 64, 8, seed=5)
    y = bq.quant_matmul(torch.zeros(0, 8, dtype=torch.bfloat16, device=dev), wq, s, b, 64, 4, transpose=False)
    assert tuple(y.shape) == (0, 64)
    x = inputs.activations_bf16(3, 8, g)
    y = bq.quant_matmul(x.cuda(), wq, s, b, 64, 4, transpose=False)
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, w_ref)
    assert_within_tolerance(y, y_ref, a_ref, "transpose=0 K=8")
    # multi with 3-bit weights: per-matrix pair launches, identical to separate calls
    ps = [Problem("affine3", n, 256, seed=n) for n in (64, 128, 192)]
    devs = [q.device() for q in ps]
    x = ps[0].x(4).cuda()
    outs = bq.quant_matmul_multi(x, devs, 64, 3)
    for (wq, s, b), o in zip(devs, outs):
        sep = bq.quant_matmul(x, wq, s, b, 64, 3)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), sep.view(torch.int16))


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("K", [100, 300, 1000, 4200])
def test_transpose0_decode_gemv(bits, G, M, K):
    """transpose = 0 at decode sizes with 2-, 4- or 8-bit codes: the GEMV over
    [K][N] (any K, split over a cluster of 3 CTAs at K = 100 and up to 8 at K = 300,
    1000 and 4200, ragged per-CTA ranges; at K = 4200 each CTA's 525 rows take two
    passes of x staging; N a multiple of the group, ragged against the 256- and
    512-column clusters) is the dispatcher's choice up to 4 tokens (auto and forced
    give the same bits) and can be forced up to 8; quant_matmul_noalloc takes
    quant_matmul's path."""
    if K != 100 and M not in (1, 8):
        pytest.skip("K = 300, 1000 and 4200 at one and eight tokens")
    N = 6 * G + 32 if G == 32 else 3 * G
    (wq, s, b), w_ref, g = _transposed_problem(bits, G, N, K, seed=bits * 100 + G + M)
    x = inputs.activations_bf16(M, K, g).cuda()
    y_ref, a_ref = reference(x.cpu(), w_ref)
    y_g = bq.quant_matmul_ex(x, wq, s, b, G, bits, False, "gemv")
    torch.cuda.synchronize()
    assert_within_tolerance(y_g, y_ref, a_ref, f"transpose=0 GEMV bits={bits} G={G} M={M}")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    if M > 4 and K % 8 != 0:
        # above 4 tokens the dispatcher takes the pair, whose x rows must be 16-byte multiples
        with pytest.raises(bq.BqError, match="SHAPE"):
            bq.quant_matmul(x, wq, s, b, G, bits, transpose=False)
        with pytest.raises(bq.BqError, match="SHAPE"):
            bq.quant_matmul_noalloc(x, wq, s, b, out, G, bits, transpose=False)
        return
    y = bq.quant_matmul(x, wq, s, b, G, bits, transpose=False)
    bq.quant_matmul_noalloc(x, wq, s, b, out, G, bits, transpose=False)
    torch.cuda.synchronize()
    assert_within_tolerance(y, y_ref, a_ref, f"transpose=0 bits={bits} G={G} M={M}")
    assert torch.equal(y.view(torch.int16), out.view(torch.int16))
    if M <= 4:      # the dispatcher's own choice up to 4 tokens; forced above
        assert torch.equal(y.view(torch.int16), y_g.view(torch.int16))


def test_transpose0_decode_limits():
    """3- and 6-bit codes and M > 8 keep the pair (forcing the GEMV there is
    unsupported); the pair and the GEMV agree within the tolerance."""
    (wq, s, b), w_ref, g = _transposed_problem(3, 64, 128, 64, seed=3)
    x = inputs.activations_bf16(2, 64, g)
    with pytest.raises(bq.BqError, match="UNSUPPORTED"):
        bq.quant_matmul_ex(x.cuda(), wq, s, b, 64, 3, False, "gemv")
    (wq, s, b), w_ref, g = _transposed_problem(4, 64, 128, 64, seed=4)
    x9 = inputs.activations_bf16(9, 64, g)
    with pytest.raises(bq.BqError, match="UNSUPPORTED"):
        bq.quant_matmul_ex(x9.cuda(), wq, s, b, 64, 4, False, "gemv")
    x = inputs.activations_bf16(4, 64, g)
    y_pair = bq.quant_matmul_ex(x.cuda(), wq, s, b, 64, 4, False, "dequant_gemm")
    y_gemv = bq.quant_matmul_ex(x.cuda(), wq, s, b, 64, 4, False, "gemv")
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, w_ref)
    assert_within_tolerance(y_pair, y_ref, a_ref, "pair")
    assert_within_tolerance(y_gemv, y_ref, a_ref, "gemv")
    assert bq.bq_device_status() == 0
