"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
entry point the header declares, rejects bad arguments before launching
anything, and the M-threshold dispatcher picks the expected path at the
boundaries (after the host-predicate gates of the vllm.cpp issue page, Gates:
T=1 / T=19 / T=64 checks of a token-count route)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bqgemm.h")


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build()
    import bit_quantized_gemm_quant_b200 as bq
    return bq.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^BQ_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("q4_0_dequantize", "affine_dequantize", "quant_matmul"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(declared_functions()) <= exported


def test_status_strings_and_version(L):
    for code in range(9):
        assert L.bq_status_string(code)
    assert L.bq_status_string(99) == b"unknown bq_status"
    assert L.bq_version() >= 100


P = ctypes.c_void_p
ALIGNED = P(0x1000)
MISALIGNED = P(0x1008)


def qmm(L, x=ALIGNED, wq=ALIGNED, s=ALIGNED, b=None, y=ALIGNED, M=16, N=256, K=512, g=32, bits=4, tr=1, path=0,
        ws=None, wsb=0):
    return L.quant_matmul_ex(x, wq, s, b, y, M, N, K, g, bits, tr, path, ws, wsb, None)


def test_quant_matmul_rejects_before_launch(L):
    # every case fails validation on the host, so no CUDA call is ever made
    assert qmm(L, tr=0) == 3                                  # transpose=0 unsupported
    assert qmm(L, path=7) == 3
    assert qmm(L, M=-1) == 2
    assert qmm(L, N=-1) == 2
    assert qmm(L, K=48) == 2                                  # Q4_0 needs K % 32 == 0
    assert qmm(L, bits=8) == 3                                # Q4_0 is 4-bit only
    assert qmm(L, g=64) == 3                                  # ... with group 32
    assert qmm(L, b=ALIGNED, g=16, bits=4) == 3               # affine groups: 32, 64 or 128
    assert qmm(L, b=ALIGNED, g=64, bits=5) == 3               # bits in {2, 3, 4, 6, 8}
    assert qmm(L, b=ALIGNED, g=64, bits=7) == 3
    assert qmm(L, tr=2) == 3
    assert qmm(L, b=ALIGNED, g=64, bits=3, M=33, path=1) == 3  # 2/3/6-bit: forced GEMV to M = 32 (passes of 8)
    assert qmm(L, b=ALIGNED, g=64, bits=6, M=64, path=2) == 3
    assert qmm(L, b=ALIGNED, g=64, bits=2, M=64, path=2) == 3
    assert qmm(L, b=ALIGNED, g=64, tr=0, path=1) == 3         # transpose=0: GEMV to M = 8, then the pair
    assert qmm(L, b=ALIGNED, g=64, tr=0, M=4, bits=3, path=1) == 3  # ... for 2-, 4- and 8-bit codes
    assert qmm(L, b=ALIGNED, g=64, tr=0, M=4, path=2) == 3
    assert qmm(L, b=ALIGNED, g=64, tr=0, M=1, path=4) == 3
    assert qmm(L, b=ALIGNED, g=64, tr=0, M=64, path=2) == 3
    assert qmm(L, b=ALIGNED, g=64, tr=0, K=12) == 2           # the pair needs K % 8 == 0
    assert qmm(L, b=ALIGNED, g=64, tr=0, M=4, bits=3, K=12) == 2
    assert qmm(L, b=ALIGNED, g=64, tr=0, N=96) == 2           # ... and groups along N
    assert qmm(L, b=ALIGNED, g=64, bits=4, K=96) == 2         # K % group
    assert qmm(L, x=None) == 1
    assert qmm(L, wq=None) == 1
    assert qmm(L, s=None) == 1
    assert qmm(L, y=None) == 1
    assert qmm(L, x=MISALIGNED) == 4
    assert qmm(L, y=MISALIGNED) == 4
    assert qmm(L, b=MISALIGNED, g=64) == 4
    assert qmm(L, M=64, path=1) == 3                          # GEMV is M <= 32 only
    assert qmm(L, K=544, M=64, path=2) == 3                   # fused TC needs K % 64 == 0
    assert qmm(L, M=64, path=3, ws=ALIGNED, wsb=16) == 7      # workspace too small
    assert L.quant_matmul(ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 16, 256, 512, 32, 4, 0, None) == 3


def test_other_entry_points_reject_before_launch(L):
    assert L.q4_0_dequantize(ALIGNED, ALIGNED, ALIGNED, 4, 48, None) == 2
    assert L.q4_0_dequantize(None, ALIGNED, ALIGNED, 4, 64, None) == 1
    assert L.q4_0_dequantize(MISALIGNED, ALIGNED, ALIGNED, 4, 64, None) == 4
    assert L.affine_dequantize(ALIGNED, ALIGNED, None, ALIGNED, 4, 64, 64, 4, None) == 1
    assert L.affine_dequantize(ALIGNED, ALIGNED, ALIGNED, ALIGNED, 4, 64, 64, 5, None) == 3
    assert L.affine_dequantize(ALIGNED, ALIGNED, ALIGNED, ALIGNED, 4, 96, 64, 4, None) == 2
    assert L.bf16_matmul(ALIGNED, ALIGNED, ALIGNED, 4, 4, 12, None) == 2
    assert L.bf16_matmul(None, ALIGNED, ALIGNED, 4, 4, 16, None) == 1
    assert L.q4_0_quantize(ALIGNED, ALIGNED, MISALIGNED, 4, 64, None) == 4
    assert L.affine_quantize(ALIGNED, ALIGNED, ALIGNED, ALIGNED, 4, 64, 16, 4, None) == 3


BOUNDARY_M = [1, 2, 8, 19, 31, 32, 33, 63, 64, 65, 127, 128, 129, 383, 384, 385, 511, 512, 513, 1023, 1024, 1025,
              2047, 2048, 2049, 4095, 4096, 4097, 8192]


def test_dispatcher_pair_only_widths(L):
    for bits in (2, 3, 6):
        for M in (1, 8, 9, 32, 33, 512, 4096):
            assert L.quant_matmul_select_path(M, 12288, 4096, 64, bits) == (1 if M <= 8 else 3)
        assert L.quant_matmul_workspace_size(8, 256, 512, 64, bits, 0) == 0              # GEMV
        assert L.quant_matmul_workspace_size(9, 256, 512, 64, bits, 0) == 256 * 512 * 2  # the pair
        assert L.quant_matmul_workspace_size(8, 256, 512, 64, bits, 2) == 0


def test_dispatcher_boundaries(L):
    for M in BOUNDARY_M:
        for g, bits in ((32, 4), (64, 4), (64, 8)):
            p = L.quant_matmul_select_path(M, 12288, 4096, g, bits)
            pair_min = 2048 if bits == 8 else 4096
            tc_min = 17 if bits == 8 else 21
            assert p == (1 if M < tc_min else 2 if M < pair_min else 3), (M, g, bits, p)
    # K % 64 != 0 (Q4_0 only): prefill goes through the unfused pair
    assert L.quant_matmul_select_path(512, 256, 544, 32, 4) == 3
    assert L.quant_matmul_select_path(8, 256, 544, 32, 4) == 1
    assert L.quant_matmul_select_path(32, 256, 544, 32, 4) == 1     # no fused tile: GEMV up to 32
    assert L.quant_matmul_select_path(33, 256, 544, 32, 4) == 3
    assert L.quant_matmul_select_path(-1, 256, 512, 32, 4) == -1
    assert L.quant_matmul_select_path(8, 256, 512, 64, 5) == -1
    assert L.quant_matmul_workspace_size(512, 256, 544, 32, 4, 0) == 256 * 544 * 2
    assert L.quant_matmul_workspace_size(512, 256, 512, 32, 4, 0) == 0
    assert L.quant_matmul_workspace_size(512, 256, 512, 64, 8, 3) == 256 * 512 * 2


TILE_PARTIAL = 128 * 4          # fp32 bytes per token of one 128-row split tile


@pytest.mark.parametrize("M,N,K,g,bits,want", [
    # 12288 x 4096 projection (96 weight tiles), on a B200's 148 SMs
    (64, 12288, 4096, 64, 4, 3 * 96 * 64 * TILE_PARTIAL),    # 96 tiles of 64 tokens, every one split 3 ways
    (256, 12288, 4096, 64, 4, 0),                            # 96 whole 256-token tiles
    (512, 12288, 4096, 64, 4, 3 * 44 * 256 * TILE_PARTIAL),  # 192 tiles: 148 whole, the other 44 split 3 ways
    (512, 12288, 4096, 32, 4, 3 * 44 * 256 * TILE_PARTIAL),  # Q4_0: the same plan
    (1024, 12288, 4096, 64, 4, 0),                           # 384 whole tiles: 88 left over, too many to split
    (2048, 12288, 4096, 64, 4, 5 * 28 * 256 * TILE_PARTIAL), # 768 tiles: 740 whole, 28 split 5 ways
    (3072, 12288, 4096, 64, 4, 0),
    (4096, 12288, 4096, 32, 4, 0),                           # 1536 tiles: splitting the last 56 does not pay
    (2048, 12288, 4096, 64, 8, 5 * 28 * 256 * TILE_PARTIAL), # affine 8-bit, fused path forced
    # the split-tail parity cases of the GPU tests
    (64, 19160, 1024, 32, 4, 4 * 2 * 64 * TILE_PARTIAL),     # 150 tiles: 2 split 4 ways
    (100, 18950, 1024, 64, 4, 4 * 1 * 112 * TILE_PARTIAL),   # 149 tiles of 112 tokens: 1 split 4 ways
    (400, 9750, 1024, 64, 8, 4 * 6 * 256 * TILE_PARTIAL),    # 154 tiles: 6 split 4 ways
    (200, 19750, 1024, 32, 4, 4 * 7 * 208 * TILE_PARTIAL),   # 155 tiles of 208 tokens: 7 split 4 ways
])
def test_fused_plan_workspace(L, M, N, K, g, bits, want):
    """The fused kernel's K-split plan, seen through the workspace it asks for:
    fp32 partials only for the split tiles (splits x split tiles x bn x 128)."""
    assert L.quant_matmul_workspace_size(M, N, K, g, bits, 2) == want


def _select_in_subprocess(env_extra, Ms):
    code = ("import sys; sys.path.insert(0, %r); import bit_quantized_gemm_quant_b200 as bq; "
            "print([bq.quant_matmul_select_path(m, 4096, 4096, 64, 4) for m in %r])" % (ROOT, Ms))
    env = dict(os.environ, **env_extra)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, check=True)
    return eval(out.stdout.strip())


def test_dispatcher_env_overrides(L):
    Ms = [1, 8, 19, 32, 33, 512, 4096]
    assert _select_in_subprocess({}, Ms) == [1, 1, 1, 2, 2, 2, 3]             # affine 4-bit: fused from 21, pair from 4096
    assert _select_in_subprocess({"BQ_TC_MIN_M": "8"}, Ms) == [1, 2, 2, 2, 2, 2, 3]
    assert _select_in_subprocess({"BQ_TC_MIN_M": "1000"}, Ms) == [1, 1, 1, 1, 2, 2, 3]   # clamped to 33
    assert _select_in_subprocess({"BQ_PAIR_MIN_M": "512"}, Ms) == [1, 1, 1, 2, 2, 3, 3]
    assert _select_in_subprocess({"BQ_PAIR_MIN_M": "0"}, Ms) == [1, 1, 1, 2, 2, 2, 2]


def test_empty_problems_need_no_pointers(L):
    # empty shapes return BQ_OK before any pointer is looked at (torch gives NULL for empty tensors)
    assert qmm(L, x=None, wq=None, s=None, y=None, M=0) == 0
    assert qmm(L, x=None, wq=None, s=None, y=None, N=0) == 0
    assert qmm(L, y=None, K=0) == 1                   # K == 0 still writes y = 0
    assert L.q4_0_dequantize(None, None, None, 0, 64, None) == 0
    assert L.affine_dequantize(None, None, None, None, 4, 0, 64, 8, None) == 0
    assert L.bf16_matmul(None, None, None, 0, 4, 16, None) == 0
    assert L.q4_0_quantize(None, None, None, 0, 64, None) == 0


def test_q4_0_import_aos_validation(L):
    assert L.q4_0_import_aos(ALIGNED, ALIGNED, ALIGNED, 4, 48, None) == 2        # K % 32
    assert L.q4_0_import_aos(None, ALIGNED, ALIGNED, 4, 64, None) == 1
    assert L.q4_0_import_aos(MISALIGNED, ALIGNED, ALIGNED, 4, 64, None) == 4
    assert L.q4_0_import_aos(None, None, None, 0, 64, None) == 0                  # empty: nothing touched


def test_quant_matmul_multi_validation(L):
    VP = ctypes.c_void_p * 2
    ptrs = VP(ALIGNED, ALIGNED)
    n = (ctypes.c_int64 * 2)(256, 128)
    assert L.quant_matmul_multi(ALIGNED, 2, ptrs, ptrs, None, ptrs, n, 4, 48, 32, 4, 1, None) == 2     # K % 32
    assert L.quant_matmul_multi(ALIGNED, 9, ptrs, ptrs, None, ptrs, n, 4, 64, 32, 4, 1, None) == 3     # count > 8
    assert L.quant_matmul_multi(ALIGNED, 2, ptrs, ptrs, None, ptrs, n, 4, 64, 32, 4, 0, None) == 3     # transpose
    assert L.quant_matmul_multi(ALIGNED, 2, None, ptrs, None, ptrs, n, 4, 64, 32, 4, 1, None) == 1
    assert L.quant_matmul_multi(MISALIGNED, 2, ptrs, ptrs, None, ptrs, n, 4, 64, 32, 4, 1, None) == 4
    assert L.quant_matmul_multi(None, 0, None, None, None, None, None, 4, 64, 32, 4, 1, None) == 0     # nothing


def test_q8_path_validation(L):
    assert L.q8_1_quantize(ALIGNED, ALIGNED, ALIGNED, ALIGNED, 2, 48, None) == 2             # K % 32
    assert L.q8_1_quantize(None, ALIGNED, ALIGNED, ALIGNED, 2, 64, None) == 1
    assert L.q8_1_quantize(ALIGNED, MISALIGNED, ALIGNED, ALIGNED, 2, 64, None) == 4
    assert L.q8_1_quantize(None, None, None, None, 0, 64, None) == 0
    assert L.quant_matmul_q8(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 2, 8, 40, None) == 2
    assert L.quant_matmul_q8(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 2, 8, 64, None) == 1
    assert L.quant_matmul_q8(None, None, None, None, None, None, 2, 0, 64, None) == 0


def test_decode_gemv_table_workspace(L):
    """The streamed GEMV (one or two tokens): the TMA-fed kernel, which applies when a
    row's codes split into stages of 8 or 16 128-byte chunks, builds its activation
    tables in shared memory and needs no workspace; the cp.async kernel, which takes
    the other shapes, needs its tables in device scratch: K/32 x 256 bytes of byte
    slices, K/group x 64 bytes of group scales and sums, a flag word per 2048
    activations rounded up to 16 bytes.  Forced (path 4) for every format; through
    the GEMV path (1, and AUTO) only where it is the dispatcher's choice (one or two
    tokens, K >= 4096 and 4 tiles per SM); none from three tokens on."""
    def tables(M, K, g):
        flags = -(-M * K // 2048)
        return K // 32 * 256 + K // g * 64 + (flags * 4 + 15) // 16 * 16
    for g, bits in ((32, 4), (64, 4), (64, 8), (128, 8), (32, 8), (128, 4)):
        for M in (1, 2):
            assert L.quant_matmul_workspace_size(M, 12288, 4096, g, bits, 4) == 0, (g, bits, M)   # TMA-fed
            assert L.quant_matmul_workspace_size(M, 12288, 4096, g, bits, 1) == 0
        assert L.quant_matmul_workspace_size(3, 12288, 4096, g, bits, 4) == 0
    for M in (1, 2):
        # K = 768: 384- or 768-byte rows, not whole 8-chunk stages: the cp.async kernel
        assert L.quant_matmul_workspace_size(M, 300, 768, 32, 4, 4) == tables(M, 768, 32)
        assert L.quant_matmul_workspace_size(M, 300, 768, 32, 8, 4) == tables(M, 768, 32)
        # not the dispatcher's choice here (K < 4096, 19 tiles): the register-streaming GEMV
        assert L.quant_matmul_workspace_size(M, 300, 768, 32, 4, 1) == 0
        assert L.quant_matmul_workspace_size(M, 300, 768, 32, 8, 1) == 0
    assert L.quant_matmul_workspace_size(1, 256, 544, 32, 4, 4) == 0      # K not a multiple of 8 blocks
    assert L.quant_matmul_workspace_size(1, 256, 512, 64, 3, 4) == 0      # 3-bit: no streamed kernel


def test_decode_kernel_query(L):
    """quant_matmul_gemv_kernel names the decode kernel that runs (host only; B200
    shared memory assumed without a device): 1 = TMA-fed streamed, 2 = cp.async
    streamed with its table kernel, 0 = register-streaming, 3 = any-width, -1 = none."""
    q = L.quant_matmul_gemv_kernel
    assert q(1, 12288, 4096, 32, 4, 0) == 1                # Q4_0, one token: streamed
    assert q(2, 12288, 4096, 32, 4, 0) == 1                # Q4_0, two tokens: streamed
    assert q(2, 12288, 4096, 64, 4, 0) == 1                # affine 4-bit, two tokens: streamed
    assert q(2, 12288, 4096, 64, 8, 0) == 1
    assert q(8, 12288, 4096, 64, 8, 0) == 0
    assert q(2, 12288, 4096, 32, 4, 4) == 1                # forced
    assert q(1, 300, 768, 32, 8, 4) == 2                   # 768-byte rows: the cp.async kernel
    assert q(1, 300, 768, 32, 8, 0) == 0                   # small: the register-streaming kernel
    assert q(1, 2048, 4096, 32, 4, 0) == 0                 # 128 tiles on 148 SMs
    assert q(1, 8192, 2048, 32, 4, 0) == 0                 # K < 4096
    assert q(3, 12288, 4096, 32, 4, 4) == -1               # forced beyond two tokens
    assert q(1, 12288, 4096, 64, 3, 0) == 3                # 3-bit: any-width GEMV
    assert q(8, 12288, 4096, 64, 6, 0) == 3                # ... up to 8 tokens by the dispatcher
    assert q(9, 12288, 4096, 64, 2, 0) == -1               # then the pair
    assert q(32, 12288, 4096, 64, 2, 1) == 3               # forced: passes of 8 tokens to 32
    assert q(33, 12288, 4096, 64, 2, 1) == -1
    assert q(64, 12288, 4096, 32, 4, 0) == -1              # prefill: not a decode path
    assert q(0, 12288, 4096, 32, 4, 0) == -1
