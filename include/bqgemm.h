/*
 * bqgemm.h -- C ABI of the B200 (sm_100a) weight-only block-quantized matmul
 * library, libbqgemm.so.
 *
 * The library computes y[M,N] = x[M,K] . dequant(Wq)[N,K]^T with bf16
 * activations x, bf16 output y and fp32 accumulation, for two weight formats:
 *
 *  - Q4_0, the llama.cpp format of "et-backend: Q4_0 matrix-engine GEMM
 *    rewrite for prefill" (Overview) and of the SYCL "reordered" MMVQ path of
 *    "2026-05-06 Q4 sync-after focused repro" (Important source touch points).
 *    Blocks of 32 weights along K share one fp16 scale d; w = d * (q - 8),
 *    q in [0, 15].  Layout (the "reordered" two-plane form):
 *      wq     u8   [N][K/2]   byte j of block b of row n at n*K/2 + 16*b + j,
 *                             low nibble = element 32b + j,
 *                             high nibble = element 32b + j + 16
 *      scales fp16 [N][K/32]  (raw IEEE half bits)
 *
 *  - MLX-style affine, the format of mx.quantize / mx.dequantize /
 *    mx.quantized_matmul on "quantized_matmul takes 14-41% longer than
 *    dequantize + bf16 matmul at prefill sizes (> 512 tokens)" (Repro).
 *    Groups of group_size weights along K share a bf16 scale and a bf16 bias;
 *    w = scale * q + bias, q in [0, 2^bits - 1], bits in {2, 3, 4, 6, 8},
 *    group_size in {32, 64, 128} (the widths and sizes mx.quantize accepts; the
 *    page's workloads use 4 and 8 bits with groups of 64).
 *      wq      u32  [N][K*bits/32]  each row a little-endian bit stream: element
 *                                   k at stream bits bits*k .. bits*k + bits - 1,
 *                                   stream bit i = bit i % 32 of word i / 32.
 *                                   For 2, 4 and 8 bits: 32/bits elements per
 *                                   word, lowest bits first; 3- and 6-bit
 *                                   elements may cross a word (reading: the page
 *                                   shows 4 and 8 bits only, whose packing is
 *                                   exactly this stream)
 *      scales  bf16 [N][K/group_size]
 *      biases  bf16 [N][K/group_size]
 *
 * Tensors are row-major and contiguous: x bf16 [M][K], y bf16 [M][N],
 * W (and its dequantized form) [N][K] -- the transpose=True convention of
 * mx.quantized_matmul, one output feature per weight row.
 *
 * Conventions for every entry point below:
 *  - Pointers marked "device" are device (HBM) addresses; the caller owns
 *    every buffer and the library never frees caller memory.
 *  - Device pointers must be 16-byte aligned (BQ_ERR_ALIGN otherwise).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and the call returns without waiting for it.
 *  - Arguments are checked on the host before anything is launched; a failed
 *    check returns its error code and enqueues nothing.  A launch failure
 *    returns BQ_ERR_CUDA.  Errors raised later on the device (a bounded wait
 *    that ran out) are reported by bq_device_status().
 *  - M == 0 or N == 0 is an empty problem and returns BQ_OK with no work.
 *  - There is no CPU fallback: every call runs on the current CUDA device.
 */
#ifndef BQGEMM_H
#define BQGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BQ_API __attribute__((visibility("default")))
#else
#define BQ_API
#endif

typedef struct CUstream_st* bq_stream_t;   /* same type as cudaStream_t */

typedef enum {
    BQ_OK = 0,
    BQ_ERR_NULL = 1,          /* a required pointer is NULL */
    BQ_ERR_SHAPE = 2,         /* negative size, or K not a multiple of the block / group */
    BQ_ERR_UNSUPPORTED = 3,   /* bits / group_size / transpose / path not supported */
    BQ_ERR_ALIGN = 4,         /* a device pointer is not 16-byte aligned */
    BQ_ERR_CUDA = 5,          /* a CUDA runtime or launch error */
    BQ_ERR_TIMEOUT = 6,       /* a device-side bounded wait ran out (see bq_device_status) */
    BQ_ERR_WORKSPACE = 7,     /* the caller's workspace is missing or too small */
    BQ_ERR_DEVICE = 8         /* the current device is not sm_100 */
} bq_status;

/* Kernel paths of quant_matmul_ex. */
typedef enum {
    BQ_PATH_AUTO = 0,          /* the M-threshold dispatcher chooses (quant_matmul_select_path) */
    BQ_PATH_GEMV = 1,          /* decode path, M <= 32: the faster of the two decode kernels below */
    BQ_PATH_TC_FUSED = 2,      /* prefill path: on-chip dequant feeding a tcgen05/TMEM GEMM */
    BQ_PATH_DEQUANT_GEMM = 3,  /* the unfused pair: *_dequantize into a bf16 workspace, then bf16_matmul */
    BQ_PATH_GEMV_STREAM = 4    /* the streamed integer-MMA decode kernel, forced (M <= 2) */
} bq_path;

/* The two decode kernels of BQ_PATH_GEMV (Q4_0, affine 4- and 8-bit):
 *  - register-streaming: codes dequantized to bf16 in registers, warp MMAs, M <= 32;
 *  - streamed integer-MMA (M <= 2, K a multiple of 8 groups): W streams through
 *    shared memory into m16n8k32 integer MMAs that multiply the codes exactly by
 *    the activations split into signed bytes, each group's scale applied once to
 *    its sum; a small first kernel builds those activation tables.
 * BQ_PATH_GEMV takes the streamed kernel for affine 8-bit with one or two tokens
 * (measured faster on B200) and the register-streaming kernel otherwise.
 * BQ_PATH_GEMV_STREAM forces the streamed kernel for any of the three formats
 * (BQ_ERR_UNSUPPORTED where it does not apply).  Both give the product within
 * the GEMM tolerance; the streamed kernel computes with the exact weights
 * d (q - 8) or s q + z, the register-streaming one with their bf16 roundings. */

/*
 * q4_0_dequantize -- out[n][k] = bf16_rne(fp32(d[n][k/32]) * (q[n][k] - 8)).
 * The fp32 product is exact, so the result is bit-exact with the plain
 * definition (sign of zero included).  The dequantize half of the workaround
 * on the MLX issue page (Repro: x @ mx.dequantize(...).T), for Q4_0.
 *   wq         device u8   [N][K/2]   packed codes (layout above)
 *   scales_f16 device u16  [N][K/32]  fp16 bits of d
 *   out_bf16   device u16  [N][K]     bf16 bits, written
 *   N, K       N >= 0, K >= 0, K % 32 == 0
 */
BQ_API bq_status q4_0_dequantize(const uint8_t* wq, const uint16_t* scales_f16, uint16_t* out_bf16,
                          int64_t N, int64_t K, bq_stream_t stream);

/*
 * affine_dequantize -- out[n][k] = bf16_rne(fmaf(scale, q, bias)) for the group
 * of k: one fp32 fused multiply-add, one rounding to bf16.  mx.dequantize on
 * the MLX issue page (Repro).
 *   wq          device u32 [N][K*bits/32]
 *   scales_bf16 device u16 [N][K/group_size]
 *   biases_bf16 device u16 [N][K/group_size]
 *   out_bf16    device u16 [N][K], written
 *   group_size  32, 64 or 128;  bits  2, 3, 4, 6 or 8;  K % group_size == 0
 * (A matrix stored the other way round -- codes and groups along N, as
 * quant_matmul's transpose = 0 takes it -- is dequantized by passing its rows
 * as N and its codes per row as K.)
 */
BQ_API bq_status affine_dequantize(const uint32_t* wq, const uint16_t* scales_bf16, const uint16_t* biases_bf16,
                            uint16_t* out_bf16, int64_t N, int64_t K, int group_size, int bits,
                            bq_stream_t stream);

/*
 * q4_0_import_aos -- split array-of-structs Q4_0 blocks into the separate code
 * and scale arrays every other call here takes.  Reading of the pages: the
 * SYCL page "2026-05-06 Q4 sync-after focused repro" (Important source touch
 * points) runs its decode kernels on "reordered" Q4_0, i.e. on ggml's Q4_0
 * blocks moved into separate arrays; the block read here is ggml's: the fp16
 * scale d (little-endian), then the 16 code bytes in the nibble order of wq.
 *   blocks      device u8 [N][K/32][18], read
 *   wq          device u8 [N][K/2], written (16 bytes per block)
 *   scales_f16  device u16 [N][K/32], written
 *   K % 32 == 0; all pointers 16-byte aligned (BQ_ERR_ALIGN otherwise).
 * Bit-exact byte moves; stream-ordered; the caller owns every buffer.
 */
BQ_API bq_status q4_0_import_aos(const uint8_t* blocks, uint8_t* wq, uint16_t* scales_f16, int64_t N, int64_t K,
                                 bq_stream_t stream);

/*
 * q8_1_quantize -- activations to the int8 form of the quantized-activation
 * decode path.  Reading of the SYCL page "2026-05-06 Q4 sync-after focused
 * repro" (Important source touch points: its Q4_0 x Q8_1 matrix-vector kernels;
 * the page does not print the Q8_1 format).  Per block of 32 consecutive
 * elements of a token row: amax = max |x|, d = amax / 127 (fp32),
 * id = d != 0 ? 1 / d : 0, q = roundf(x * id) (half away from zero, in
 * [-127, 127]), qsum = the sum of the block's q.
 *   x_bf16  device u16 [M][K];  xq device i8 [M][K];  dx device f32 [M][K/32];
 *   qsum device i32 [M][K/32].  K % 32 == 0; pointers 16-byte aligned.
 * Bit-exact with the plain definition (IEEE division and product, one rounding each).
 */
BQ_API bq_status q8_1_quantize(const uint16_t* x_bf16, int8_t* xq, float* dx, int32_t* qsum, int64_t M, int64_t K,
                               bq_stream_t stream);

/*
 * quant_matmul_q8 -- Q4_0 weights times quantized activations (q8_1_quantize):
 *   y[m][n] = bf16( sum_b d[n][b] * dx[m][b] * sum_j xq[m][32b+j] * (q[n][32b+j] - 8) ).
 * The block dot products are exact integers; the per-block scaling and the sum
 * over blocks are fp32.  An approximation of quant_matmul (by the activation
 * quantization: at most dx / 2 per activation), offered as a separate path.
 *   xq, dx, qsum  as written by q8_1_quantize for the same M, K
 *   wq device u8 [N][K/2];  scales_f16 device u16 [N][K/32];  y_bf16 device u16 [M][N]
 *   Any M (8 tokens per launch); errors as quant_matmul.
 */
BQ_API bq_status quant_matmul_q8(const int8_t* xq, const float* dx, const int32_t* qsum, const uint8_t* wq,
                                 const uint16_t* scales_f16, uint16_t* y_bf16, int64_t M, int64_t N, int64_t K,
                                 bq_stream_t stream);

/*
 * quant_matmul -- y[M][N] = bf16_rne(sum_k x[m][k] * dequant(W)[n][k]), fp32
 * accumulation.  mx.quantized_matmul(x, wq, scales, biases, transpose=True,
 * group_size, bits) on the MLX issue page (Repro); its result equals
 * x @ dequantize(...).T up to accumulation order.
 *   x_bf16   device u16 [M][K]
 *   wq       device: u8 [N][K/2] (Q4_0) or u32 [N][K*bits/32] (affine)
 *   scales   device: fp16 [N][K/32] (Q4_0) or bf16 [N][K/group_size] (affine)
 *   biases   device bf16 [N][K/group_size]; NULL selects Q4_0 (then bits must be
 *            4 and group_size 32)
 *   y_bf16   device u16 [M][N], written
 *   transpose  1: W stored [N][K] as above.  0 (affine only; Q4_0 returns
 *            BQ_ERR_UNSUPPORTED): y = x . W with W stored [K][N], codes and
 *            groups along N -- wq u32 [K][N*bits/32], scales/biases bf16
 *            [K][N/group_size], N % group_size == 0 -- the transpose=False form
 *            of mx.quantized_matmul.  Up to 4 tokens of 2-, 4- or 8-bit codes
 *            run a decode GEMV over the [K][N] layout (any K; a cluster of up
 *            to 8 CTAs splits K and sums its partials in a fixed order; up to
 *            8 tokens when BQ_PATH_GEMV is forced); other sizes run the
 *            unfused pair, W dequantized into its [N][K] transpose, which
 *            needs K % 8 == 0 (BQ_ERR_SHAPE otherwise).
 *            Other values: BQ_ERR_UNSUPPORTED.
 * Affine 2-, 3- and 6-bit weights have a decode GEMV up to 8 tokens (over the
 * exact weights scale*q + bias, within the GEMM tolerance of their bf16
 * roundings; forced with BQ_PATH_GEMV it takes up to 32 tokens, in launches of
 * 8 tokens that each read W) and run as the unfused pair above that; 4- and 8-bit and Q4_0 have
 * the decode GEMV and the fused kernel as well.  With transpose = 0 only the
 * GEMV over [K][N] (see transpose) and the pair exist.
 * The path is chosen by quant_matmul_select_path.  A path that needs scratch
 * memory (the unfused pair's bf16 copy of W, the fused kernel's split-K
 * partial sums, the decode GEMV's activation tables for one or two tokens)
 * uses a library buffer, one per (device, stream):
 *   - it is allocated on first need and grows on demand; a call that
 *     allocates must not be made during stream capture, so make one call per
 *     stream and problem size before capturing;
 *   - growing never frees the old block (it is kept until the process exits),
 *     so graphs captured before a growth stay valid;
 *   - calls on one stream are ordered and share the stream's buffer safely;
 *     calls on different streams use different buffers and do not race;
 *   - a captured graph keeps the buffer of the stream it was captured on:
 *     replays of it must not overlap on the GPU with each other or with
 *     other calls that use that stream's buffer.
 */
BQ_API bq_status quant_matmul(const uint16_t* x_bf16, const void* wq, const void* scales, const void* biases,
                       uint16_t* y_bf16, int64_t M, int64_t N, int64_t K, int group_size, int bits,
                       int transpose, bq_stream_t stream);

/*
 * quant_matmul_noalloc -- quant_matmul for callers that must not allocate.
 * No page has a counterpart of this call; it exists for programs where the
 * library may not call cudaMalloc: hosts that own all device memory through
 * their own pool or that budget it once at start-up, and latency-critical
 * callers that cannot afford an allocation's implicit synchronization on a
 * first call.  It takes quant_matmul's own path, with a fixed 32 MiB array
 * that is part of the library's device image as its scratch: the decode GEMV
 * keeps its activation tables there (one or two tokens: 8 K + 64 K / group
 * bytes and a few more); the fused tensor-core kernel keeps its K-split partial sums there
 * (and runs without splitting K when they would not fit); the unfused pair
 * (q4_0_dequantize / affine_dequantize, then the bf16 tensor-core GEMM) stages
 * the bf16 copy of W there.  y is the same as quant_matmul's.
 *   Arguments, layouts, validation and errors are those of quant_matmul
 *   (both orientations).
 *   Limit: where the path is the unfused pair, N * K * 2 bytes must fit in
 *   BQ_NOALLOC_SCRATCH_BYTES (N * K at most 16,777,216 weights, e.g. 4096 x
 *   4096); larger problems there return BQ_ERR_WORKSPACE before anything is
 *   launched.
 *   Memory: every device that loads the library holds the 32 MiB array until
 *   the process exits.  The call itself makes no cudaMalloc / cudaFree and calls
 *   no allocating library routine.
 *   Set-up: every call looks up the array's device address on the current
 *   device (cudaGetSymbolAddress: no allocation), so the address is never
 *   stale, also after cudaDeviceReset.  The first call on a device also loads
 *   the library's device code there; make it before any stream capture.
 *   Sharing: all calls on a device use the same array and it keeps the last
 *   call's contents (each call overwrites the part it uses before reading it).
 *   Calls whose execution overlaps on the GPU -- on different streams without
 *   ordering between them -- race on the array; order them on one stream.
 */
#define BQ_NOALLOC_SCRATCH_BYTES (32u << 20)
BQ_API bq_status quant_matmul_noalloc(const uint16_t* x_bf16, const void* wq, const void* scales,
                                      const void* biases, uint16_t* y_bf16, int64_t M, int64_t N, int64_t K,
                                      int group_size, int bits, int transpose, bq_stream_t stream);

/*
 * quant_matmul_multi -- count (<= 8) quantized matmuls that share one
 * activation x: y[i] = quant_matmul(x, wq[i], scales[i], biases[i], N[i]) for
 * every i, all with the same M, K, format and group size.  After the SYCL
 * page "2026-05-06 Q4 sync-after focused repro" (Important source touch
 * points), which fuses adjacent Q4_0 matrix-vector products sharing one
 * token's activation (ffn_gate + ffn_up, Vcur + Kcur) into one kernel.
 *   wq, scales, y_bf16, N: host arrays of count device pointers / row counts
 *   biases: host array of count device pointers (affine), or NULL (Q4_0 for all)
 * At decode sizes (the dispatcher's GEMV path) all matrices run in one launch
 * and give the same bits as separate quant_matmul calls (with one or two
 * tokens their activation tables go in the stream's library buffer, as in
 * quant_matmul); at larger M each
 * matrix runs its own quant_matmul path.  Errors as quant_matmul; transpose
 * must be 1 and count > 8 returns BQ_ERR_UNSUPPORTED, count == 0 or M == 0
 * does nothing.
 */
BQ_API bq_status quant_matmul_multi(const uint16_t* x_bf16, int count, const void* const* wq,
                                    const void* const* scales, const void* const* biases, uint16_t* const* y_bf16,
                                    const int64_t* N, int64_t M, int64_t K, int group_size, int bits, int transpose,
                                    bq_stream_t stream);

/*
 * quant_matmul_ex -- quant_matmul with an explicit path (bq_path) and an
 * optional caller-owned device workspace.  With workspace == NULL the library's
 * per-device buffer is used as in quant_matmul.  Otherwise, for the unfused
 * pair workspace_bytes must be >= quant_matmul_workspace_size(...)
 * (BQ_ERR_WORKSPACE if not); the fused path given a smaller workspace runs
 * without K splits (same result within the tolerance, possibly slower); the
 * decode GEMV of one or two tokens given a smaller workspace runs the
 * register-streaming GEMV of three and more tokens instead (same tolerance).  Forcing
 * BQ_PATH_GEMV with M > 32, BQ_PATH_TC_FUSED
 * for 2-, 3- or 6-bit weights, BQ_PATH_TC_FUSED or BQ_PATH_GEMV_STREAM with
 * transpose = 0, or BQ_PATH_GEMV with transpose = 0 beyond 8 tokens or for 3-
 * or 6-bit codes, returns BQ_ERR_UNSUPPORTED.
 */
BQ_API bq_status quant_matmul_ex(const uint16_t* x_bf16, const void* wq, const void* scales, const void* biases,
                          uint16_t* y_bf16, int64_t M, int64_t N, int64_t K, int group_size, int bits,
                          int transpose, int path, void* workspace, size_t workspace_bytes,
                          bq_stream_t stream);

/* Bytes of workspace quant_matmul_ex needs for this problem and path
 * (path AUTO: the dispatcher's choice).  The pair: the bf16 copy of W (N x K x
 * 2).  The fused path: the fp32 partial sums of the tiles its plan splits over
 * K (splits x split tiles x tile tokens x 128 x 4; with more tiles than SMs,
 * only the tiles of the last, partly filled round are split), planned for the
 * current device, or for a B200 when there is none.  The decode GEMV with one
 * or two tokens: its activation tables, K / 32 x 256 bytes of byte slices of
 * x, K / group x 64 bytes of per-group scales and sums, and a flag word per
 * 2048 activations, rounded up to 16 bytes.  0 when the path needs none or
 * the arguments are invalid.  Having no biases pointer, this call and
 * quant_matmul_select_path take group_size 32 with bits 4 as Q4_0 and any
 * other combination as affine. */
BQ_API size_t quant_matmul_workspace_size(int64_t M, int64_t N, int64_t K, int group_size, int bits, int path);

/* Which decode kernel quant_matmul_ex runs for this problem on path (AUTO: the
 * dispatcher's choice) -- host only, for tools and benchmarks:
 *   0 the register-streaming GEMV (gemv_kernel), one launch;
 *   1 the streamed integer-MMA GEMV fed by the tensor-memory accelerator
 *     (gemv_tma_kernel), one launch, no workspace;
 *   2 the streamed integer-MMA GEMV fed by cp.async, after the kernel that builds
 *     its activation tables (gemv_int_prep_kernel, gemv_stream_kernel), two
 *     launches, the tables in workspace;
 *   3 the any-width affine GEMV (2-, 3- and 6-bit), one launch;
 *  -1 the path is not a decode path, or the arguments are invalid.
 * A caller workspace smaller than quant_matmul_workspace_size turns 2 into 0. */
BQ_API int quant_matmul_gemv_kernel(int64_t M, int64_t N, int64_t K, int group_size, int bits, int path);

/*
 * quant_matmul_select_path -- the M-threshold dispatcher (host only, no CUDA
 * call).  After the size threshold asked for on the MLX issue page (Question:
 * pick the dequantize path above some M) and the decode/prefill split of
 * "et-backend: Q4_0 matrix-engine GEMM rewrite for prefill" (Overview: decode
 * routes to the vector-dot kernel).  Returns a bq_path other than AUTO:
 * (transpose = 1; 2-, 3- and 6-bit affine weights get GEMV up to M = 8 and
 * DEQUANT_GEMM above):
 *   M <  tc_min_m                 -> BQ_PATH_GEMV        (tc_min_m by format, from the
 *                                    measured GEMV/fused crossovers on B200: 21 for
 *                                    Q4_0 and affine 4-bit, 17 for 8-bit; with
 *                                    K % 64 != 0 the GEMV up to M = 32)
 *   M >= pair_min_m               -> BQ_PATH_DEQUANT_GEMM (pair_min_m by format, from
 *                                    the measured fused/unfused crossovers on B200:
 *                                    4096 for Q4_0 and affine 4-bit, 2048 for 8-bit)
 *   otherwise                     -> BQ_PATH_TC_FUSED when K % 64 == 0,
 *                                    else BQ_PATH_DEQUANT_GEMM
 * Environment overrides, read once per process: BQ_TC_MIN_M (all formats,
 * clamped to [1, 33]; the GEMV handles at most 32 tokens) and BQ_PAIR_MIN_M
 * (all formats; 0: never).  Returns -1 for arguments quant_matmul would reject.
 */
BQ_API int quant_matmul_select_path(int64_t M, int64_t N, int64_t K, int group_size, int bits);

/*
 * bf16_matmul -- y[M][N] = bf16_rne(sum_k x[m][k] * w[n][k]), fp32
 * accumulation on the tcgen05 tensor cores: the plain bf16 matmul of the
 * unfused pair (MLX issue page, Repro: "x @ dense.T").
 *   x_bf16 device [M][K]; w_bf16 device [N][K]; y_bf16 device [M][N]; K % 8 == 0.
 */
BQ_API bq_status bf16_matmul(const uint16_t* x_bf16, const uint16_t* w_bf16, uint16_t* y_bf16,
                      int64_t M, int64_t N, int64_t K, bq_stream_t stream);

/*
 * q4_0_quantize -- fp32 w[N][K] -> Q4_0 (input preparation, mx.quantize's
 * counterpart).  Per block of 32: m = the element of largest |w| (first wins a
 * tie), d = m / -8 (fp32), stored as fp16; q = min(15, trunc(w * (1/d) + 8.5))
 * with 1/d taken as 0 when d == 0.
 *   w device f32 [N][K]; wq device u8 [N][K/2]; scales_f16 device u16 [N][K/32].
 */
BQ_API bq_status q4_0_quantize(const float* w, uint8_t* wq, uint16_t* scales_f16, int64_t N, int64_t K,
                        bq_stream_t stream);

/*
 * affine_quantize -- fp32 w[N][K] -> affine codes (mx.quantize on the MLX issue
 * page, Repro).  Per group: scale = bf16((max - min) / (2^bits - 1)),
 * bias = bf16(min), q = clamp(round_half_even((w - bias) / scale), 0, 2^bits - 1)
 * from the stored bf16 scale and bias (q = 0 when scale == 0).
 *   w device f32 [N][K]; wq device u32 [N][K*bits/32] (the bit-stream layout
 *   above); scales/biases device bf16 [N][K/group_size]; bits 2, 3, 4, 6 or 8.
 */
BQ_API bq_status affine_quantize(const float* w, uint32_t* wq, uint16_t* scales_bf16, uint16_t* biases_bf16,
                          int64_t N, int64_t K, int group_size, int bits, bq_stream_t stream);

/*
 * bq_selftest_wait_timeout -- exercises the failure detection of the device-side
 * bounded waits (no page has a counterpart; it tests this library's own
 * mechanism).  Launches one thread that waits on an mbarrier nothing will ever
 * complete, with the kernels' try_wait, and gives up after limit_cycles SM
 * clocks (1000 .. 4e9), recording the timeout in the device error word exactly
 * as a kernel's timed-out wait does.  bq_device_status() then returns
 * BQ_ERR_TIMEOUT (and clears it); the context stays usable.  No fault, no trap.
 */
BQ_API bq_status bq_selftest_wait_timeout(long long limit_cycles, bq_stream_t stream);

/*
 * bq_device_status -- waits for the current device to finish its work, then
 * reads and clears the library's device error word: BQ_OK, or BQ_ERR_TIMEOUT
 * when a kernel's bounded wait on a shared-memory barrier ran out (the kernel
 * then skipped its remaining work and exited cleanly; its output is not valid).
 * BQ_ERR_CUDA if the device cannot be queried.
 */
BQ_API bq_status bq_device_status(void);

/* Human-readable name of a status code (static storage, never NULL). */
BQ_API const char* bq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
BQ_API int bq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BQGEMM_H */
