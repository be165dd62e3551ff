// gemv_stream.cuh -- decode path for one or two tokens.  The packed weights
// stream once from HBM through per-warp shared-memory rings (16-byte
// asynchronous copies) into integer tensor-core MMAs that multiply the codes,
// as unsigned bytes, with the activations split into signed bytes: every inner
// sum is an exact integer, and each block's (or group's) scale is applied once.
//
// The pages' decode kernels are prior art for this path: decode routes to a
// vector-dot kernel in "et-backend: Q4_0 matrix-engine GEMM rewrite for
// prefill" (Overview), and the SYCL page "2026-05-06 Q4 sync-after focused
// repro" runs MMVQ kernels, which take the activations as 8-bit integers, over
// "reordered" Q4_0 (Important source touch points).  Here the integer form of
// x is exact, not a quantization.  The operation is the MLX issue's
// quantized_matmul ("Repro"): y = x . dequant(W)^T, which is
//
//   y[m][n] = sum over blocks b of  d[n][b] * sum_{j in b} x[m][j] * (q[n][j] - 8)      (Q4_0)
//   y[m][n] = sum over groups g of  s[n][g] * sum_{j in g} x[m][j] * q[n][j]
//                                 + z[n][g] * sum_{j in g} x[m][j]                  (affine)
//
// computed in that order; the result differs from a product with the
// bf16-rounded dequantized weights only by those weights' roundings.
//
// Activations.  With one or two tokens most of an n8 MMA's columns would carry
// nothing; they hold the tokens' activations split into signed bytes instead.
// With S = 8 slices for one token, 4 for each of two:
//
//   per token and scale group, e = the exponent of the group's largest |x|, P = 8 S - 3;
//   v_k = x_k * 2^(P - e), an integer whenever x_k's exponent is >= e - (P - 7);
//   v_k = sum_j 2^(8 j) l_j,k, l_j in [-128, 127] below the top slice, |l_top| <= 64;
//   the MMA column of slice j holds l_j, and its sum is scaled by 2^(e - P + 8 j).
//
// So every bf16 activation within 2^54 (one token) or 2^22 (two tokens) of its
// group's largest is held exactly.  A launch whose activations are not all held
// exactly computes plain fp32 dot products instead (gemv_exact): the integer
// route never rounds x.  Q4_0's -8 enters as the MMA addend -8 * sum_k l_j,k
// (an exact integer), the affine bias as z * sum_g x (the fp32 sum of the bf16
// activations).  A group holding Inf or NaN gives NaN.
//
// Codes.  An m16n8k32 step covers 32 elements of 16 rows: a Q4_0 block or an
// affine-4 code unit (one 16-byte unit per row), or two affine-8 units, so the
// codes reach the MMA with no arithmetic at all (affine 8-bit) or one AND and
// one shift-AND per word (the two nibbles of each byte become separate bytes).
// The k-slot order this gives is folded into the activation table:
//   Q4_0, affine 8-bit: lane t's bytes are elements 4t..4t+3 (register 0) and 16+4t..16+4t+3 (register 1)
//   affine 4-bit:       register 0 holds elements 8t, 8t+2, 8t+4, 8t+6 and register 1 elements 8t+1, +3, +5, +7
//
// Work.  gemv_int_prep_kernel builds the activation tables once per call, in a
// device buffer; gemv_stream_kernel runs one CTA per SM over a contiguous range
// of 16-row weight tiles (of one matrix, or of up to eight matrices that share
// x, as the fused one-token MMVQ nodes on the SYCL page; a tile is computed
// the same way whichever launch it is in, so the bits do not depend on it).
// Each of its KW warps owns a fixed K slice of every tile and streams exactly
// that slice (codes and scales of its 16 rows) into its own ring of S stages
// with cp.async, so no warp waits for another; its part of the activation
// tables travels with its first stage.  Rows are padded by 16 bytes so that
// ldmatrix reads them without bank conflicts; ldmatrix hands each thread the
// 4-byte word of a 16-byte code unit that its MMA fragment needs.  Per-warp
// partial sums of each tile are summed in warp order at the end, so the
// result is deterministic.
//
// Launch: both kernels use programmatic stream serialization.  The prep kernel
// reads x after its griddepcontrol.wait and lets the GEMV launch only then; the
// cp.async GEMV reads everything after its own wait, the TMA-fed one streams W
// before it (see there) and reads x's tables and writes y after it.
#pragma once

#include "gemv.cuh"
#include "tcgen05.cuh"

namespace bq {

// ------------------------------------------------------------------ PTX wrappers
BQ_DEVINL void cp_async16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
BQ_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
BQ_DEVINL void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

BQ_DEVINL void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
BQ_DEVINL void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Not volatile: the compiler may move it among arithmetic and MMAs (the memory
// clobber keeps it after the cp.async wait that makes its data visible).
BQ_DEVINL void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}

// D = A x B + C, m16n8k32, A unsigned bytes, B signed bytes, s32 accumulate: exact.
BQ_DEVINL void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                              uint32_t b1, int c0, int c1, int c2, int c3)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1), "r"(c2), "r"(c3));
}

BQ_DEVINL uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
BQ_DEVINL uint32_t lds16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

// A lane's walk over the 16-byte units of a [rows][n] block, 32 units apart:
// its first unit (r, c) and the step (dr, dc) -- one division when the block
// width changes instead of one per copied unit.
struct LaneWalk {
    int n, r, c, dr, dc;
    BQ_DEVINL void init(int width, int lane)
    {
        n = width;
        r = width > 0 ? lane / width : 0;
        c = lane - r * width;
        dr = width > 0 ? 32 / width : 0;
        dc = 32 - dr * width;
    }
};

// cp.async of a [rows][w.n] block of 16-byte units: source rows `spitch` bytes
// apart, destination rows `dpitch` bytes apart.
BQ_DEVINL void copy_block(uint32_t dst, uint32_t dpitch, const uint8_t* src, int64_t spitch, int rows,
                          const LaneWalk& w)
{
    if (w.n <= 0) return;
    int r = w.r, c = w.c;
    while (r < rows) {
        cp_async16(dst + (uint32_t)r * dpitch + (uint32_t)c * 16u, src + r * spitch + c * 16);
        r += w.dr;
        c += w.dc;
        if (c >= w.n) {
            c -= w.n;
            ++r;
        }
    }
}

// ------------------------------------------------------------------ formats
// A 16-byte code unit of one row holds E elements.
template <Fmt F> struct SFmt;
template <> struct SFmt<Fmt::Q4_0> { static constexpr int E = 32, kBits = 4; };
template <> struct SFmt<Fmt::AFF4> { static constexpr int E = 32, kBits = 4; };
template <> struct SFmt<Fmt::AFF8> { static constexpr int E = 16, kBits = 8; };

// ------------------------------------------------------------------ parameters
constexpr int kSgIntTokens = 2;                // 8 slices of one token, or 4 of each of two: one n8 MMA
constexpr int kSgMaxMats = 8;                  // matrices sharing x in one launch
constexpr int kSgIntCtabBytes = 64;            // group table: 4 quad positions x (c0, c1, X0, X1)
constexpr uint32_t kSgIntStepBytes = 256;      // slice table per 32-element step: 8 columns x 4 x 8 bytes
constexpr int kSgPrepThreads = 256;
constexpr int kSgWarpsTma = 8;                 // compute warps of the TMA-fed kernel (plus one producer)
constexpr int kSgMaxStagesTma = 4;

struct SGemvParams {
    const uint16_t* x;                   // bf16 [M][K], shared by every matrix
    int count;                           // matrices (1 .. kSgMaxMats)
    int tile_begin[kSgMaxMats + 1];      // matrix i owns global tiles [tile_begin[i], tile_begin[i+1])
    const uint8_t* wq[kSgMaxMats];       // packed codes, N[i] rows of K * bits / 8 bytes
    const uint16_t* scales[kSgMaxMats];  // [N][K / group] (fp16 for Q4_0, bf16 for affine)
    const uint16_t* biases[kSgMaxMats];  // bf16 [N][K / group] (affine)
    uint16_t* y[kSgMaxMats];             // bf16 [M][N]
    int N[kSgMaxMats];
    int M, K;
    int kc;                   // K elements per chunk (multiple of 8 x group size)
    int nchunks;              // ceil(K / kc)
    int ntiles;               // sum over matrices of ceil(N / 16)
    int stages;               // ring depth per warp (2 .. 4)
    uint32_t code_pitch;      // shared bytes per code row of a warp's stage (slice bytes + padding)
    uint32_t scale_pitch;     // shared bytes per scale (or bias) row of a warp's stage
    uint32_t wstage_bytes;    // one stage of one warp
    int red_cols;             // token columns of the partial-sum buffer
    uint32_t off_x, off_c, off_red, off_ring;   // offsets into dynamic shared memory
    uint8_t* tab;             // activation tables built by gemv_int_prep_kernel: slices at 0,
    uint32_t tab_c_off;       //   the group table at tab_c_off,
    uint32_t tab_f_off;       //   one inexactness flag word per prep CTA at tab_f_off
    int nflags;
};

// fp32 bits of 2^n: normal, subnormal (n >= -149) or zero.
BQ_DEVINL uint32_t pow2_bits(int n)
{
    return n >= -126 ? (uint32_t)(n + 127) << 23 : n >= -149 ? 1u << (n + 149) : 0u;
}

// MMA column of slice j of token m (slices per token: 8 for one token, 4 for two).
BQ_DEVINL int int_column(int M, int m, int j) { return M == 1 ? j : 4 * m + j; }

// ------------------------------------------------------------------ activation tables
// One item (token m, 32-element step, quad position t) per thread: its eight
// activations, their slices in the two B registers of column (m, j) for every
// slice j, and -- by the first lane of each group -- the group's column scales
// and addends.  Tables (in `tab`): slices [K / 32 steps][8 columns][4 quad
// positions] x (register 0, register 1); groups [K / group][4 quad positions] x
// (scale of column 2t, of column 2t + 1, Q4_0 addend or affine bias sum of
// column 2t, of 2t + 1); then one flag word per CTA, nonzero when one of its
// activations is not held exactly.
//
// Integer arithmetic on the bf16 bits: |x| = m 2^(E' - 134) with m = 128 + f
// (E' = E) for normal values, m = f (E' = 1) for subnormal ones, so v = m 2^sh
// with sh = E' - 134 - (e - P).  m << (sh mod 8) spans at most two bytes; its
// signed-digit form (three digits, the last one 0 or +-1) lands at slice
// sh / 8, and a byte transpose (prmt) gathers each slice's four bytes per MMA
// register.  The top slice absorbs the carry, which keeps it within +-64.
// One item of the activation tables (token m, 32-element step, quad position
// t) by one lane of a warp whose lanes all take part (a lane with valid ==
// false computes on clamped data and stores nothing): the slices of its eight
// activations into `xt` (the slice table), and -- by the first lane of each
// group -- the group's column scales and addends into `ct` (the group table).
// A group's lanes must be consecutive lanes of the warp, aligned to 4 SPG.
// Returns nonzero when one of its activations is not held exactly.
// The item's eight activations as bf16 pairs in the order of the two MMA B
// registers: element i is half (i & 1) of word i >> 1.
template <Fmt F>
BQ_DEVINL void int_item_load(const uint16_t* __restrict__ x, int K, int m, int step, int t, uint32_t (&raw)[4])
{
    const uint16_t* xr = x + (int64_t)m * K + (int64_t)step * 32;
    if constexpr (F == Fmt::AFF4) {
        // register 0 <- elements 8t + 2i (low halves), register 1 <- 8t + 2i + 1 (high halves)
        const uint4 q = *reinterpret_cast<const uint4*>(xr + 8 * t);
        raw[0] = __byte_perm(q.x, q.y, 0x5410);
        raw[1] = __byte_perm(q.z, q.w, 0x5410);
        raw[2] = __byte_perm(q.x, q.y, 0x7632);
        raw[3] = __byte_perm(q.z, q.w, 0x7632);
    } else {
        const uint2 a = *reinterpret_cast<const uint2*>(xr + 4 * t);
        const uint2 c = *reinterpret_cast<const uint2*>(xr + 16 + 4 * t);
        raw[0] = a.x;
        raw[1] = a.y;
        raw[2] = c.x;
        raw[3] = c.y;
    }
}

template <Fmt F, int GS>
BQ_DEVINL int int_table_item_raw(const uint32_t (&raw)[4], int M, int m, int step, int t, int lane, bool valid,
                                 uint8_t* xt, uint8_t* ct)
{
    constexpr int SPG = GS / 32;                        // MMA steps per group
    constexpr int GL = 4 * SPG;                         // lanes that hold one group
    static_assert(GL <= 32, "a group's lanes lie in one warp");
    const int S = M == 1 ? 8 : 4, P = 8 * S - 3;
    int inexact = 0;
    {
        uint32_t key[8];
        uint32_t kmax = 0u;
        int bad = 0;
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t bits = (raw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
            key[i] = bits;
            bad |= (bits & 0x7FFFu) >= 0x7F80u;
            kmax = max(kmax, bits & 0x7FFFu);
            if constexpr (F != Fmt::Q4_0) sum += bf16_bits_to_f32(bits);
        }
#pragma unroll
        for (int o = 1; o < GL; o <<= 1) {
            kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
            bad |= __shfl_xor_sync(0xFFFFFFFFu, bad, o);
            if constexpr (F != Fmt::Q4_0) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        }
        // e = exponent of the group's largest |x| (0 for an all-zero or non-finite group)
        const int emax = (int)(kmax >> 7);
        const int e = (bad || kmax == 0u) ? 0 : emax > 0 ? emax - 127 : (31 - __clz((int)kmax)) - 133;
        const int lsb = e - P;                          // exponent of v's unit
        uint32_t lo[8], hi[8];                          // slices 0-3 and 4-7 of each element's v
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t bits = key[i];
            const int E = (int)((bits >> 7) & 0xFFu);
            const int mant = E ? (int)((bits & 0x7Fu) | 0x80u) : (int)(bits & 0x7Fu);
            const int sh = (E ? E : 1) - 134 - lsb;
            int W, j0;
            if (sh >= 0) {
                W = mant << (sh & 7);
                j0 = sh >> 3;
            } else {
                const int rs = -sh;
                W = rs >= 8 ? 0 : mant >> rs;
                inexact |= valid && (rs >= 8 ? mant : mant - (W << rs)) != 0;
                j0 = 0;
            }
            if (bad) {
                W = 0;
                j0 = 0;
            }
            if (bits & 0x8000u) W = -W;
            const int d0 = (W << 24) >> 24;
            const int W1 = (W - d0) >> 8;
            int d1 = (W1 << 24) >> 24, d2 = (W1 - d1) >> 8;
            if (j0 + 2 >= S) {                          // top slice: keep the whole rest
                d1 = W1;
                d2 = 0;
            }
            const uint32_t D = ((uint32_t)d0 & 0xFFu) | (((uint32_t)d1 & 0xFFu) << 8) | (((uint32_t)d2 & 0xFFu) << 16);
            const uint64_t T = (uint64_t)D << (8 * j0);
            lo[i] = (uint32_t)T;
            hi[i] = (uint32_t)(T >> 32);
        }
        // transpose: slice j of register r holds byte j of elements 4r .. 4r + 3
        uint32_t r0[8], r1[8];
        auto transpose4 = [](const uint32_t* a, uint32_t* out) {
            const uint32_t t01l = __byte_perm(a[0], a[1], 0x5140), t01h = __byte_perm(a[0], a[1], 0x7362);
            const uint32_t t23l = __byte_perm(a[2], a[3], 0x5140), t23h = __byte_perm(a[2], a[3], 0x7362);
            out[0] = __byte_perm(t01l, t23l, 0x5410);
            out[1] = __byte_perm(t01l, t23l, 0x7632);
            out[2] = __byte_perm(t01h, t23h, 0x5410);
            out[3] = __byte_perm(t01h, t23h, 0x7632);
        };
        transpose4(lo, r0);
        transpose4(lo + 4, r1);
        transpose4(hi, r0 + 4);
        transpose4(hi + 4, r1 + 4);
        int L[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (j < S) {
                if (valid)
                    *reinterpret_cast<uint2*>(xt + (size_t)step * kSgIntStepBytes +
                                              (size_t)(int_column(M, m, j) * 4 + t) * 8u) = make_uint2(r0[j], r1[j]);
                L[j] = __dp4a((int)r0[j], 0x01010101, __dp4a((int)r1[j], 0x01010101, 0));
#pragma unroll
                for (int o = 1; o < GL; o <<= 1) L[j] += __shfl_xor_sync(0xFFFFFFFFu, L[j], o);
            }
        }
        if (valid && (lane & (GL - 1)) == 0) {
            uint8_t* cg = ct + (size_t)(step / SPG) * kSgIntCtabBytes;
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                if (j < S) {
                    uint32_t c[2], X[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        c[h] = bad ? 0x7FC00000u : pow2_bits(lsb + 8 * (j + h));
                        if constexpr (F == Fmt::Q4_0) X[h] = (uint32_t)(-8 * L[j + h]);
                        else X[h] = j + h == 0 ? __float_as_uint(sum) : 0u;
                    }
                    *reinterpret_cast<uint4*>(cg + (int_column(M, m, j) / 2) * 16) = make_uint4(c[0], c[1], X[0], X[1]);
                }
            }
        }
    }
    return inexact;
}

template <Fmt F, int GS>
BQ_DEVINL int int_table_item(const uint16_t* __restrict__ x, int M, int K, int m, int step, int t, int lane,
                             bool valid, uint8_t* xt, uint8_t* ct)
{
    uint32_t raw[4];
    int_item_load<F>(x, K, m, step, t, raw);
    return int_table_item_raw<F, GS>(raw, M, m, step, t, lane, valid, xt, ct);
}

template <Fmt F, int GS>
__global__ void __launch_bounds__(kSgPrepThreads)
gemv_int_prep_kernel(const uint16_t* __restrict__ x, int M, int K, uint8_t* __restrict__ tab, uint32_t c_off,
                     uint32_t f_off)
{
    grid_dependency_wait();                             // x comes from the previous kernel
    // Only now may the GEMV launch: every kernel before this one has completed
    // and its writes are visible.
    grid_dependents_launch();
    const int tid = threadIdx.x, lane = tid & 31;
    const int nsteps = K / 32;
    const int items = M * nsteps * 4;                   // a multiple of 32 (K is a multiple of 256)
    const int idx = blockIdx.x * kSgPrepThreads + tid;
    int inexact = 0;
    if (idx - lane < items)                             // whole warps
        inexact = int_table_item<F, GS>(x, M, K, (idx >> 2) / nsteps, (idx >> 2) % nsteps, idx & 3, lane, true, tab,
                                        tab + c_off);
    inexact = __syncthreads_or(inexact);
    if (tid == 0) reinterpret_cast<uint32_t*>(tab + f_off)[blockIdx.x] = inexact ? 1u : 0u;
}

// Exact fallback of the streamed GEMV for the CTA's tiles: fp32 dot products of
// x with the weights dequantized in fp32 (d (q - 8) exactly, s q + z rounded
// once), read straight from global memory; one warp per row, deterministic.
template <Fmt F, int GS>
BQ_DEVINL void gemv_exact(const SGemvParams& p, int t_begin, int t_end, int warp, int lane, int nwarps)
{
    const int M = p.M, K = p.K;
    const int64_t row_bytes = (int64_t)K * SFmt<F>::kBits / 8, srow = K / GS;
    for (int rl = warp; rl < (t_end - t_begin) * 16; rl += nwarps) {
        const int tile = t_begin + (rl >> 4);
        int mat = 0;
        while (mat + 1 < p.count && tile >= p.tile_begin[mat + 1]) ++mat;
        const int64_t row = (int64_t)(tile - p.tile_begin[mat]) * 16 + (rl & 15);
        if (row >= p.N[mat]) continue;
        const uint8_t* wr = p.wq[mat] + row * row_bytes;
        const uint16_t* sr = p.scales[mat] + row * srow;
        const uint16_t* br = F == Fmt::Q4_0 ? nullptr : p.biases[mat] + row * srow;
        for (int m = 0; m < M; ++m) {
            const uint16_t* xr = p.x + (int64_t)m * K;
            float acc = 0.0f;
            for (int k = lane; k < K; k += 32) {
                float w;
                if constexpr (F == Fmt::Q4_0) {
                    const int j = k & 31;
                    const uint32_t byte = wr[(k >> 5) * 16 + (j & 15)];
                    const int q = (int)(j < 16 ? byte & 15u : byte >> 4);
                    w = __half2float(__ushort_as_half(sr[k >> 5])) * (float)(q - 8);
                } else {
                    const uint32_t q = F == Fmt::AFF8 ? (uint32_t)wr[k] : (uint32_t)(wr[k >> 1] >> (4 * (k & 1))) & 15u;
                    w = __fmaf_rn(bf16_bits_to_f32(sr[k / GS]), (float)q, bf16_bits_to_f32(br[k / GS]));
                }
                acc = __fmaf_rn(bf16_bits_to_f32(xr[k]), w, acc);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
            if (lane == 0) p.y[mat][(int64_t)m * p.N[mat] + row] = (uint16_t)f32_to_bf16_bits(acc);
        }
    }
}

// Scale (or bias) of row r's group `a` of the stage, as fp32: fp16 for Q4_0, bf16 for affine.
template <Fmt F>
BQ_DEVINL float stage_scale(const uint8_t* p)
{
    if constexpr (F == Fmt::Q4_0) return __half2float(*reinterpret_cast<const __half*>(p));
    else return bf16_bits_to_f32(lds16(p));
}


// One warp's K slice of one stage, integer route: xp is this lane's slice-table
// entry of the slice's first step, cp its group-table
// entry of the slice's first group; sc as in slice_mma.
template <Fmt F, int GS, int NU, typename LdAddr, typename ScAddr>
BQ_DEVINL void slice_int(float (&yv)[4], LdAddr ld, ScAddr sa, const uint8_t* xp, const uint8_t* cp, int nu_rt)
{
    using T = SFmt<F>;
    constexpr int UPG = GS / T::E;                      // code units per group
    constexpr uint32_t kLo = 0x0F0F0F0Fu;
    constexpr bool kAffine = F != Fmt::Q4_0;
    const int nu = NU > 0 ? NU : nu_rt;
    if constexpr (T::E == 32 && UPG == 1) {
        // one group per unit (Q4_0, affine-4 with groups of 32): two per ldmatrix.x4
#pragma unroll (NU > 0 ? NU / 2 : 2)
        for (int s = 0; s < nu / 2; ++s) {
            uint32_t w[4];                                      // (g, u) (g+8, u) (g, u+1) (g+8, u+1)
            ldsm_x4(ld(2 * s), w[0], w[1], w[2], w[3]);
            const uint32_t sg = lds32(sa(0, 0, 2 * s)), sg8 = lds32(sa(1, 0, 2 * s));   // groups u, u + 1, rows g, g + 8
            [[maybe_unused]] uint32_t bg = 0u, bg8 = 0u;
            if constexpr (kAffine) {
                bg = lds32(sa(0, 1, 2 * s));
                bg8 = lds32(sa(1, 1, 2 * s));
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int u = 2 * s + h;
                const uint32_t wg = w[2 * h], wg8 = w[2 * h + 1];
                const uint2 b = *reinterpret_cast<const uint2*>(xp + (uint32_t)u * kSgIntStepBytes);
                const uint4 ce = *reinterpret_cast<const uint4*>(cp + u * kSgIntCtabBytes);
                const int c0 = kAffine ? 0 : (int)ce.z, c1 = kAffine ? 0 : (int)ce.w;
                int acc[4];
                mma_u8s8_16832(acc, wg & kLo, wg8 & kLo, (wg >> 4) & kLo, (wg8 >> 4) & kLo, b.x, b.y, c0, c1, c0, c1);
                float dg, dg8;
                if constexpr (kAffine) {
                    dg = __uint_as_float(h ? sg & 0xFFFF0000u : sg << 16);
                    dg8 = __uint_as_float(h ? sg8 & 0xFFFF0000u : sg8 << 16);
                } else {
                    const float2 d2 = __half22float2(*reinterpret_cast<const __half2*>(&sg));
                    const float2 d28 = __half22float2(*reinterpret_cast<const __half2*>(&sg8));
                    dg = h ? d2.y : d2.x;
                    dg8 = h ? d28.y : d28.x;
                }
                const float k0 = __uint_as_float(ce.x), k1 = __uint_as_float(ce.y);
                if constexpr (kAffine) {
                    const float zg = __uint_as_float(h ? bg & 0xFFFF0000u : bg << 16);
                    const float zg8 = __uint_as_float(h ? bg8 & 0xFFFF0000u : bg8 << 16);
                    const float b0 = __uint_as_float(ce.z), b1 = __uint_as_float(ce.w);
                    yv[0] = __fmaf_rn(zg, b0, yv[0]);
                    yv[1] = __fmaf_rn(zg, b1, yv[1]);
                    yv[2] = __fmaf_rn(zg8, b0, yv[2]);
                    yv[3] = __fmaf_rn(zg8, b1, yv[3]);
                }
                yv[0] = __fmaf_rn(dg * k0, (float)acc[0], yv[0]);
                yv[1] = __fmaf_rn(dg * k1, (float)acc[1], yv[1]);
                yv[2] = __fmaf_rn(dg8 * k0, (float)acc[2], yv[2]);
                yv[3] = __fmaf_rn(dg8 * k1, (float)acc[3], yv[3]);
            }
        }
    } else {
        // groups of two or more units, every MMA of a group into one accumulator
#pragma unroll (NU > 0 ? NU / UPG : 1)
        for (int a = 0; a < nu / UPG; ++a) {
            int acc[4] = {0, 0, 0, 0};
#pragma unroll
            for (int s = 0; s < UPG / 2; ++s) {
                const int u = a * UPG + 2 * s;
                uint32_t w[4];
                ldsm_x4(ld(u), w[0], w[1], w[2], w[3]);
                if constexpr (F == Fmt::AFF8) {
                    const uint2 b = *reinterpret_cast<const uint2*>(xp + (uint32_t)(u / 2) * kSgIntStepBytes);
                    mma_u8s8_16832(acc, w[0], w[1], w[2], w[3], b.x, b.y, acc[0], acc[1], acc[2], acc[3]);
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t wg = w[2 * h], wg8 = w[2 * h + 1];
                        const uint2 b = *reinterpret_cast<const uint2*>(xp + (uint32_t)(u + h) * kSgIntStepBytes);
                        mma_u8s8_16832(acc, wg & kLo, wg8 & kLo, (wg >> 4) & kLo, (wg8 >> 4) & kLo, b.x, b.y, acc[0],
                                       acc[1], acc[2], acc[3]);
                    }
                }
            }
            const uint4 ce = *reinterpret_cast<const uint4*>(cp + a * kSgIntCtabBytes);
            const float dg = stage_scale<F>(sa(0, 0, a)), dg8 = stage_scale<F>(sa(1, 0, a));
            const float zg = stage_scale<F>(sa(0, 1, a)), zg8 = stage_scale<F>(sa(1, 1, a));
            const float k0 = __uint_as_float(ce.x), k1 = __uint_as_float(ce.y);
            const float b0 = __uint_as_float(ce.z), b1 = __uint_as_float(ce.w);
            yv[0] = __fmaf_rn(dg * k0, (float)acc[0], __fmaf_rn(zg, b0, yv[0]));
            yv[1] = __fmaf_rn(dg * k1, (float)acc[1], __fmaf_rn(zg, b1, yv[1]));
            yv[2] = __fmaf_rn(dg8 * k0, (float)acc[2], __fmaf_rn(zg8, b0, yv[2]));
            yv[3] = __fmaf_rn(dg8 * k1, (float)acc[3], __fmaf_rn(zg8, b1, yv[3]));
        }
    }
}

// ------------------------------------------------------------------ kernel
// SU: code units of every warp's slice of a full chunk when they are all equal
// and known at compile time (the inner loop is then fully unrolled), else 0.
template <Fmt F, int GS, int KW, int SU>
__global__ void __launch_bounds__(32 * KW, 1)
gemv_stream_kernel(const __grid_constant__ SGemvParams p)
{
    using T = SFmt<F>;
    constexpr int E = T::E;
    constexpr int UPG = GS / E;                          // code units per scale group
    constexpr bool kAffine = F != Fmt::Q4_0;
    constexpr int kAtomUnits = UPG > 2 ? UPG : 2;        // K-split atom: 2 units (one ldmatrix.x4), whole groups
    static_assert(GS % E == 0, "group must hold whole code units");

    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    const int M = p.M, K = p.K, S = p.stages, nchunks = p.nchunks;
    const int t_begin = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
    const int t_end = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
    const int nt = t_end - t_begin;
    const int total = nt * nchunks;
    const int64_t row_bytes = (int64_t)K * T::kBits / 8;
    const int64_t srow = K / GS;                         // scale entries per row
    const uint32_t ring = sbase + p.off_ring + (uint32_t)warp * S * p.wstage_bytes;

    // This warp's slice of a chunk of kn elements (atoms [a_b, a_e)), with the
    // lane walks of its copies: the code units of its 16 rows, and the
    // 16-byte-aligned run of scale (and bias) bytes that covers its groups,
    // starting sb bytes into the chunk's scales.
    struct Slice {
        int a_b, nu, sb;
        LaneWalk wc, ws;
    };
    auto make_slice = [&](int kn, Slice& sl) {
        const int natoms = kn / E / kAtomUnits;
        const int a_b = warp * natoms / KW, a_e = (warp + 1) * natoms / KW;
        sl.a_b = a_b;
        sl.nu = (a_e - a_b) * kAtomUnits;
        sl.wc.init(sl.nu, lane);
        const int g_b = a_b * kAtomUnits / UPG, g_e = a_e * kAtomUnits / UPG;   // groups within the chunk
        sl.sb = (2 * g_b) & ~15;
        sl.ws.init((2 * g_e - sl.sb + 15) / 16, lane);
    };
    Slice sl_full, sl_last;
    const int kn_last = K - (nchunks - 1) * p.kc;
    make_slice(nchunks > 1 ? p.kc : K, sl_full);
    make_slice(kn_last, sl_last);

    // Copy cursor: the (tile, chunk) of the next stage to fill, and its matrix.
    int c_tile = t_begin, c_chunk = 0, c_mat = 0;
    while (c_mat + 1 < p.count && c_tile >= p.tile_begin[c_mat + 1]) ++c_mat;
    auto issue_next = [&](int i) {
        if (i < total) {
            const int64_t row0 = (int64_t)(c_tile - p.tile_begin[c_mat]) * 16;
            const int64_t left = (int64_t)p.N[c_mat] - row0;
            const int rows = left < 16 ? (int)left : 16;
            const int k0 = c_chunk * p.kc;
            const Slice& sl = c_chunk == nchunks - 1 ? sl_last : sl_full;
            const uint32_t st = ring + (uint32_t)(i % S) * p.wstage_bytes;
            copy_block(st, p.code_pitch,
                       p.wq[c_mat] + row0 * row_bytes + (int64_t)k0 * T::kBits / 8 + (int64_t)sl.a_b * kAtomUnits * 16,
                       row_bytes, rows, sl.wc);
            const int64_t sbyte = 2 * (int64_t)(k0 / GS) + sl.sb;
            const uint32_t sdst = st + 16u * p.code_pitch;
            copy_block(sdst, p.scale_pitch, reinterpret_cast<const uint8_t*>(p.scales[c_mat] + row0 * srow) + sbyte,
                       srow * 2, rows, sl.ws);
            if constexpr (kAffine)
                copy_block(sdst + 16u * p.scale_pitch, p.scale_pitch,
                           reinterpret_cast<const uint8_t*>(p.biases[c_mat] + row0 * srow) + sbyte, srow * 2, rows,
                           sl.ws);
            if (++c_chunk == nchunks) {
                c_chunk = 0;
                ++c_tile;
                while (c_mat + 1 < p.count && c_tile >= p.tile_begin[c_mat + 1]) ++c_mat;
            }
        }
        cp_async_commit();
    };

    grid_dependency_wait();
    grid_dependents_launch();

    // A launch whose activations the slices do not hold exactly computes fp32
    // dot products (every warp reads the same flags, so the choice is uniform).
    {
        const uint32_t* flags = reinterpret_cast<const uint32_t*>(p.tab + p.tab_f_off);
        uint32_t inexact = 0u;
        for (int i = lane; i < p.nflags; i += 32) inexact |= flags[i];
        if (__any_sync(0xFFFFFFFFu, inexact != 0u)) {
            gemv_exact<F, GS>(p, t_begin, t_end, warp, lane, KW);
            return;
        }
    }
    // This warp's part of the activation tables -- the steps and groups of its
    // slice in every chunk -- travels in the commit group of its first stage.
    for (int c = 0; c < nchunks; ++c) {
        const Slice& sl = c == nchunks - 1 ? sl_last : sl_full;
        const int u0 = c * (p.kc / E) + sl.a_b * kAtomUnits;        // the slice's first unit in the row
        const uint32_t xo = (uint32_t)(u0 * E / 32) * kSgIntStepBytes;
        const uint32_t xn = (uint32_t)(sl.nu * E / 32) * kSgIntStepBytes;
        const uint32_t co = (uint32_t)(u0 / UPG) * kSgIntCtabBytes;
        const uint32_t cn = (uint32_t)(sl.nu / UPG) * kSgIntCtabBytes;
        for (uint32_t o = (uint32_t)lane * 16u; o < xn; o += 512u) cp_async16(sbase + p.off_x + xo + o, p.tab + xo + o);
        for (uint32_t o = (uint32_t)lane * 16u; o < cn; o += 512u)
            cp_async16(sbase + p.off_c + co + o, p.tab + p.tab_c_off + co + o);
    }
    for (int i = 0; i < S - 1; ++i) issue_next(i);

    // ------------------------------------------------------------ main loop
    const int g = lane >> 2, t = lane & 3;
    const uint8_t* x_lane = smem + p.off_x + (size_t)((g * 4 + t) * 8);     // slice column g
    const uint8_t* c_lane = smem + p.off_c + (size_t)t * 16;
    // ldmatrix.x4 row addresses: matrices (rows 0-7, unit u), (rows 8-15, unit u),
    // (rows 0-7, unit u+1), (rows 8-15, unit u+1)
    const uint32_t ld_lane =
        (uint32_t)((lane & 7) + ((lane >> 3) & 1) * 8) * p.code_pitch + (uint32_t)(lane >> 4) * 16u;
    float* red = reinterpret_cast<float*>(smem + p.off_red);
    float yv[4] = {0.0f, 0.0f, 0.0f, 0.0f};

    int tl = 0, chunk = 0;
    for (int i = 0; i < total; ++i) {
        issue_next(i + S - 1);
        if (S == 4) cp_async_wait<3>();
        else if (S == 3) cp_async_wait<2>();
        else cp_async_wait<1>();
        __syncwarp();
        if (chunk == 0) yv[0] = yv[1] = yv[2] = yv[3] = 0.0f;
        const bool last = chunk == nchunks - 1;
        const Slice& sl = last ? sl_last : sl_full;
        const int k0 = chunk * p.kc;
        const uint32_t st = ring + (uint32_t)(i % S) * p.wstage_bytes;
        const int u_b = k0 / E + sl.a_b * kAtomUnits;           // first unit of the slice (in the row)
        const int g_b = u_b / UPG;                              // its first group
        const uint8_t* sc = smem + (st - sbase) + 16u * p.code_pitch + (size_t)g * p.scale_pitch +
                            ((2 * (g_b - k0 / GS)) & 15);
        const uint8_t* xp = x_lane + (size_t)(u_b * E / 32) * kSgIntStepBytes;
        const uint8_t* cp = c_lane + (size_t)g_b * kSgIntCtabBytes;
        const uint32_t ld0 = st + ld_lane;
        auto ld = [ld0](int u) { return ld0 + (uint32_t)u * 16u; };       // padded rows: units 16 bytes apart
        const uint32_t sp = p.scale_pitch;
        auto sa = [sc, sp](int h, int z, int G) { return sc + (uint32_t)(8 * h + 16 * z) * sp + 2 * G; };
        if (SU > 0 && !(last && nchunks > 1))
            slice_int<F, GS, SU>(yv, ld, sa, xp, cp, SU);
        else
            slice_int<F, GS, 0>(yv, ld, sa, xp, cp, sl.nu);
        if (last) {
            // the slice columns of token m: all four lanes of the quad (one
            // token), lanes t = 2m and 2m + 1 (two tokens)
            float r = yv[0] + yv[1], r8 = yv[2] + yv[3];
            r += __shfl_xor_sync(0xFFFFFFFFu, r, 1);
            r8 += __shfl_xor_sync(0xFFFFFFFFu, r8, 1);
            if (M == 1) {
                r += __shfl_xor_sync(0xFFFFFFFFu, r, 2);
                r8 += __shfl_xor_sync(0xFFFFFFFFu, r8, 2);
            }
            if ((t & 1) == 0 && (t >> 1) < M) {
                float* rp = red + ((tl * KW + warp) * 16 + g) * p.red_cols + (t >> 1);
                rp[0] = r;
                rp[8 * p.red_cols] = r8;
            }
        }
        if (++chunk == nchunks) {
            chunk = 0;
            ++tl;
        }
        __syncwarp();                   // every lane is done with stage i % S before it is refilled
    }
    cp_async_wait<0>();

    // ------------------------------------------------------------ cross-warp sum and store
    __syncthreads();
    const int rows_cta = nt * 16;
    for (int o = tid; o < M * rows_cta; o += 32 * KW) {
        const int m = o / rows_cta, rl = o - m * rows_cta;
        const int tl2 = rl >> 4, r = rl & 15;
        const int tile = t_begin + tl2;
        int mat = 0;
        while (mat + 1 < p.count && tile >= p.tile_begin[mat + 1]) ++mat;
        const int64_t row = (int64_t)(tile - p.tile_begin[mat]) * 16 + r;
        if (row >= p.N[mat]) continue;
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < KW; ++w) sum += red[((tl2 * KW + w) * 16 + r) * p.red_cols + m];
        p.y[mat][(int64_t)m * p.N[mat] + row] = (uint16_t)f32_to_bf16_bits(sum);
    }
}


// ------------------------------------------------------------------ TMA-fed variant
// The same integer core, fed by the tensor-memory accelerator: one producer
// warp (one elected lane) issues, per 16-row tile and stage, one 3-D box of
// codes and one 2-D box of scales (and biases) that complete on the stage's
// mbarrier, so the warps that compute never stall on issuing copies.
//
// Codes are viewed as a 3-D tensor [chunk][row][128 bytes] (strides 128 and
// row_bytes), and a stage's box [CH chunks][16 rows][128 bytes] lands with the
// 128-byte swizzle: byte chunk j of 128-byte line L is stored at chunk
// j ^ (L mod 8).  Line L = 16 c + r for row r of chunk c, so the 8 rows that
// one ldmatrix reads fall in 8 distinct bank groups.  Scales (and biases) are
// viewed the same way with 16-byte lines, [8-group unit][row][16 bytes], so the
// rows of one unit are 16 bytes apart, again in distinct banks.  Each of the 8
// compute warps owns units [CH w, CH w + CH) of the stage (16-byte code units,
// 8 per chunk); CH is the stage's chunk count.
//
// No table kernel runs ahead of it: after griddepcontrol.wait the producer
// starts the ring while each compute warp builds, in shared memory, the slices
// and group entries of its own K slice of x (int_table_item, the prep kernel's
// per-item work), which overlaps the first stages' flight.  A CTA that finds an
// activation the slices do not hold exactly drains the ring and computes its
// tiles with fp32 dot products (gemv_exact); every CTA sees the same x, so all
// make the same choice.
struct STmaParams {
    SGemvParams g;                          // shapes, tables, outputs (ring fields unused)
    CUtensorMap codes[kSgMaxMats];
    CUtensorMap scales[kSgMaxMats];
    CUtensorMap biases[kSgMaxMats];
    uint32_t off_stage;                     // first stage (1024-byte aligned)
    uint32_t stage_pitch;                   // bytes between stages (multiple of 1024)
    uint32_t scale_row_bytes;               // one row's scales of a stage (a multiple of 16): 16 rows x this per box
    uint32_t stage_tx;                      // bytes a stage's copies complete
    uint32_t off_bar;                       // 2 S + 1 mbarriers: full[S], empty[S], x (S <= kSgMaxStagesTma)
    uint32_t off_raw;                       // x, bf16 [M][K], copied in before the first stage
};

template <Fmt F, int GS, int CH>
__global__ void __launch_bounds__(32 * (kSgWarpsTma + 1), 1)
gemv_tma_kernel(const __grid_constant__ STmaParams q)
{
    using T = SFmt<F>;
    constexpr int E = T::E;
    constexpr int UPG = GS / E;
    constexpr bool kAffine = F != Fmt::Q4_0;
    constexpr int KW = kSgWarpsTma;
    constexpr int NU = CH;                               // units per warp per stage
    constexpr int kStageElems = CH * 128 * 8 / T::kBits;
    constexpr int kStageGroups = kStageElems / GS;
    static_assert(NU % (UPG > 2 ? UPG : 2) == 0, "a warp's units are whole atoms");
    static_assert(CH == 8 || CH == 16, "every warp's units start on a 128-byte chunk");
    const SGemvParams& p = q.g;

    // the swizzle pattern is relative to 1024-byte blocks: everything below
    // lives at offsets from a 1024-byte aligned base (1 KB extra is allocated)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    const int M = p.M, S = p.stages, nchunks = p.nchunks;
    const int t_begin = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
    const int t_end = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
    const int nt = t_end - t_begin;
    const int total = nt * nchunks;
    auto full_bar = [&](int s) { return sbase + q.off_bar + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return sbase + q.off_bar + 8u * (uint32_t)(S + s); };
    const uint32_t x_bar = sbase + q.off_bar + 16u * (uint32_t)S;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), KW);
        }
        mbar_init(x_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    grid_dependency_wait();
    grid_dependents_launch();

    if (warp == KW) {
        // ---------------------------------------------------------- producer
        int tile = t_begin, chunk = 0, mat = 0;
        while (mat + 1 < p.count && tile >= p.tile_begin[mat + 1]) ++mat;
        auto issue = [&](int i) {
            const int s = i % S;
            const uint32_t st = sbase + q.off_stage + (uint32_t)s * q.stage_pitch;
            const int row0 = (tile - p.tile_begin[mat]) * 16;
            mbar_arrive_expect_tx(full_bar(s), q.stage_tx);
            tma_load_3d(st, &q.codes[mat], full_bar(s), 0, row0, chunk * CH);
            const uint32_t sdst = st + (uint32_t)CH * 2048u;
            tma_load_3d(sdst, &q.scales[mat], full_bar(s), 0, row0, chunk * (kStageGroups / 8));
            if constexpr (kAffine)
                tma_load_3d(sdst + 16u * q.scale_row_bytes, &q.biases[mat], full_bar(s), 0, row0,
                            chunk * (kStageGroups / 8));
            if (++chunk == nchunks) {
                chunk = 0;
                ++tile;
                while (mat + 1 < p.count && tile >= p.tile_begin[mat + 1]) ++mat;
            }
        };
        if (lane == 0) {
            // x first, so that it is ahead of the weights in the copy engine's queue
            const uint32_t xbytes = (uint32_t)(M * p.K * 2);
            mbar_arrive_expect_tx(x_bar, xbytes);
            bulk_load(sbase + q.off_raw, p.x, xbytes, x_bar);
            for (int i = 0; i < total; ++i) {
                if (i >= S && !mbar_wait(empty_bar(i % S), (uint32_t)((i / S) - 1) & 1u)) break;
                issue(i);
            }
        }
        return;
    }

    // ------------------------------------------------------------ activation tables
    // This warp's K slice of x, in every chunk: steps [st0, st0 + nst), items
    // (token, step, quad position) 32 at a time; a group's lanes are consecutive.
    // The loads of up to four batches go out together, then their arithmetic; x
    // comes from this CTA's shared-memory copy.
    int inexact = 0;
    if (!mbar_wait_warp(x_bar, 0u)) inexact = 1;         // timed out (device error set): the fp32 path
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(smem + q.off_raw);
    {
        constexpr int nst = NU * E / 32;
        constexpr int kB = 4;
        const int items = M * nst * 4;                  // per chunk
        const int bpc = (items + 31) / 32;              // batches per chunk
        const int nb = nchunks * bpc;
        for (int b0 = 0; b0 < nb; b0 += kB) {
            uint32_t raw[kB][4];
            int mm[kB], stp[kB], tt[kB];
            bool ok[kB];
#pragma unroll
            for (int j = 0; j < kB; ++j) {
                const int b = b0 + j;
                const int c = b / bpc, idx = (b - c * bpc) * 32 + lane;
                ok[j] = b < nb && idx < items;
                const int ic = idx < items ? idx : items - 1;
                mm[j] = (ic >> 2) / nst;
                stp[j] = (c * kStageElems + warp * NU * E) / 32 + (ic >> 2) % nst;
                tt[j] = ic & 3;
                if (b < nb) int_item_load<F>(xs, p.K, mm[j], stp[j], tt[j], raw[j]);
            }
#pragma unroll
            for (int j = 0; j < kB; ++j)
                if (b0 + j < nb)                        // warp-uniform
                    inexact |= int_table_item_raw<F, GS>(raw[j], M, mm[j], stp[j], tt[j], lane, ok[j], smem + p.off_x,
                                                         smem + p.off_c);
        }
    }
    // the same answer in every compute warp (and every CTA: they all read the same x)
    int any_inexact;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, 2, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
                 : "=r"(any_inexact) : "r"(inexact), "n"(32 * KW) : "memory");
    if (any_inexact) {
        // release every stage so the producer finishes, then the fp32 path
        for (int i = 0; i < total; ++i) {
            if (!mbar_wait_warp(full_bar(i % S), (uint32_t)(i / S) & 1u)) break;
            if (lane == 0) mbar_arrive(empty_bar(i % S));
        }
        gemv_exact<F, GS>(p, t_begin, t_end, warp, lane, KW);
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const uint8_t* x_lane = smem + p.off_x + (size_t)((g * 4 + t) * 8);     // slice column g
    const uint8_t* c_lane = smem + p.off_c + (size_t)t * 16;
    // ldmatrix.x4 rows: lanes 0-7 rows 0-7 of unit u, 8-15 rows 8-15 of u, 16-31 the same of u + 1
    const int r = (lane & 7) + ((lane >> 3) & 1) * 8, hi = lane >> 4;
    uint32_t swz[4];                                     // swizzled byte offset of unit 2j + hi in its chunk
#pragma unroll
    for (int j = 0; j < 4; ++j) swz[j] = (uint32_t)(((2 * j + hi) ^ (r & 7)) << 4);
    const uint32_t lane_row = (uint32_t)r * 128u + (uint32_t)(warp * NU / 8) * 2048u;
    float* red = reinterpret_cast<float*>(smem + p.off_red);
    float yv[4] = {0.0f, 0.0f, 0.0f, 0.0f};

    int tl = 0, chunk = 0;
    for (int i = 0; i < total; ++i) {
        const int s = i % S;
        if (!mbar_wait_warp(full_bar(s), (uint32_t)(i / S) & 1u)) break;
        if (chunk == 0) yv[0] = yv[1] = yv[2] = yv[3] = 0.0f;
        const bool last = chunk == nchunks - 1;
        const uint32_t st = sbase + q.off_stage + (uint32_t)s * q.stage_pitch;
        const int u_b = chunk * (kStageElems / E) + warp * NU;            // first unit of the slice (in the row)
        const int g_b = u_b / UPG;                                        // its first group
        // scales: [8-group unit][16 rows][16 bytes], biases the same after them
        const uint8_t* sbox = smem + (st - sbase) + (size_t)CH * 2048u + (size_t)g * 16u;
        const int G0 = warp * NU / UPG;                 // the warp's first group of the stage
        const uint32_t zb = 16u * q.scale_row_bytes;
        auto sa = [sbox, G0, zb](int h, int z, int G) {
            const int Ga = G0 + G;
            return sbox + (uint32_t)z * zb + (uint32_t)h * 128u + (uint32_t)(Ga >> 3) * 256u + (uint32_t)(Ga & 7) * 2u;
        };
        const uint8_t* xp = x_lane + (size_t)(u_b * E / 32) * kSgIntStepBytes;
        const uint8_t* cp = c_lane + (size_t)g_b * kSgIntCtabBytes;
        const uint32_t ld0 = st + lane_row;
        // unit pair starting at relative unit u (even): chunk u / 8, pair (u mod 8) / 2
        auto ld = [&](int u) { return ld0 + (uint32_t)(u >> 3) * 2048u + swz[(u & 7) >> 1]; };
        slice_int<F, GS, NU>(yv, ld, sa, xp, cp, NU);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));       // this warp is done with stage s
        if (last) {
            float rr = yv[0] + yv[1], r8 = yv[2] + yv[3];
            rr += __shfl_xor_sync(0xFFFFFFFFu, rr, 1);
            r8 += __shfl_xor_sync(0xFFFFFFFFu, r8, 1);
            if (M == 1) {
                rr += __shfl_xor_sync(0xFFFFFFFFu, rr, 2);
                r8 += __shfl_xor_sync(0xFFFFFFFFu, r8, 2);
            }
            if ((t & 1) == 0 && (t >> 1) < M) {
                float* rp = red + ((tl * KW + warp) * 16 + g) * p.red_cols + (t >> 1);
                rp[0] = rr;
                rp[8 * p.red_cols] = r8;
            }
        }
        if (++chunk == nchunks) {
            chunk = 0;
            ++tl;
        }
    }

    // ------------------------------------------------------------ cross-warp sum and store
    asm volatile("bar.sync 1, %0;" ::"n"(32 * KW) : "memory");   // the compute warps only
    const int rows_cta = nt * 16;
    for (int o = tid; o < M * rows_cta; o += 32 * KW) {
        const int m = o / rows_cta, rl = o - m * rows_cta;
        const int tl2 = rl >> 4, rw = rl & 15;
        const int tile = t_begin + tl2;
        int mat = 0;
        while (mat + 1 < p.count && tile >= p.tile_begin[mat + 1]) ++mat;
        const int64_t row = (int64_t)(tile - p.tile_begin[mat]) * 16 + rw;
        if (row >= p.N[mat]) continue;
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < KW; ++w) sum += red[((tl2 * KW + w) * 16 + rw) * p.red_cols + m];
        p.y[mat][(int64_t)m * p.N[mat] + row] = (uint16_t)f32_to_bf16_bits(sum);
    }
}

}  // namespace bq
