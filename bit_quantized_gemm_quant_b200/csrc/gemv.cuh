// gemv.cuh -- decode path (M <= 32): streams the packed weights once from HBM
// with 128-bit loads, dequantizes in registers and feeds warp-level bf16 MMAs
// with fp32 accumulation.
//
// The pages' decode kernels are prior art for this path: decode (one token)
// routes to a vector-dot kernel in "et-backend: Q4_0 matrix-engine GEMM
// rewrite for prefill" (Overview), the SYCL MMVQ kernel over "reordered" Q4_0
// in "2026-05-06 Q4 sync-after focused repro" (Important source touch
// points), and the quantized kernel wins at 1-32 tokens on the MLX issue page
// (Summary).  Here each warp owns 16*RT weight rows; the 4 threads of a quad
// share a row and take consecutive 16-byte chunks of it, so a warp reads 64
// contiguous bytes per row per step.  The CTA's KSPLIT warps split K and
// reduce through shared memory.
//
// Exactness: the dequantized weight fed to the MMA is bf16_rne of the exact
// product for Q4_0 and affine-8 (bit-identical to *_dequantize), and one
// fma.rn.bf16x2 of (q, scale, bias) for affine-4 (single rounding of the exact
// value; identical whenever scale*q + bias is exact in fp32).
//
// Q4_0 trick: d (fp16, 11 significant bits) = d_hi + d_lo with d_hi = bf16(d)
// and d_lo exact in bf16 (<= 3 significant bits).  With qm8 = q - 8 exact in
// bf16, u = qm8 * d_lo is exact, and fma(qm8, d_hi, u) rounds the exact
// qm8 * d once: bf16_rne(d * (q - 8)) in three packed bf16x2 ops per 2 weights.
#pragma once

#include "common.cuh"

namespace bq {


enum class Fmt : int { Q4_0 = 0, AFF4 = 1, AFF8 = 2 };

#ifndef BQ_Q4_ROUTE
#define BQ_Q4_ROUTE 0
#endif
// Q4_0 dequant route of the decode kernel: 0 = packed-bf16 split-scale, 1 = fp32 FMA magic.
constexpr int kQ4Route = BQ_Q4_ROUTE;

template <Fmt F> struct FmtTraits;
template <> struct FmtTraits<Fmt::Q4_0> { static constexpr int kChunkElems = 32; static constexpr int kBits = 4; };
template <> struct FmtTraits<Fmt::AFF4> { static constexpr int kChunkElems = 32; static constexpr int kBits = 4; };
template <> struct FmtTraits<Fmt::AFF8> { static constexpr int kChunkElems = 16; static constexpr int kBits = 8; };

BQ_DEVINL void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                              uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-chunk scale data of one row, expanded for the conversion.
//  Q4_0: fp32 (d * 2^-s, -(2^(23-s) + 8) * d) for s = 8, 12, 16 (see dequant_word)
//  AFF4: bf16x2 (scale, scale) and (bias, bias)
//  AFF8: fp32 scale and bias
struct ChunkScale {
    float a[3], c[3];
    uint32_t s2, b2;
};

// Raw 16-bit scale (and bias) bits of one row's chunk; zero for masked rows/chunks.
template <Fmt F>
BQ_DEVINL void load_scale_raw(const uint16_t* scales, const uint16_t* biases, int64_t idx, bool valid,
                              uint32_t& s_raw, uint32_t& b_raw)
{
    s_raw = valid ? (uint32_t)__ldg(scales + idx) : 0u;
    if constexpr (F != Fmt::Q4_0) b_raw = valid ? (uint32_t)__ldg(biases + idx) : 0u;
    else b_raw = 0u;
}

// Expansion happens where the scale is used, so the load above stays asynchronous.
template <Fmt F>
BQ_DEVINL ChunkScale expand_scale(uint32_t s_raw, uint32_t b_raw)
{
    ChunkScale cs;
    if constexpr (F == Fmt::Q4_0 && kQ4Route == 0) {
        const float d = f16_bits_to_f32(s_raw);
        cs.s2 = pack_bf16x2_rn(d, d);                                           // d_hi in both halves
        const float lo = __fsub_rn(d, __uint_as_float(cs.s2 << 16));           // d - d_hi, exact
        cs.b2 = pack_bf16x2_rn(lo, lo);                                         // exact in bf16
    } else if constexpr (F == Fmt::Q4_0) {
        const float d = f16_bits_to_f32(s_raw);
        // (2^(23-s) + 8) has at most 13 significant bits and d at most 11, so
        // every constant below is exact in fp32.
        cs.a[0] = __fmul_rn(d, 0x1p-8f);  cs.c[0] = __fmul_rn(d, -32776.0f);
        cs.a[1] = __fmul_rn(d, 0x1p-12f); cs.c[1] = __fmul_rn(d, -2056.0f);
        cs.a[2] = __fmul_rn(d, 0x1p-16f); cs.c[2] = __fmul_rn(d, -136.0f);
    } else if constexpr (F == Fmt::AFF4) {
        cs.s2 = s_raw | (s_raw << 16);
        cs.b2 = b_raw | (b_raw << 16);
    } else {
        cs.a[0] = bf16_bits_to_f32(s_raw);
        cs.c[0] = bf16_bits_to_f32(b_raw);
    }
    return cs;
}

// Dequantize one 32-bit word of codes into the A pairs of the MMAs it feeds:
// p[0], p[1] = (first, second) of the first MMA, p[2], p[3] of the second
// (AFF8: one MMA, p[0], p[1]).  "first" fills k-slots (2t, 2t+1) and "second"
// (2t+8, 2t+9) of the thread's quad position t.
//
// Q4_0, exact: a nibble q placed at bit s >= 8 of the fp32 magic 2^23 gives
// f = 2^23 + q*2^s, and fma(f, d*2^-s, -(2^(23-s)+8)*d) = (q-8)*d exactly (the
// addend is exact because s >= 8, the result has <= 14 significant bits), so
// cvt.rn.bf16x2 rounds d*(q-8) once: bit-identical to the plain definition.
// The word holds bytes 4i..4i+3 of the block: nibbles n0..n7 are elements
// 4i, 4i+16, 4i+1, 4i+17, 4i+2, 4i+18, 4i+3, 4i+19; pairs are emitted in
// natural element order so the activations need no permutation.
template <Fmt F>
BQ_DEVINL void dequant_word(uint32_t word, const ChunkScale& cs, uint32_t (&p)[4])
{
    if constexpr (F == Fmt::Q4_0 && kQ4Route == 0) {
        // bf16 route: d = d_hi + d_lo (d_hi = bf16(d), d_lo exact in bf16); with
        // qm8 = q - 8 exact, fma(qm8, d_hi, qm8 * d_lo) rounds the exact qm8 * d once.
        // Pairs: (4i, 4i+2), (4i+16, 4i+18), (4i+1, 4i+3), (4i+17, 4i+19).
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t qm8 = hsub2_bf16_i<0x43084308u>(and_or_i<0x000F000Fu, 0x43004300u>(word >> (4 * k)));
            p[k] = hfma2_bf16(qm8, cs.s2, hmul2_bf16(qm8, cs.b2));
        }
    } else if constexpr (F == Fmt::Q4_0) {
        constexpr uint32_t kMagic = 0x4B000000u;
        const uint32_t lo = word << 8, hi = word >> 12;
        const float w0 = __fmaf_rn(__uint_as_float(and_or_i<0x00F00u, kMagic>(lo)), cs.a[0], cs.c[0]);    // 4i
        const float w1 = __fmaf_rn(__uint_as_float(and_or_i<0x0F000u, kMagic>(lo)), cs.a[1], cs.c[1]);    // 4i+16
        const float w2 = __fmaf_rn(__uint_as_float(and_or_i<0x00F00u, kMagic>(word)), cs.a[0], cs.c[0]);  // 4i+1
        const float w3 = __fmaf_rn(__uint_as_float(and_or_i<0x0F000u, kMagic>(word)), cs.a[1], cs.c[1]);  // 4i+17
        const float w4 = __fmaf_rn(__uint_as_float(and_or_i<0xF0000u, kMagic>(word)), cs.a[2], cs.c[2]);  // 4i+2
        const float w5 = __fmaf_rn(__uint_as_float(and_or_i<0x00F00u, kMagic>(hi)), cs.a[0], cs.c[0]);    // 4i+18
        const float w6 = __fmaf_rn(__uint_as_float(and_or_i<0x0F000u, kMagic>(hi)), cs.a[1], cs.c[1]);    // 4i+3
        const float w7 = __fmaf_rn(__uint_as_float(and_or_i<0xF0000u, kMagic>(hi)), cs.a[2], cs.c[2]);    // 4i+19
        p[0] = pack_bf16x2_rn(w0, w2);   // (4i, 4i+1)
        p[1] = pack_bf16x2_rn(w1, w3);   // (4i+16, 4i+17)
        p[2] = pack_bf16x2_rn(w4, w6);   // (4i+2, 4i+3)
        p[3] = pack_bf16x2_rn(w5, w7);   // (4i+18, 4i+19)
    } else if constexpr (F == Fmt::AFF4) {
        // nibble n = element 8i+n.  (word >> 4n) & 0x000F000F | 0x4300 -> bf16 (128+q_n, 128+q_{n+4});
        // subtracting 128 is exact; one fma.rn.bf16x2 rounds scale*q + bias once.
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const uint32_t r = and_or_i<0x000F000Fu, 0x43004300u>(word >> (4 * n));
            p[n] = hfma2_bf16(hsub2_bf16_i<0x43004300u>(r), cs.s2, cs.b2);   // (8i+n, 8i+n+4)
        }
    } else {
        // bytes (0, 1) and (2, 3), two weights per packed fp32x2 subtract and FMA
        const uint64_t s2 = f32x2_splat(cs.a[0]), b2 = f32x2_splat(cs.c[0]);
        p[0] = deq_aff8_pair<0>(word, s2, b2);
        p[1] = deq_aff8_pair<2>(word, s2, b2);
        p[2] = p[3] = 0u;
    }
}

// B pairs (activations) matching dequant_word's A pairs for word i of the
// chunk; xw holds the chunk's activations as u32 pairs (x[2j], x[2j+1]).
template <Fmt F>
BQ_DEVINL void x_word_pairs(const uint32_t* xw, int i, uint32_t (&b)[4])
{
    if constexpr (F == Fmt::Q4_0 && kQ4Route == 0) {
        // p[0] = (4i, 4i+2) / p[1] = (4i+16, 4i+18) feed the first MMA, p[2], p[3] the second
        b[0] = prmt(xw[2 * i], xw[2 * i + 1], 0x5410u);            // x[4i], x[4i+2]
        b[1] = prmt(xw[8 + 2 * i], xw[9 + 2 * i], 0x5410u);        // x[4i+16], x[4i+18]
        b[2] = prmt(xw[2 * i], xw[2 * i + 1], 0x7632u);            // x[4i+1], x[4i+3]
        b[3] = prmt(xw[8 + 2 * i], xw[9 + 2 * i], 0x7632u);        // x[4i+17], x[4i+19]
    } else if constexpr (F == Fmt::Q4_0) {
        b[0] = xw[2 * i];         // x[4i], x[4i+1]
        b[1] = xw[8 + 2 * i];     // x[4i+16], x[4i+17]
        b[2] = xw[2 * i + 1];     // x[4i+2], x[4i+3]
        b[3] = xw[9 + 2 * i];     // x[4i+18], x[4i+19]
    } else if constexpr (F == Fmt::AFF4) {
        b[0] = prmt(xw[4 * i], xw[4 * i + 2], 0x5410u);       // (8i, 8i+4)
        b[1] = prmt(xw[4 * i], xw[4 * i + 2], 0x7632u);       // (8i+1, 8i+5)
        b[2] = prmt(xw[4 * i + 1], xw[4 * i + 3], 0x5410u);   // (8i+2, 8i+6)
        b[3] = prmt(xw[4 * i + 1], xw[4 * i + 3], 0x7632u);   // (8i+3, 8i+7)
    } else {
        b[0] = xw[2 * i];
        b[1] = xw[2 * i + 1];
        b[2] = b[3] = 0u;
    }
}

template <Fmt F, int RT>
struct GemvStage {
    uint4 w[RT][2];          // 16 code bytes of rows g and g+8 of each m16 tile
    uint32_t s[RT][2];       // raw scale bits
    uint32_t b[RT][2];       // raw bias bits (affine)
};

template <Fmt F, int NT>
BQ_DEVINL void load_x_chunk(const uint16_t* __restrict__ x, int M, int K, int g, int c, bool cvalid,
                            uint32_t (&xw)[NT][FmtTraits<F>::kChunkElems / 2])
{
    constexpr int kCE = FmtTraits<F>::kChunkElems;
    constexpr int kXWords = kCE / 2;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int m = 8 * n + g;
        if (cvalid && m < M) {
            const uint16_t* xp = x + (int64_t)m * K + (int64_t)c * kCE;
#pragma unroll
            for (int v = 0; v < kXWords / 4; ++v) {
                const uint4 q = ldg_cached(xp + 8 * v);
                xw[n][4 * v] = q.x; xw[n][4 * v + 1] = q.y; xw[n][4 * v + 2] = q.z; xw[n][4 * v + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int v = 0; v < kXWords; ++v) xw[n][v] = 0u;
        }
    }
}

// Loads of one 4-chunk step (per thread: one 16-byte chunk of each of its rows).
template <Fmt F, int RT>
BQ_DEVINL void load_step(GemvStage<F, RT>& st, const uint8_t* __restrict__ wq, const uint16_t* __restrict__ scales,
                         const uint16_t* __restrict__ biases, int row_base, int g, int N, int c, bool cvalid,
                         int64_t row_bytes, int64_t scale_row, int chunks_per_group)
{
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = row_base + 16 * r + 8 * h + g;
            const bool v = cvalid && row < N;
            st.w[r][h] = v ? ldg_stream(wq + row * row_bytes + 16 * (int64_t)c) : make_uint4(0, 0, 0, 0);
            load_scale_raw<F>(scales, biases, row * scale_row + c / chunks_per_group, v, st.s[r][h], st.b[r][h]);
        }
}

// One CTA: 16*RT weight rows x all K; KSPLIT warps split K into contiguous
// ranges and reduce through shared memory; M <= 8*NT tokens.  Each warp runs a
// software pipeline over its 4-chunk steps with PIPE register stages: the
// weight loads of step s + PIPE are issued before step s is computed, so every
// load has PIPE steps of other work to hide behind and no warp ever waits a
// full memory round trip between batches.
template <Fmt F, int NT, int RT, int KSPLIT, int PIPE>
__device__ __forceinline__ void gemv_body(const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
                                          const uint16_t* __restrict__ scales, const uint16_t* __restrict__ biases,
                                          uint16_t* __restrict__ y, int M, int N, int K, int group_size, int row_base)
{
    using T = FmtTraits<F>;
    constexpr int kCE = T::kChunkElems;
    constexpr int kWords = 4;                                   // 16-byte chunk
    constexpr int kMmaPerWord = (F == Fmt::AFF8) ? 1 : 2;
    constexpr int kXWords = kCE / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t row_bytes = (int64_t)K * T::kBits / 8;
    const int nchunks = K / kCE;
    const int per_warp = (nchunks + KSPLIT - 1) / KSPLIT;
    const int c_begin = warp * per_warp;
    const int c_end = min(nchunks, c_begin + per_warp);
    const int nsteps = (c_end - c_begin + 3) / 4;
    const int64_t scale_row = (F == Fmt::Q4_0) ? (K / 32) : (K / group_size);
    const int chunks_per_group = (F == Fmt::Q4_0) ? 1 : group_size / kCE;

    // Two accumulator sets (even / odd MMA of a word) halve the dependent MMA chain.
    float acc[2][RT][NT][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int r = 0; r < RT; ++r)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[e][r][n][i] = 0.0f;

    auto step_chunk = [&](int s) { return c_begin + 4 * s + t; };
    GemvStage<F, RT> ring[PIPE];
#pragma unroll
    for (int d = 0; d < PIPE; ++d)
        load_step<F, RT>(ring[d], wq, scales, biases, row_base, g, N, step_chunk(d), d < nsteps && step_chunk(d) < c_end,
                         row_bytes, scale_row, chunks_per_group);

    for (int s0 = 0; s0 < nsteps; s0 += PIPE) {
#pragma unroll
        for (int d = 0; d < PIPE; ++d) {
            const int s = s0 + d;
            if (s < nsteps) {
                const int c = step_chunk(s);
                uint32_t xw[NT][kXWords];
                load_x_chunk<F, NT>(x, M, K, g, c, c < c_end, xw);
                ChunkScale cs[RT][2];
#pragma unroll
                for (int r = 0; r < RT; ++r)
#pragma unroll
                    for (int h = 0; h < 2; ++h) cs[r][h] = expand_scale<F>(ring[d].s[r][h], ring[d].b[r][h]);
#pragma unroll
                for (int i = 0; i < kWords; ++i) {
                    uint32_t b[NT][4];
#pragma unroll
                    for (int n = 0; n < NT; ++n) x_word_pairs<F>(xw[n], i, b[n]);
#pragma unroll
                    for (int r = 0; r < RT; ++r) {
                        uint32_t pa[2][4];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint4 wv = ring[d].w[r][h];
                            const uint32_t word = i == 0 ? wv.x : i == 1 ? wv.y : i == 2 ? wv.z : wv.w;
                            dequant_word<F>(word, cs[r][h], pa[h]);
                        }
#pragma unroll
                        for (int mm = 0; mm < kMmaPerWord; ++mm)
#pragma unroll
                            for (int n = 0; n < NT; ++n)
                                // A regs: row g first, row g+8 first, row g second, row g+8 second
                                mma_bf16_16816(acc[mm][r][n], pa[0][2 * mm], pa[1][2 * mm], pa[0][2 * mm + 1],
                                               pa[1][2 * mm + 1], b[n][2 * mm], b[n][2 * mm + 1]);
                    }
                }
                // refill this ring slot with step s + PIPE (PIPE - 1 steps of cover)
                const int cn = step_chunk(s + PIPE);
                load_step<F, RT>(ring[d], wq, scales, biases, row_base, g, N, cn, s + PIPE < nsteps && cn < c_end,
                                 row_bytes, scale_row, chunks_per_group);
            }
        }
    }

    // Reduce the KSPLIT partial tiles through shared memory.
    __shared__ float red[KSPLIT][16 * RT][8 * NT + 1];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            red[warp][16 * r + g][8 * n + 2 * t] = acc[0][r][n][0] + acc[1][r][n][0];
            red[warp][16 * r + g][8 * n + 2 * t + 1] = acc[0][r][n][1] + acc[1][r][n][1];
            red[warp][16 * r + g + 8][8 * n + 2 * t] = acc[0][r][n][2] + acc[1][r][n][2];
            red[warp][16 * r + g + 8][8 * n + 2 * t + 1] = acc[0][r][n][3] + acc[1][r][n][3];
        }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 16 * RT * 8 * NT; idx += 32 * KSPLIT) {
        const int row = idx % (16 * RT), m = idx / (16 * RT);
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < KSPLIT; ++w) s += red[w][row][m];
        if (m < M && row_base + row < N)
            y[(int64_t)m * N + row_base + row] = (uint16_t)f32_to_bf16_bits(s);
    }
}

// One matrix: CTA b owns rows [16*RT*b, 16*RT*(b+1)).
template <Fmt F, int NT, int RT, int KSPLIT, int PIPE, int MINB>
__global__ void __launch_bounds__(32 * KSPLIT, MINB)
gemv_kernel(const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
            const uint16_t* __restrict__ scales, const uint16_t* __restrict__ biases,
            uint16_t* __restrict__ y, int M, int N, int K, int group_size)
{
    gemv_body<F, NT, RT, KSPLIT, PIPE>(x, wq, scales, biases, y, M, N, K, group_size, blockIdx.x * 16 * RT);
}

// Several matrices that share x (and K, format, group size), one launch: the
// CTAs of matrix i are [tile_begin[i], tile_begin[i+1]).
constexpr int kMultiMax = 8;
struct GemvMultiTable {
    int count;
    int tile_begin[kMultiMax + 1];
    const uint8_t* wq[kMultiMax];
    const uint16_t* scales[kMultiMax];
    const uint16_t* biases[kMultiMax];
    uint16_t* y[kMultiMax];
    int N[kMultiMax];
};

template <Fmt F, int NT, int RT, int KSPLIT, int PIPE, int MINB>
__global__ void __launch_bounds__(32 * KSPLIT, MINB)
gemv_multi_kernel(const uint16_t* __restrict__ x, const __grid_constant__ GemvMultiTable tab, int M, int K,
                  int group_size)
{
    int i = 0;
    while (i + 1 < tab.count && (int)blockIdx.x >= tab.tile_begin[i + 1]) ++i;
    gemv_body<F, NT, RT, KSPLIT, PIPE>(x, tab.wq[i], tab.scales[i], tab.biases[i], tab.y[i], M, tab.N[i], K,
                                       group_size, ((int)blockIdx.x - tab.tile_begin[i]) * 16 * RT);
}

}  // namespace bq
