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

// Per-chunk scale data of one row, already expanded for the conversion.
struct ChunkScale {
    uint32_t s0, s1;   // Q4_0: d_hi2, d_lo2 | AFF4: scale2, bias2 | AFF8: fp32 bits of scale, bias
};

template <Fmt F>
BQ_DEVINL ChunkScale load_scale(const uint16_t* scales, const uint16_t* biases, int64_t idx, bool valid)
{
    ChunkScale cs{0u, 0u};
    if (!valid) return cs;
    if constexpr (F == Fmt::Q4_0) {
        const float d = f16_bits_to_f32(__ldg(scales + idx));
        const uint32_t hi = f32_to_bf16_bits(d);
        const uint32_t lo = f32_to_bf16_bits(__fsub_rn(d, bf16_bits_to_f32(hi)));   // exact
        cs.s0 = hi | (hi << 16);
        cs.s1 = lo | (lo << 16);
    } else if constexpr (F == Fmt::AFF4) {
        const uint32_t s = __ldg(scales + idx), b = __ldg(biases + idx);
        cs.s0 = s | (s << 16);
        cs.s1 = b | (b << 16);
    } else {
        cs.s0 = __float_as_uint(bf16_bits_to_f32(__ldg(scales + idx)));
        cs.s1 = __float_as_uint(bf16_bits_to_f32(__ldg(biases + idx)));
    }
    return cs;
}

// Dequantize one 32-bit word of codes into the two A pairs of MMA `j` of the
// chunk: `first` for k-slots (2t, 2t+1), `second` for (2t+8, 2t+9).
template <Fmt F>
BQ_DEVINL void dequant_pairs(uint32_t word, int sub, const ChunkScale& cs, uint32_t& first, uint32_t& second)
{
    if constexpr (F == Fmt::Q4_0) {
        // sub 0: (e, e+2) from low nibbles of bytes 0,2 and (e+16, e+18) from high nibbles
        // sub 1: (e+1, e+3) and (e+17, e+19)   [e = 4 * word index]
        const uint32_t w = word >> (8 * sub);
        const uint32_t r0 = and_or(w, 0x000F000Fu, 0x43004300u);        // 128 + q
        const uint32_t r1 = and_or(w >> 4, 0x000F000Fu, 0x43004300u);
        const uint32_t q0 = hsub2_bf16(r0, 0x43084308u);                 // q - 8, exact
        const uint32_t q1 = hsub2_bf16(r1, 0x43084308u);
        first = hfma2_bf16(q0, cs.s0, hmul2_bf16(q0, cs.s1));
        second = hfma2_bf16(q1, cs.s0, hmul2_bf16(q1, cs.s1));
    } else if constexpr (F == Fmt::AFF4) {
        // sub 0: (e, e+4), (e+1, e+5); sub 1: (e+2, e+6), (e+3, e+7)   [e = 8 * word index]
        const uint32_t w = word >> (8 * sub);
        const uint32_t r0 = and_or(w, 0x000F000Fu, 0x43004300u);
        const uint32_t r1 = and_or(w >> 4, 0x000F000Fu, 0x43004300u);
        const uint32_t q0 = hsub2_bf16(r0, 0x43004300u);                 // q, exact
        const uint32_t q1 = hsub2_bf16(r1, 0x43004300u);
        first = hfma2_bf16(q0, cs.s0, cs.s1);
        second = hfma2_bf16(q1, cs.s0, cs.s1);
    } else {
        // one word per MMA: (e, e+1) and (e+2, e+3)   [e = 4 * word index]
        const float s = __uint_as_float(cs.s0), b = __uint_as_float(cs.s1);
        float f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            f[i] = __fsub_rn(__uint_as_float(prmt(word, 0x4B000000u, 0x7650u | i)), 8388608.0f);
        first = pack_bf16x2_rn(__fmaf_rn(s, f[0], b), __fmaf_rn(s, f[1], b));
        second = pack_bf16x2_rn(__fmaf_rn(s, f[2], b), __fmaf_rn(s, f[3], b));
    }
}

// B pairs of MMA j (0..7 for 32-element chunks, 0..3 for 16) from the 32 (or
// 16) activations of the chunk, held as 16 (or 8) u32 pairs (x[2i], x[2i+1]).
template <Fmt F>
BQ_DEVINL void x_pairs(const uint32_t* xw, int j, uint32_t& first, uint32_t& second)
{
    if constexpr (F == Fmt::Q4_0) {
        const int w = j >> 1;
        const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
        first = prmt(xw[2 * w], xw[2 * w + 1], sel);
        second = prmt(xw[8 + 2 * w], xw[8 + 2 * w + 1], sel);
    } else if constexpr (F == Fmt::AFF4) {
        const int w = j >> 1, o = j & 1;
        first = prmt(xw[4 * w + o], xw[4 * w + o + 2], 0x5410u);
        second = prmt(xw[4 * w + o], xw[4 * w + o + 2], 0x7632u);
    } else {
        first = xw[2 * j];
        second = xw[2 * j + 1];
    }
}

template <Fmt F, int RT>
struct GemvStage {
    uint4 w[RT][2];
    ChunkScale s[RT][2];
};

// One CTA: 16*RT weight rows x all K, KSPLIT warps splitting K; M <= 8*NT tokens.
template <Fmt F, int NT, int RT, int KSPLIT>
__global__ void __launch_bounds__(32 * KSPLIT)
gemv_kernel(const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
            const uint16_t* __restrict__ scales, const uint16_t* __restrict__ biases,
            uint16_t* __restrict__ y, int M, int N, int K, int group_size)
{
    using T = FmtTraits<F>;
    constexpr int kCE = T::kChunkElems;
    constexpr int kMmaPerChunk = kCE / 4;     // each MMA takes 4 of a thread's chunk elements
    constexpr int kXWords = kCE / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int row_base = blockIdx.x * 16 * RT;
    const int64_t row_bytes = (int64_t)K * T::kBits / 8;
    const int nchunks = K / kCE;
    const int per_warp = (nchunks + KSPLIT - 1) / KSPLIT;
    const int c_begin = warp * per_warp;
    const int c_end = min(nchunks, c_begin + per_warp);
    const int64_t scale_row = (F == Fmt::Q4_0) ? (K / 32) : (K / group_size);
    const int chunks_per_group = (F == Fmt::Q4_0) ? 1 : group_size / kCE;

    float acc[RT][NT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][n][i] = 0.0f;

    auto load_stage = [&](GemvStage<F, RT>& st, int c0) {
        const int c = c0 + t;
        const bool cvalid = c < c_end;
#pragma unroll
        for (int r = 0; r < RT; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = row_base + 16 * r + 8 * h + g;
                const bool v = cvalid && row < N;
                st.w[r][h] = v ? ldg_stream(wq + row * row_bytes + 16 * (int64_t)c) : make_uint4(0, 0, 0, 0);
                st.s[r][h] = load_scale<F>(scales, biases, row * scale_row + c / chunks_per_group, v);
            }
    };

    GemvStage<F, RT> cur, nxt;
    if (c_begin < c_end) load_stage(cur, c_begin);
    for (int c0 = c_begin; c0 < c_end; c0 += 4) {
        if (c0 + 4 < c_end) load_stage(nxt, c0 + 4);
        const int c = c0 + t;
        const bool cvalid = c < c_end;
        // activations of this chunk for each token tile
        uint32_t xw[NT][kXWords];
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
#pragma unroll
        for (int j = 0; j < kMmaPerChunk; ++j) {
            uint32_t b0[NT], b1[NT];
#pragma unroll
            for (int n = 0; n < NT; ++n) x_pairs<F>(xw[n], j, b0[n], b1[n]);
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                uint32_t a[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 wv = cur.w[r][h];
                    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
                    uint32_t f, s;
                    if constexpr (F == Fmt::AFF8) dequant_pairs<F>(words[j], 0, cur.s[r][h], f, s);
                    else dequant_pairs<F>(words[j >> 1], j & 1, cur.s[r][h], f, s);
                    a[h] = f;          // a0a1 (row g) / a2a3 (row g+8)
                    a[2 + h] = s;      // a4a5 / a6a7
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) mma_bf16_16816(acc[r][n], a[0], a[1], a[2], a[3], b0[n], b1[n]);
            }
        }
        cur = nxt;
    }

    // Reduce the KSPLIT partial tiles through shared memory.
    __shared__ float red[KSPLIT][16 * RT][8 * NT + 1];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            red[warp][16 * r + g][8 * n + 2 * t] = acc[r][n][0];
            red[warp][16 * r + g][8 * n + 2 * t + 1] = acc[r][n][1];
            red[warp][16 * r + g + 8][8 * n + 2 * t] = acc[r][n][2];
            red[warp][16 * r + g + 8][8 * n + 2 * t + 1] = acc[r][n][3];
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

}  // namespace bq
