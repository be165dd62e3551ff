// dequant.cuh -- Q4_0 / affine dequantize and quantize kernels (HBM-bound, bit-exact).
//
// Dequantize is the first half of the unfused pair the MLX issue page measures
// ("quantized_matmul takes 14-41% longer than dequantize + bf16 matmul at
// prefill sizes (> 512 tokens)", Repro: x @ mx.dequantize(...).T).  Quantize is
// input preparation (mx.quantize on the same page); its integer codes are
// decided in fp32 with explicitly rounded operations so they are reproducible.
#pragma once

#include "common.cuh"

namespace bq {

// ----------------------------------------------------------------------------
// Q4_0 dequantize: one thread per 32-weight block (16 code bytes + one fp16 d).
// out = bf16_rne(d * (q - 8)); the fp32 product is exact (11 x 4 significant
// bits), so this matches the plain definition bit for bit.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
q4_0_dequant_kernel(const uint8_t* __restrict__ wq, const uint16_t* __restrict__ d16,
                    uint16_t* __restrict__ out, int64_t nblocks)
{
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        const uint4 raw = ldg_stream(wq + b * 16);
        const float d = f16_bits_to_f32(__ldg(d16 + b));
        const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t lo[8], hi[8];   // lo: elements 0..15, hi: elements 16..31, packed in pairs
#pragma unroll
        for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t b0 = (words[w] >> (16 * p)) & 0xFFu;
                const uint32_t b1 = (words[w] >> (16 * p + 8)) & 0xFFu;
                const float l0 = __fmul_rn(d, (float)((int)(b0 & 15u) - 8));
                const float l1 = __fmul_rn(d, (float)((int)(b1 & 15u) - 8));
                const float h0 = __fmul_rn(d, (float)((int)(b0 >> 4) - 8));
                const float h1 = __fmul_rn(d, (float)((int)(b1 >> 4) - 8));
                lo[2 * w + p] = pack_bf16x2_rn(l0, l1);
                hi[2 * w + p] = pack_bf16x2_rn(h0, h1);
            }
        }
        uint4* o = reinterpret_cast<uint4*>(out + b * 32);
        o[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        o[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        o[2] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        o[3] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    }
}

// ----------------------------------------------------------------------------
// Affine codes: each row is a little-endian bit stream, code k at stream bits
// BITS*k .. BITS*k + BITS - 1 (lowest first; stream bit i = bit i%32 of word
// i/32).  For 2, 4 and 8 bits that is 32/BITS codes per word, lowest bits
// first, as on the MLX issue page's 4- and 8-bit weights; 3- and 6-bit codes
// may cross a word.  A unit of W words holds E whole codes, E divides every
// group size (32, 64, 128), so a unit never straddles a group.
// ----------------------------------------------------------------------------
template <int BITS> struct AffUnit;
template <> struct AffUnit<2> { static constexpr int W = 2, E = 32; };
template <> struct AffUnit<3> { static constexpr int W = 3, E = 32; };
template <> struct AffUnit<4> { static constexpr int W = 4, E = 32; };
template <> struct AffUnit<6> { static constexpr int W = 3, E = 16; };
template <> struct AffUnit<8> { static constexpr int W = 4, E = 16; };

// Code e of a unit (e a compile-time constant after unrolling).
template <int BITS>
BQ_DEVINL uint32_t unit_code(const uint32_t (&w)[AffUnit<BITS>::W], int e)
{
    const int bit = BITS * e, i = bit >> 5, sh = bit & 31;
    uint32_t q = w[i] >> sh;
    if (sh + BITS > 32) q |= w[i + 1] << (32 - sh);
    return q & ((1u << BITS) - 1u);
}

// The W words of unit u of a packed array (16-, 8- or 4-byte loads by W).
template <int BITS>
BQ_DEVINL void load_unit(const uint32_t* __restrict__ wq, int64_t u, uint32_t (&w)[AffUnit<BITS>::W])
{
    constexpr int W = AffUnit<BITS>::W;
    const uint32_t* p = wq + u * W;
    if constexpr (W == 4) {
        const uint4 v = ldg_stream(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (W == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < W; ++i) w[i] = __ldg(p + i);
    }
}

// ----------------------------------------------------------------------------
// Affine dequantize: one thread per unit.  out = bf16_rne(fmaf(scale, q, bias)).
// ----------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256)
affine_dequant_kernel(const uint32_t* __restrict__ wq, const uint16_t* __restrict__ scales,
                      const uint16_t* __restrict__ biases, uint16_t* __restrict__ out,
                      int64_t nunits, int64_t K, int group_size)
{
    constexpr int W = AffUnit<BITS>::W, E = AffUnit<BITS>::E;
    const int64_t units_per_row = K / E;
    const int64_t groups_per_row = K / group_size;
    for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < nunits;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = u / units_per_row;
        const int64_t k0 = (u % units_per_row) * E;
        uint32_t w[W];
        load_unit<BITS>(wq, u, w);
        const int64_t gi = n * groups_per_row + k0 / group_size;
        const float s = bf16_bits_to_f32(__ldg(scales + gi));
        const float bb = bf16_bits_to_f32(__ldg(biases + gi));
        uint32_t packed[E / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2)
            packed[e / 2] = pack_bf16x2_rn(__fmaf_rn(s, (float)unit_code<BITS>(w, e), bb),
                                           __fmaf_rn(s, (float)unit_code<BITS>(w, e + 1), bb));
        uint4* o = reinterpret_cast<uint4*>(out + n * K + k0);
#pragma unroll
        for (int v = 0; v < E / 8; ++v)
            o[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    }
}

// ----------------------------------------------------------------------------
// Affine dequantize with a transposed result: the packed matrix is W[R][C]
// (codes along C, groups of C), the output its transpose out[C][R] in bf16.
// One CTA per tile of 64 rows x 128 columns: consecutive threads dequantize
// the same unit column of consecutive rows into a shared tile kept as
// [column][row], which is then written out 16 bytes per thread along R.
// ----------------------------------------------------------------------------
constexpr int kTrRows = 64, kTrCols = 128;

template <int BITS>
__global__ void __launch_bounds__(256)
affine_dequant_t_kernel(const uint32_t* __restrict__ wq, const uint16_t* __restrict__ scales,
                        const uint16_t* __restrict__ biases, uint16_t* __restrict__ out, int64_t R, int64_t C,
                        int group_size)
{
    constexpr int W = AffUnit<BITS>::W, E = AffUnit<BITS>::E;
    constexpr int kUnitsPerTileRow = kTrCols / E;
    __shared__ __align__(16) uint16_t tile[kTrCols][kTrRows + 8];   // [column][row]; rows padded by 16 bytes
    const int64_t units_per_row = C / E, groups_per_row = C / group_size;
    const int64_t tiles_r = (R + kTrRows - 1) / kTrRows, tiles_c = (C + kTrCols - 1) / kTrCols;
    for (int64_t t = blockIdx.x; t < tiles_r * tiles_c; t += gridDim.x) {
        const int64_t r0 = (t / tiles_c) * kTrRows, c0 = (t % tiles_c) * kTrCols;
        for (int i = threadIdx.x; i < kTrRows * kUnitsPerTileRow; i += blockDim.x) {
            const int rr = i % kTrRows, cu = i / kTrRows;    // consecutive threads: consecutive rows
            const int64_t r = r0 + rr, c = c0 + (int64_t)cu * E;
            if (r >= R || c >= C) continue;
            uint32_t w[W];
            load_unit<BITS>(wq, r * units_per_row + c / E, w);
            const int64_t gi = r * groups_per_row + c / group_size;
            const float s = bf16_bits_to_f32(__ldg(scales + gi));
            const float bb = bf16_bits_to_f32(__ldg(biases + gi));
#pragma unroll
            for (int e = 0; e < E; ++e)
                tile[cu * E + e][rr] = (uint16_t)f32_to_bf16_bits(__fmaf_rn(s, (float)unit_code<BITS>(w, e), bb));
        }
        __syncthreads();
        // out[c][r0 .. r0 + 63]: 8 threads per column, 8 rows (16 bytes) each
        for (int i = threadIdx.x; i < kTrCols * (kTrRows / 8); i += blockDim.x) {
            const int cc = i / (kTrRows / 8), rq = (i % (kTrRows / 8)) * 8;
            const int64_t c = c0 + cc, r = r0 + rq;
            if (c >= C || r >= R) continue;
            uint16_t* dst = out + c * R + r;
            if (r + 8 <= R) {
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&tile[cc][rq]);
            } else {
                for (int j = 0; j < 8 && r + j < R; ++j) dst[j] = tile[cc][rq + j];
            }
        }
        __syncthreads();
    }
}

// ----------------------------------------------------------------------------
// Q4_0 quantize: one thread per block, same operation order as the definition.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
q4_0_quant_kernel(const float* __restrict__ w, uint8_t* __restrict__ wq, uint16_t* __restrict__ d16,
                  int64_t nblocks)
{
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        const float* blk = w + b * 32;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            const float4 t = *reinterpret_cast<const float4*>(blk + j);
            v[j] = t.x; v[j + 1] = t.y; v[j + 2] = t.z; v[j + 3] = t.w;
        }
        float amax = 0.0f, mx = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float a = fabsf(v[j]);
            if (a > amax) { amax = a; mx = v[j]; }
        }
        const float d = __fdiv_rn(mx, -8.0f);
        d16[b] = __half_as_ushort(__float2half_rn(d));
        uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            // IEEE division by the unrounded fp32 d (an all-zero block has d == 0 and q = 8)
            int q0 = (int)__fadd_rn(d != 0.0f ? __fdiv_rn(v[j], d) : 0.0f, 8.5f);
            int q1 = (int)__fadd_rn(d != 0.0f ? __fdiv_rn(v[j + 16], d) : 0.0f, 8.5f);
            q0 = min(15, max(0, q0));
            q1 = min(15, max(0, q1));
            out[j / 4] |= (uint32_t)(q0 | (q1 << 4)) << (8 * (j % 4));
        }
        *reinterpret_cast<uint4*>(wq + b * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ----------------------------------------------------------------------------
// Affine quantize: one thread per group.  scale = bf16((max - min) / L),
// bias = bf16(min); q = clamp(rint((w - bias) / scale), 0, L) from the stored
// bf16 values (q = 0 when scale == 0).  Codes are packed unit by unit into the
// row's bit stream (a group holds whole units).
// ----------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256)
affine_quant_kernel(const float* __restrict__ w, uint32_t* __restrict__ wq, uint16_t* __restrict__ scales,
                    uint16_t* __restrict__ biases, int64_t ngroups, int group_size)
{
    constexpr int L = (1 << BITS) - 1;
    constexpr int W = AffUnit<BITS>::W, E = AffUnit<BITS>::E;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < ngroups;
         g += (int64_t)gridDim.x * blockDim.x) {
        const float* grp = w + g * group_size;
        float mn = grp[0], mx = grp[0];
        for (int j = 1; j < group_size; ++j) {
            const float v = grp[j];
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        const float scale_f = __fdiv_rn(__fsub_rn(mx, mn), (float)L);
        const uint32_t s16 = f32_to_bf16_bits(scale_f);
        const uint32_t b16 = f32_to_bf16_bits(mn);
        scales[g] = (uint16_t)s16;
        biases[g] = (uint16_t)b16;
        const float s = bf16_bits_to_f32(s16);
        const float bb = bf16_bits_to_f32(b16);
        uint32_t* out = wq + g * (group_size / E) * W;
        for (int j0 = 0; j0 < group_size; j0 += E) {
            uint32_t word[W];
#pragma unroll
            for (int i = 0; i < W; ++i) word[i] = 0u;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                uint32_t q = 0u;
                if (s != 0.0f) {
                    float r = rintf(__fdiv_rn(__fsub_rn(grp[j0 + e], bb), s));
                    r = fminf(fmaxf(r, 0.0f), (float)L);
                    q = (uint32_t)r;
                }
                const int bit = BITS * e, i = bit >> 5, sh = bit & 31;
                word[i] |= q << sh;
                if (sh + BITS > 32) word[i + 1] |= q >> (32 - sh);
            }
#pragma unroll
            for (int i = 0; i < W; ++i) out[(j0 / E) * W + i] = word[i];
        }
    }
}

// Array-of-structs Q4_0 import: blocks of 18 bytes (fp16 d little-endian, then
// the 16 code bytes) -> separate code and scale arrays.  One warp moves 32
// consecutive blocks (576 bytes, 16-byte aligned when the base is) per step:
// 16-byte loads into shared memory, then each lane splits out its own block.
constexpr int kImportWarps = 8;

__global__ void __launch_bounds__(32 * kImportWarps) q4_0_import_aos_kernel(const uint8_t* __restrict__ blocks,
                                                                           uint8_t* __restrict__ wq,
                                                                           uint16_t* __restrict__ d16, int64_t nb)
{
    __shared__ __align__(16) uint8_t buf[kImportWarps][576];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* sb = buf[warp];
    const int64_t nchunks = (nb + 31) / 32;
    for (int64_t c = (int64_t)blockIdx.x * kImportWarps + warp; c < nchunks; c += (int64_t)gridDim.x * kImportWarps) {
        const int64_t b0 = c * 32;
        const int cnt = (int)(nb - b0 < 32 ? nb - b0 : 32);
        const uint8_t* src = blocks + b0 * 18;
        if (cnt == 32) {
            reinterpret_cast<uint4*>(sb)[lane] = ldg_stream(src + 16 * lane);
            if (lane < 4) reinterpret_cast<uint4*>(sb)[32 + lane] = ldg_stream(src + 512 + 16 * lane);
        } else {
            for (int i = lane; i < cnt * 18; i += 32) sb[i] = src[i];
        }
        __syncwarp();
        if (lane < cnt) {
            const uint8_t* blk = sb + lane * 18;
            d16[b0 + lane] = (uint16_t)(blk[0] | (blk[1] << 8));
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                w[k] = (uint32_t)blk[2 + 4 * k] | ((uint32_t)blk[3 + 4 * k] << 8) | ((uint32_t)blk[4 + 4 * k] << 16) |
                       ((uint32_t)blk[5 + 4 * k] << 24);
            reinterpret_cast<uint4*>(wq)[b0 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncwarp();
    }
}

}  // namespace bq
