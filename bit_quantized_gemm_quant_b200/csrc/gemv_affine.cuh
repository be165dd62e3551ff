// gemv_affine.cuh -- decode path (M <= 8) for affine weights of any supported
// width (2, 3, 4, 6, 8 bits), used for the 2-, 3- and 6-bit layouts that the
// 16-byte-chunk MMA GEMV (gemv.cuh) does not cover.
//
// mx.quantized_matmul at 1-32 tokens on the MLX issue page (Summary: the
// quantized kernel wins there) is a matrix-vector product over packed codes.
// Here one warp owns kRows weight rows and its lanes take whole code units
// (AffUnit<BITS>: W words holding E codes, never straddling a group).  Per unit
// and token the lane forms the fp32 sums  sum_e x[e] * q[e]  and  sum_e x[e]
// (even and odd e in the two lanes of packed fp32x2 operations, the lanes added
// at the unit's end), and adds  scale * (first) + bias * (second)  to the row's
// result: the dot product of x with the weights scale * q + bias, over the
// exact weights rather than their bf16 roundings (within the GEMM tolerance,
// which covers a 2^-9 relative difference per weight).  Codes become floats
// exactly through the 2^23 magic number.  Lane partials are reduced with
// shuffles; the summation order is fixed, so results are deterministic.
#pragma once

#include "common.cuh"
#include "dequant.cuh"

namespace bq {

constexpr int kGaRows = 4;      // weight rows per warp
constexpr int kGaWarps = 4;     // warps per CTA

template <int BITS, int MT>
__global__ void __launch_bounds__(32 * kGaWarps)
gemv_affine_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ wq,
                   const uint16_t* __restrict__ scales, const uint16_t* __restrict__ biases,
                   uint16_t* __restrict__ y, int M, int N, int K, int group_size)
{
    constexpr int W = AffUnit<BITS>::W, E = AffUnit<BITS>::E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = (blockIdx.x * kGaWarps + warp) * kGaRows;
    if (row0 >= N) return;                                   // warp-uniform
    const int units = K / E, groups = K / group_size;
    float acc[kGaRows][MT];
#pragma unroll
    for (int r = 0; r < kGaRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

    for (int u = lane; u < units; u += 32) {
        const int k0 = u * E;
        uint32_t w[kGaRows][W];
        float sc[kGaRows], bi[kGaRows];
#pragma unroll
        for (int r = 0; r < kGaRows; ++r) {
            const int row = min(row0 + r, N - 1);             // rows past N repeat the last row, not stored
            load_unit<BITS>(wq + (int64_t)row * (units * W), u, w[r]);
            const int64_t gi = (int64_t)row * groups + k0 / group_size;
            sc[r] = bf16_bits_to_f32(__ldg(scales + gi));
            bi[r] = bf16_bits_to_f32(__ldg(biases + gi));
        }
        // (even, odd) element pairs: x, the codes and the sums in packed fp32x2
        uint64_t xq[kGaRows][MT], xs[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            xs[m] = 0u;
#pragma unroll
            for (int r = 0; r < kGaRows; ++r) xq[r][m] = 0u;
        }
        const uint64_t magic2 = f32x2_splat(8388608.0f);
#pragma unroll
        for (int e0 = 0; e0 < E; e0 += 8) {
            uint64_t xv[MT][4];                               // (x[e0 + 2i], x[e0 + 2i + 1])
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4 v = (m < M) ? ldg_cached(x + (int64_t)m * K + k0 + e0) : make_uint4(0, 0, 0, 0);
                const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xv[m][i] = f32x2_pack(vw[i] << 16, vw[i] & 0xFFFF0000u);
                    xs[m] = add_f32x2(xs[m], xv[m][i]);
                }
            }
#pragma unroll
            for (int r = 0; r < kGaRows; ++r)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint64_t q = sub_f32x2(f32x2_pack(unit_code<BITS>(w[r], e0 + 2 * i) | 0x4B000000u,
                                                            unit_code<BITS>(w[r], e0 + 2 * i + 1) | 0x4B000000u),
                                                 magic2);
#pragma unroll
                    for (int m = 0; m < MT; ++m) xq[r][m] = fma_f32x2(xv[m][i], q, xq[r][m]);
                }
        }
#pragma unroll
        for (int r = 0; r < kGaRows; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                acc[r][m] = __fmaf_rn(sc[r], f32x2_sum(xq[r][m]), __fmaf_rn(bi[r], f32x2_sum(xs[m]), acc[r][m]));
    }
#pragma unroll
    for (int r = 0; r < kGaRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = acc[r][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[r][m] = v;
        }
    if (lane < kGaRows * MT) {
        const int r = lane / MT, m = lane % MT;
        float v = 0.0f;
#pragma unroll
        for (int rr = 0; rr < kGaRows; ++rr)
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
                if (rr == r && mm == m) v = acc[rr][mm];
        if (row0 + r < N && m < M) y[(int64_t)m * N + row0 + r] = (uint16_t)f32_to_bf16_bits(v);
    }
}

}  // namespace bq
