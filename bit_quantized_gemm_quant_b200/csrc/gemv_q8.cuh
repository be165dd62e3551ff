// gemv_q8.cuh -- the quantized-activation decode path for Q4_0 weights.
//
// After the SYCL page "2026-05-06 Q4 sync-after focused repro" (Important source
// touch points), whose decode kernels multiply reordered Q4_0 weights by Q8_1
// activations: the activations are quantized per block of 32 to int8 with an
// fp32 scale, and each block's dot product is an exact integer sum of
// (weight code) x (activation code), scaled once per block.  The weights need
// no floating-point dequantization at all, which is what bounds the exact
// bf16 decode kernel.  The result is an approximation of the bf16 product (by
// the activation quantization), so it is a separate, opt-in path.
#pragma once

#include "common.cuh"

namespace bq {

// One thread per block of 32 activations: amax, d = amax / 127, id = 1 / d,
// q = roundf(x * id) (half away from zero), qsum = sum of q.  IEEE division and
// a single-rounding product, as the plain definition states.
__global__ void q8_1_quantize_kernel(const uint16_t* __restrict__ x, int8_t* __restrict__ xq, float* __restrict__ dx,
                                     int32_t* __restrict__ qsum, int64_t nblocks)
{
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 q = ldg_stream(x + b * 32 + 8 * v);
            w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
        }
        float f[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            f[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
            f[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(f[j]));
        const float d = __fdiv_rn(amax, 127.0f);
        const float id = d != 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
        int32_t sum = 0;
        uint32_t packed[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t word = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int q = (int)roundf(__fmul_rn(f[4 * i + e], id));
                sum += q;
                word |= ((uint32_t)q & 0xFFu) << (8 * e);
            }
            packed[i] = word;
        }
        uint4* out = reinterpret_cast<uint4*>(xq + b * 32);
        out[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        out[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        dx[b] = d;
        qsum[b] = sum;
    }
}

// y[m][n] = bf16( sum_b d_w[n][b] * dx[m][b] * (sum_j xq[m][32b+j] * q[n][32b+j] - 8 qsum[m][b]) ).
// One CTA owns 8 weight rows; its KS warps split the K blocks into contiguous
// ranges, and lane (g, t) of a warp takes row g and every fourth block of the
// warp's range (a quad reads 64 contiguous bytes of a row per step).  Block j's
// code word i holds the low nibbles of elements 4i..4i+3 and the high nibbles of
// 4i+16..4i+19, so (word & 0x0F0F0F0F) and ((word >> 4) & 0x0F0F0F0F) are four
// unsigned codes each, matched with the activation words i and i + 4 of the
// block by dp4a.  Codes are < 16, so the signed dp4a sees them unchanged; the -8
// offset is applied once per block via qsum.  All loads of a group of kUnroll
// blocks are issued before their arithmetic.  Partial sums: quad shuffles, then
// shared memory across the KS warps.
template <int MT, int KS>
__global__ void __launch_bounds__(32 * KS) gemv_q8_kernel(const int8_t* __restrict__ xq, const float* __restrict__ dx,
                                                          const int32_t* __restrict__ qsum,
                                                          const uint8_t* __restrict__ wq,
                                                          const uint16_t* __restrict__ scales,
                                                          uint16_t* __restrict__ y, int M, int N, int K)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int row = blockIdx.x * 8 + g;
    const int nb = K / 32;
    const int per_warp = (nb + KS - 1) / KS;
    const int bw0 = warp * per_warp, bw1 = min(nb, bw0 + per_warp);
    const bool valid = row < N;
    const uint8_t* wrow = wq + (int64_t)(valid ? row : 0) * (K / 2);
    const uint16_t* srow = scales + (int64_t)(valid ? row : 0) * nb;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

    constexpr int kUnroll = 4;                     // blocks of this lane in flight per iteration
    for (int b0 = bw0 + t; b0 < bw1; b0 += 4 * kUnroll) {
        uint4 wv[kUnroll];
        float dw[kUnroll];
        uint4 xa[kUnroll][MT], xb[kUnroll][MT];
        float sx[kUnroll][MT];
        int qs[kUnroll][MT];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int b = b0 + 4 * u;
            const bool in = b < bw1;
            wv[u] = (in && valid) ? ldg_stream(wrow + 16 * (int64_t)b) : make_uint4(0, 0, 0, 0);
            dw[u] = (in && valid) ? f16_bits_to_f32(__ldg(srow + b)) : 0.0f;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const bool use = in && m < M;
                const int64_t xi = (int64_t)m * nb + b;
                xa[u][m] = use ? ldg_cached(xq + xi * 32) : make_uint4(0, 0, 0, 0);
                xb[u][m] = use ? ldg_cached(xq + xi * 32 + 16) : make_uint4(0, 0, 0, 0);
                sx[u][m] = use ? __ldg(dx + xi) : 0.0f;
                qs[u][m] = use ? __ldg(qsum + xi) : 0;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t words[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo[i] = words[i] & 0x0F0F0F0Fu;
                hi[i] = (words[i] >> 4) & 0x0F0F0F0Fu;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int dot = __dp4a((int)lo[0], (int)xa[u][m].x, 0);
                dot = __dp4a((int)lo[1], (int)xa[u][m].y, dot);
                dot = __dp4a((int)lo[2], (int)xa[u][m].z, dot);
                dot = __dp4a((int)lo[3], (int)xa[u][m].w, dot);
                dot = __dp4a((int)hi[0], (int)xb[u][m].x, dot);
                dot = __dp4a((int)hi[1], (int)xb[u][m].y, dot);
                dot = __dp4a((int)hi[2], (int)xb[u][m].z, dot);
                dot = __dp4a((int)hi[3], (int)xb[u][m].w, dot);
                dot -= 8 * qs[u][m];
                acc[m] = __fmaf_rn(__fmul_rn(dw[u], sx[u][m]), (float)dot, acc[m]);
            }
        }
    }
    __shared__ float red[KS][8][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float v = acc[m];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (t == 0) red[warp][g][m] = v;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * MT; i += 32 * KS) {
        const int gg = i / MT, m = i % MT;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < KS; ++w) v += red[w][gg][m];
        const int r = blockIdx.x * 8 + gg;
        if (r < N && m < M) y[(int64_t)m * N + r] = (uint16_t)f32_to_bf16_bits(v);
    }
}

}  // namespace bq
