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


// ------------------------------------------------------------------ transpose = 0
// Decode GEMV for affine weights stored [K][N] (mx.quantize of the [K][N]
// matrix: codes and groups along N, the transpose = False form of the MLX
// issue's quantized_matmul): y[m][n] = sum_k x[m][k] (s[k][g(n)] q[k][n] + z[k][g(n)]).
// A cluster of KS CTAs (up to 8 along the grid's y) owns 32 CPL output columns
// and splits K into KS contiguous ranges, one per CTA.  A warp takes every 8th
// row of its CTA's range, and its lanes read one contiguous run of that row:
// lane l owns columns CPL l .. CPL l + CPL - 1 (CPL = 8 or 16 columns: 16 to
// 128 bits of the bit stream, so 2-, 4- and 8-bit codes; they share one group
// since groups are >= 32 columns).  Rows come in batches of U, two batches in
// registers: the next batch's loads are in flight while the current one is
// computed.  x is staged in shared memory as fp32 [row][token], 512 rows at a
// time.  Per row and token a lane adds (x s) q for its columns and x z
// once.  The 8 warps are summed through shared memory, then the KS CTAs'
// partial sums through distributed shared memory, each in a fixed order, so the
// result depends only on the shape and the cluster size.  The product is over
// the exact weights s q + z (within the GEMM tolerance of their bf16
// roundings), as the any-width GEMV's.
constexpr int kGtWarps = 8;     // rows in flight per CTA step (one per warp)
constexpr int kGtMaxSplit = 8;  // CTAs per cluster (portable cluster size)
constexpr int kGtXRows = 512;   // rows of x staged per pass

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster arrives; shared-memory writes before
// it are visible to the cluster after it.
__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float of CTA `rank`'s shared memory at the offset of `p` in this CTA's.
__device__ __forceinline__ float ld_cluster_f32(const float* p, uint32_t rank)
{
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    uint32_t ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

// Columns per lane by token count: 16 up to two tokens, 8 above (registers).
template <int MT> constexpr int gemv_t_cpl() { return MT <= 2 ? 16 : 8; }

// Bit position, inside the word it is read from, of code c of a lane's run, as
// the kernel reads it: codes that end at or below bit 23 are masked in place in
// their word, the others in the word shifted right by 12.  Masked in place and
// OR'd into the bits of 2^23, a code at position p reads as 2^23 + q 2^p
// (exact while p + BITS <= 23); the column's sum is scaled back by 2^-p at the end.
template <int BITS> __host__ __device__ constexpr int gt_pos(int b) { return b + BITS <= 23 ? b : b - 12; }

// One batch of U rows of a lane: code words, scale and bias bits.
template <int U, int WPL>
struct GtBatch {
    uint32_t w[U][WPL];
    uint16_t s[U], z[U];
};

template <int BITS, int MT, int U, int MINB>
__global__ void __launch_bounds__(32 * kGtWarps, MINB)
gemv_t_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ wq, const uint16_t* __restrict__ scales,
              const uint16_t* __restrict__ biases, uint16_t* __restrict__ y, int M, int N, int K, int group_size)
{
    static_assert(BITS == 2 || BITS == 4 || BITS == 8, "a lane's columns must be whole bytes of its words");
    constexpr int CPL = gemv_t_cpl<MT>();
    constexpr int COLS = 32 * CPL;                            // columns per cluster
    constexpr int WB = CPL * BITS;                            // code bits per lane and row: 16 .. 128
    constexpr int WPL = WB >= 32 ? WB / 32 : 1;               // words loaded per lane and row
    constexpr int EPW = WB >= 32 ? 32 / BITS : CPL;           // codes per loaded word
    constexpr int XST = MT;                                   // x row stride in smem (floats)
    constexpr int XV = MT <= 4 ? MT : 4;                      // floats per x vector load
    constexpr int STEP = kGtWarps * U;                        // rows of a CTA per batch
    __shared__ float red[kGtWarps][COLS];                     // one token's per-warp partials
    __shared__ float part[MT][COLS];                          // the CTA's partial sums
    __shared__ __align__(16) float xsm[kGtXRows * XST];
    const uint32_t ks = cluster_rank(), nks = cluster_size();
    const int kc = (int)(((int64_t)K + nks - 1) / nks);
    const int k0 = (int)ks * kc, k1 = min(K, k0 + kc);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * COLS + lane * CPL;
    const bool live = n0 < N;                                 // N is a multiple of the group (>= 32)
    const int64_t words_per_row = (int64_t)N * BITS / 32;
    const int64_t groups_per_row = N / group_size;
    const int wbit = WB >= 32 ? 0 : (n0 * BITS) & 31;         // first bit of the lane's codes in its word
    const int64_t widx = (int64_t)n0 * BITS / 32;             // a multiple of WPL: vector loads are aligned
    const int64_t gidx = n0 / group_size;
    const uint32_t* wrow = wq + widx;
    const uint16_t* srow = scales + gidx;
    const uint16_t* zrow = biases + gidx;

    auto load = [&](GtBatch<U, WPL>& bt, int kb, int kend) {
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int k = kb + kGtWarps * i;
#pragma unroll
            for (int j = 0; j < WPL; ++j) bt.w[i][j] = 0u;
            bt.s[i] = bt.z[i] = 0;
            if (live && k < kend) {
                const uint32_t* src = wrow + (int64_t)k * words_per_row;
                if constexpr (WPL == 4) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
                    bt.w[i][0] = v.x; bt.w[i][WPL > 1 ? 1 : 0] = v.y;
                    bt.w[i][WPL > 2 ? 2 : 0] = v.z; bt.w[i][WPL > 3 ? 3 : 0] = v.w;
                } else if constexpr (WPL == 2) {
                    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
                    bt.w[i][0] = v.x; bt.w[i][WPL > 1 ? 1 : 0] = v.y;
                } else {
                    bt.w[i][0] = __ldg(src);
                }
                bt.s[i] = __ldg(srow + (int64_t)k * groups_per_row);
                bt.z[i] = __ldg(zrow + (int64_t)k * groups_per_row);
            }
        }
    };

    float acc[CPL][MT], accb[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        accb[m] = 0.0f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c][m] = 0.0f;
    }
    auto compute = [&](const GtBatch<U, WPL>& bt, int kb, int kend, int c0) {
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int k = kb + kGtWarps * i;
            if (k < kend) {
                const float s = bf16_bits_to_f32(bt.s[i]), z = bf16_bits_to_f32(bt.z[i]);
                float xv[MT];
                const float* xr = xsm + (k - c0) * XST;
#pragma unroll
                for (int m = 0; m < MT; m += XV) {
                    if constexpr (XV == 4) {
                        const float4 t = *reinterpret_cast<const float4*>(xr + m);
                        xv[m] = t.x; xv[m + 1] = t.y; xv[m + 2] = t.z; xv[m + 3] = t.w;
                    } else if constexpr (XV == 2) {
                        const float2 t = *reinterpret_cast<const float2*>(xr + m);
                        xv[m] = t.x; xv[m + 1] = t.y;
                    } else {
                        xv[m] = xr[m];
                    }
                }
                float q[CPL];                                  // q 2^pos, exact
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    const uint32_t base = WB >= 32 ? bt.w[i][j] : bt.w[i][0] >> wbit;
                    const uint32_t high = base >> 12;
#pragma unroll
                    for (int e = 0; e < EPW; ++e) {
                        const int b = e * BITS;
                        const uint32_t src = b + BITS <= 23 ? base : high;
                        const uint32_t mask = ((1u << BITS) - 1u) << gt_pos<BITS>(b);
                        q[j * EPW + e] = __uint_as_float((src & mask) | 0x4B000000u) - 8388608.0f;
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const float xs = xv[m] * s;
#pragma unroll
                    for (int c = 0; c < CPL; ++c) acc[c][m] = __fmaf_rn(xs, q[c], acc[c][m]);
                    accb[m] = __fmaf_rn(xv[m], z, accb[m]);
                }
            }
        }
    };

    GtBatch<U, WPL> cur, nxt;
    for (int c0 = k0; c0 < k1; c0 += kGtXRows) {
        const int cend = min(k1, c0 + kGtXRows);
        load(cur, c0 + warp, cend);                           // in flight while x is staged
        __syncthreads();                                      // the previous pass is done with xsm
        for (int o = threadIdx.x; o < (cend - c0) * MT; o += 32 * kGtWarps) {
            const int r = o / MT, m = o - r * MT;
            xsm[r * XST + m] = m < M ? bf16_bits_to_f32(__ldg(x + (int64_t)m * K + c0 + r)) : 0.0f;
        }
        __syncthreads();
        if (!live) continue;
        for (int kb = c0 + warp; kb < cend; kb += STEP) {
            load(nxt, kb + STEP, cend);                       // the next batch's loads overlap this one's math
            compute(cur, kb, cend, c0);
            cur = nxt;
        }
    }
    // scale each column's sum back by 2^-pos; per token, the warps' partials in order
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int pos = gt_pos<BITS>((c % EPW) * BITS);
            const float back = __uint_as_float((uint32_t)(127 - pos) << 23);
            red[warp][lane * CPL + c] = __fmaf_rn(acc[c][m], back, accb[m]);
        }
        __syncthreads();
        for (int c = threadIdx.x; c < COLS; c += 32 * kGtWarps) {
            float v = red[0][c];
#pragma unroll
            for (int w = 1; w < kGtWarps; ++w) v += red[w][c];
            part[m][c] = v;
        }
        __syncthreads();
    }
    cluster_barrier();
    // the cluster's CTAs in rank order; CTA ks writes every nks-th block of 256 entries
    for (int o = (int)ks * 32 * kGtWarps + threadIdx.x; o < MT * COLS; o += (int)nks * 32 * kGtWarps) {
        const int m = o / COLS, c = o - m * COLS;
        const int n = blockIdx.x * COLS + c;
        if (m >= M || n >= N) continue;
        float pv[kGtMaxSplit];
#pragma unroll
        for (int r = 0; r < kGtMaxSplit; ++r) pv[r] = (uint32_t)r < nks ? ld_cluster_f32(&part[m][c], r) : 0.0f;
        float v = pv[0];
#pragma unroll
        for (int r = 1; r < kGtMaxSplit; ++r)
            if ((uint32_t)r < nks) v += pv[r];
        y[(int64_t)m * N + n] = (uint16_t)f32_to_bf16_bits(v);
    }
    cluster_barrier();    // no CTA leaves while another may still read its shared memory
}

}  // namespace bq
