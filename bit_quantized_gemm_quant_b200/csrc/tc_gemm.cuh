// tc_gemm.cuh -- prefill path: tcgen05 tensor-core GEMM with TMEM accumulators.
//
// Computes y[M][N] = x[M][K] . W[N][K]^T.  The MMA runs "weights as M": one CTA
// owns 128 weight rows (the MMA's M = 128, TMEM lane = weight row) and a tile
// of `bn` tokens (the MMA's N, 16..256, TMEM column = token).  K advances 64
// elements (one 128-byte swizzle atom) per pipeline stage.
//
// Modes:
//   kModeBF16  -- A (weights) arrives by TMA as bf16: the second kernel of the
//                 unfused pair the MLX issue page measures ("quantized_matmul
//                 takes 14-41% longer than dequantize + bf16 matmul at prefill
//                 sizes (> 512 tokens)", Repro: x @ dequantize(...).T).
//   kModeQ4_0 / kModeAff4 / kModeAff8 -- the fused kernel: TMA brings the
//                 packed codes, eight dequant warps expand them to bf16 in the
//                 swizzled shared-memory A tile, and the MMA consumes it.  The
//                 expanded tile never touches HBM.  Each dequantized weight is
//                 reused across the whole token tile (bn tokens): the "static
//                 reuse" of dequantized weight tiles across activation tiles of
//                 "et-backend: Q4_0 matrix-engine GEMM rewrite for prefill"
//                 (Overview), mapped to the B200 tensor cores.
//
// Warp roles: warps [0, kDeqWarps) dequantize (fused modes); warps 0..3 also
// run the epilogue (TMEM -> registers -> bf16 -> global); one warp issues TMA,
// one issues tcgen05.mma (one elected thread) and owns the TMEM allocation.
// Every mbarrier wait is bounded (see mbar_wait); on a timeout each role skips
// its remaining work, the MMA thread still commits, and TMEM is freed.
#pragma once

#include "tcgen05.cuh"

namespace bq {

enum : int { kModeBF16 = 0, kModeQ4_0 = 1, kModeAff4 = 2, kModeAff8 = 3 };

template <int MODE> struct TcCfg {
    static constexpr int kDeqWarps = (MODE == kModeBF16) ? 0 : 8;
    static constexpr int kTmaWarp = (MODE == kModeBF16) ? 4 : kDeqWarps;
    static constexpr int kMmaWarp = kTmaWarp + 1;
    static constexpr int kThreads = 32 * (kMmaWarp + 1);
    static constexpr int kCodeBytesPerRow = (MODE == kModeAff8) ? 64 : 32;   // per 64-element k-block
    static constexpr uint32_t kABytes = 128 * 128;
    static constexpr uint32_t kCBytes = (MODE == kModeBF16) ? 0 : 128 * kCodeBytesPerRow;
};

struct TcParams {
    const uint16_t* scales;   // fused modes
    const uint16_t* biases;   // affine modes
    uint16_t* y;
    int M, N, K;
    int bn;                   // token tile = MMA N, multiple of 16 in [16, 256]
    int stages;
    int tmem_cols;            // power of two >= max(32, bn)
};

__host__ __device__ constexpr uint32_t tc_stage_bytes(int mode, int bn)
{
    return 128u * 128u + (uint32_t)bn * 128u + (mode == kModeBF16 ? 0u : (mode == kModeAff8 ? 128u * 64u : 128u * 32u));
}

// Byte offset of the 16-byte chunk `c` (K elements 8c..8c+7) of row `r` in a
// 128B-swizzled K-major tile with 128-byte rows.
BQ_DEVINL uint32_t sw128_offset(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

BQ_DEVINL void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}


// --- dequantization of one thread's 32 weights (half a k-block of one row) ---

// Q4_0: d = d_hi + d_lo split (see gemv.cuh); the 16 code bytes of one block.
BQ_DEVINL void deq_q4_0_half(uint4 raw, uint32_t dhi2, uint32_t dlo2, uint32_t a_tile, int r, int h)
{
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t lo[8], hi[8];   // natural-order pairs: lo = elements 0..15, hi = 16..31
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const uint32_t t = prmt(words[w], 0u, p ? 0x4342u : 0x4140u);   // [b, 0, b', 0]
            const uint32_t l = hsub2_bf16_i<0x43084308u>(and_or_i<0x000F000Fu, 0x43004300u>(t));
            const uint32_t u = hsub2_bf16_i<0x43084308u>(and_or_i<0x000F000Fu, 0x43004300u>(t >> 4));
            lo[2 * w + p] = hfma2_bf16(l, dhi2, hmul2_bf16(l, dlo2));
            hi[2 * w + p] = hfma2_bf16(u, dhi2, hmul2_bf16(u, dlo2));
        }
    }
    const int c0 = 4 * h;
    st_shared_v4(a_tile + sw128_offset(r, c0 + 0), lo[0], lo[1], lo[2], lo[3]);
    st_shared_v4(a_tile + sw128_offset(r, c0 + 1), lo[4], lo[5], lo[6], lo[7]);
    st_shared_v4(a_tile + sw128_offset(r, c0 + 2), hi[0], hi[1], hi[2], hi[3]);
    st_shared_v4(a_tile + sw128_offset(r, c0 + 3), hi[4], hi[5], hi[6], hi[7]);
}

// Affine 4-bit: 4 words of sequential nibbles; w = fma.rn.bf16x2(q, scale, bias).
BQ_DEVINL void deq_aff4_half(uint4 raw, uint32_t s2, uint32_t b2, uint32_t a_tile, int r, int h)
{
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t v[4];   // v[n] = (element n, element n+4) of the word
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const uint32_t q = hsub2_bf16_i<0x43004300u>(and_or_i<0x000F000Fu, 0x43004300u>(words[i] >> (4 * n)));
            v[n] = hfma2_bf16(q, s2, b2);
        }
        st_shared_v4(a_tile + sw128_offset(r, 4 * h + i), prmt(v[0], v[1], 0x5410u), prmt(v[2], v[3], 0x5410u),
                     prmt(v[0], v[1], 0x7632u), prmt(v[2], v[3], 0x7632u));
    }
}

// Affine 8-bit: 8 words of bytes; w = bf16_rne(fmaf(scale, q, bias)).
BQ_DEVINL void deq_aff8_half(uint4 raw0, uint4 raw1, float s, float b, uint32_t a_tile, int r, int h)
{
    const uint32_t words[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            f[e] = __fsub_rn(__uint_as_float(prmt(words[i], 0x4B000000u, 0x7650u | e)), 8388608.0f);
        o[2 * i] = pack_bf16x2_rn(__fmaf_rn(s, f[0], b), __fmaf_rn(s, f[1], b));
        o[2 * i + 1] = pack_bf16x2_rn(__fmaf_rn(s, f[2], b), __fmaf_rn(s, f[3], b));
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        st_shared_v4(a_tile + sw128_offset(r, 4 * h + c), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

struct DeqScale { uint32_t a, b; };

template <int MODE>
BQ_DEVINL DeqScale deq_load_scale(const TcParams& p, int row, int it, int h)
{
    DeqScale r{0u, 0u};
    if (row >= p.N) return r;
    if constexpr (MODE == kModeQ4_0) {
        const float d = f16_bits_to_f32(__ldg(p.scales + (int64_t)row * (p.K / 32) + 2 * it + h));
        const uint32_t hi = f32_to_bf16_bits(d);
        const uint32_t lo = f32_to_bf16_bits(__fsub_rn(d, bf16_bits_to_f32(hi)));
        r.a = hi | (hi << 16);
        r.b = lo | (lo << 16);
    } else {
        const int64_t gi = (int64_t)row * (p.K / 64) + it;
        r.a = __ldg(p.scales + gi);
        r.b = __ldg(p.biases + gi);
    }
    return r;
}

template <int MODE>
__global__ void __launch_bounds__(TcCfg<MODE>::kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a, TcParams p)
{
    using C = TcCfg<MODE>;
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * p.bn;
    const int n0 = blockIdx.y * 128;
    const int nk = (p.K + 63) / 64;
    const int S = p.stages;
    const uint32_t b_bytes = (uint32_t)p.bn * 128u;

    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t a_base = base;
    const uint32_t b_base = a_base + (uint32_t)S * C::kABytes;
    const uint32_t c_base = b_base + (uint32_t)S * b_bytes;
    const uint32_t bar_base = c_base + (uint32_t)S * C::kCBytes;
    auto full_bar = [&](int s) { return bar_base + 8u * (uint32_t)s; };
    auto afull_bar = [&](int s) { return bar_base + 8u * (uint32_t)(S + s); };
    auto empty_bar = [&](int s) { return bar_base + 8u * (uint32_t)(2 * S + s); };
    const uint32_t tmem_full_bar = bar_base + 8u * (uint32_t)(3 * S);
    const uint32_t tmem_slot = tmem_full_bar + 8u;
    uint8_t* smem_gen = smem_raw + (base - smem_u32(smem_raw));
    volatile uint32_t* tmem_slot_ptr = reinterpret_cast<volatile uint32_t*>(smem_gen + (tmem_slot - base));

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(afull_bar(s), C::kDeqWarps * 32);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tmem_full_bar, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(tmem_slot, (uint32_t)p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot_ptr;

    if (warp == C::kTmaWarp) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_a);
            int issued = 0;
            for (int it = 0; it < nk; ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u)) break;
                mbar_arrive_expect_tx(full_bar(s), b_bytes + (MODE == kModeBF16 ? C::kABytes : C::kCBytes));
                tma_load_2d(b_base + (uint32_t)s * b_bytes, &tm_x, full_bar(s), it * 64, m0);
                if constexpr (MODE == kModeBF16)
                    tma_load_2d(a_base + (uint32_t)s * C::kABytes, &tm_a, full_bar(s), it * 64, n0);
                else
                    tma_load_2d(c_base + (uint32_t)s * C::kCBytes, &tm_a, full_bar(s), it * C::kCodeBytesPerRow, n0);
                ++issued;
            }
            // Drain: every issued copy has landed before this CTA may exit.
            for (int it = (issued > S ? issued - S : 0); it < issued; ++it)
                mbar_wait(full_bar(it % S), (uint32_t)(it / S) & 1u);
        }
    } else if (warp == C::kMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16_f32(128, p.bn);
            for (int it = 0; it < nk; ++it) {
                const int s = it % S;
                const uint32_t ph = (uint32_t)(it / S) & 1u;
                if (!mbar_wait(full_bar(s), ph)) break;
                if constexpr (MODE != kModeBF16) {
                    if (!mbar_wait(afull_bar(s), ph)) break;
                }
                tc_fence_after();
                const uint32_t a_addr = a_base + (uint32_t)s * C::kABytes;
                const uint32_t b_addr = b_base + (uint32_t)s * b_bytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ss(tmem_base, umma_desc_k_sw128(a_addr + 32u * kk), umma_desc_k_sw128(b_addr + 32u * kk),
                                idesc, (it | kk) != 0 ? 1u : 0u);
                umma_commit(empty_bar(s));
            }
            umma_commit(tmem_full_bar);   // also on an early exit: nothing stays in flight
            mbar_wait(tmem_full_bar, 0);
        }
        __syncwarp();
    } else if (MODE != kModeBF16 && warp < C::kDeqWarps) {
        const int r = 32 * (warp & 3) + lane;   // weight row within the tile
        const int h = warp >> 2;                // which 32-element half of each k-block
        const int row = n0 + r;
        DeqScale sc = deq_load_scale<MODE>(p, row, 0, h);
        for (int it = 0; it < nk; ++it) {
            const int s = it % S;
            const uint32_t ph = (uint32_t)(it / S) & 1u;
            const DeqScale sc_next = (it + 1 < nk) ? deq_load_scale<MODE>(p, row, it + 1, h) : sc;
            if (!mbar_wait(full_bar(s), ph)) break;
            const uint32_t codes = c_base + (uint32_t)s * C::kCBytes + (uint32_t)(r * C::kCodeBytesPerRow);
            const uint32_t a_tile = a_base + (uint32_t)s * C::kABytes;
            if constexpr (MODE == kModeQ4_0) {
                deq_q4_0_half(ld_shared_v4(codes + 16u * h), sc.a, sc.b, a_tile, r, h);
            } else if constexpr (MODE == kModeAff4) {
                deq_aff4_half(ld_shared_v4(codes + 16u * h), sc.a | (sc.a << 16), sc.b | (sc.b << 16), a_tile, r, h);
            } else {
                deq_aff8_half(ld_shared_v4(codes + 32u * h), ld_shared_v4(codes + 32u * h + 16u),
                              bf16_bits_to_f32(sc.a), bf16_bits_to_f32(sc.b), a_tile, r, h);
            }
            fence_proxy_async_smem();
            mbar_arrive(afull_bar(s));
            sc = sc_next;
        }
    }

    // Epilogue: warps 0..3, TMEM lane quarter = warp.
    if (warp < 4) {
        const bool ok = mbar_wait(tmem_full_bar, 0);
        tc_fence_after();
        if (ok) {
            const int row = n0 + 32 * warp + lane;
            const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * warp) << 16);
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(lane_addr + (uint32_t)c0, v);
                tmem_wait_ld();
                if (row < p.N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < p.M) p.y[(int64_t)m * p.N + row] = (uint16_t)f32_to_bf16_bits(__uint_as_float(v[j]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::kMmaWarp) tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
}

}  // namespace bq
