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
// The kernel is persistent: one CTA per SM walks a static schedule of
// (weight tile, token tile) pairs, token tiles fastest so that concurrently
// running CTAs share weight tiles in L2.  Two TMEM accumulators let a separate
// epilogue warpgroup drain tile i while the MMA warp already accumulates tile
// i + 1, and the producer runs ahead across tile boundaries.
// Warp roles: [0, kDeqWarps) dequantize (fused modes: groups of eight that take
// k-blocks in turn), four epilogue warps
// (TMEM -> registers -> bf16 -> global), one TMA producer warp, one MMA warp
// (one elected thread issues every tcgen05.mma and owns the TMEM allocation).
// Every mbarrier wait is bounded (see mbar_wait); on a timeout each role skips
// its remaining work, the MMA thread still commits, and TMEM is freed.
#pragma once

#include "tcgen05.cuh"

namespace bq {

enum : int { kModeBF16 = 0, kModeQ4_0 = 1, kModeAff4 = 2, kModeAff8 = 3 };

template <int MODE> struct TcCfg {
    // Fused modes: kDeqGroups groups of dequant warps take k-blocks in turn.  A
    // group covers the 128 rows of a k-block: 4 warps (one per TMEM lane quarter)
    // expanding 64 weights per thread, or 8 warps expanding 32.
    static constexpr int kDeqGroups = 2;
    static constexpr int kDeqWarpsPerGroup = 8;
    static constexpr int kDeqWarps = (MODE == kModeBF16) ? 0 : kDeqWarpsPerGroup * kDeqGroups;
    static constexpr int kEpiWarp0 = kDeqWarps;          // 4 warps: lane quarter = warp % 4
    static constexpr int kTmaWarp = kEpiWarp0 + 4;
    static constexpr int kMmaWarp = kTmaWarp + 1;
    static constexpr int kThreads = 32 * (kMmaWarp + 1);
    static constexpr int kCodeBytesPerRow = (MODE == kModeAff8) ? 64 : 32;   // per 64-element k-block
    static constexpr uint32_t kABytes = (MODE == kModeBF16) ? 128 * 128 : 0;   // fused: weight tile in TMEM
    static constexpr uint32_t kCBytes = (MODE == kModeBF16) ? 0 : 128 * kCodeBytesPerRow;
};

struct TcParams {
    const uint16_t* scales;   // fused modes
    const uint16_t* biases;   // affine modes
    uint16_t* y;
    int M, N, K;
    int bn;                   // token tile = MMA N, multiple of 16 in [16, 256]
    int stages;
    int m_tiles;              // token tiles per weight tile
    int tiles;                // total tiles
    int acc_stride;           // TMEM columns between the two accumulators
    int num_acc;              // 2: the epilogue drains one tile while the next accumulates; 1: bn up to 256
    int gs_shift;             // log2 of the group size (Q4_0: 5; affine: 5, 6 or 7)
    int vec_scales;           // scale rows are 16-byte aligned and hold whole 8-group windows
    int dp_tiles;             // tiles [0, dp_tiles) run whole, one unit each
    int splits;               // K splits of each later tile (fused modes); > 1: fp32 partials to ws
    float* ws;                // fp32 partials of the split tiles when splits > 1:
                              // [split][tile - dp_tiles][token of the tile (bn)][weight row of the tile (128)]
};

// Shared memory per pipeline stage: the activation tile (bn x 64 bf16, 128B
// swizzled K-major) plus the bf16 weight tile (kModeBF16, same layout) or the
// packed codes (fused modes; their dequantized tile goes to TMEM).
__host__ __device__ constexpr uint32_t tc_stage_bytes(int mode, int bn)
{
    return (uint32_t)bn * 128u + (mode == kModeBF16 ? 128u * 128u : (mode == kModeAff8 ? 128u * 64u : 128u * 32u));
}

// Byte offset of the 16-byte chunk `c` (K elements 8c..8c+7) of row `r` in a
// 128B-swizzled K-major tile with 128-byte rows (the layout TMA writes and the
// UMMA descriptor describes): chunk c of row r sits at position c ^ (r mod 8).
BQ_DEVINL uint32_t sw128_offset(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// --- dequantization of one thread's 32 weights (half a k-block of one row) ---
// Each returns 16 bf16x2 registers in natural K order: out[j] = (2j, 2j+1).

// Q4_0: exact, d = d_hi + d_lo split (see gemv.cuh); the 16 code bytes of one block.
BQ_DEVINL void deq_q4_0_half(uint4 raw, uint32_t dhi2, uint32_t dlo2, uint32_t (&out)[16])
{
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const uint32_t t = prmt(words[w], 0u, p ? 0x4342u : 0x4140u);   // [b, 0, b', 0]
            const uint32_t l = hsub2_bf16_i<0x43084308u>(and_or_i<0x000F000Fu, 0x43004300u>(t));
            const uint32_t u = hsub2_bf16_i<0x43084308u>(and_or_i<0x000F000Fu, 0x43004300u>(t >> 4));
            out[2 * w + p] = hfma2_bf16(l, dhi2, hmul2_bf16(l, dlo2));        // elements 4w+2p, +1
            out[8 + 2 * w + p] = hfma2_bf16(u, dhi2, hmul2_bf16(u, dlo2));    // elements 16+4w+2p, +1
        }
    }
}

// Affine 4-bit: 4 words of sequential nibbles; w = fma.rn.bf16x2(q, scale, bias).
BQ_DEVINL void deq_aff4_half(uint4 raw, uint32_t s2, uint32_t b2, uint32_t (&out)[16])
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
        out[4 * i + 0] = prmt(v[0], v[1], 0x5410u);
        out[4 * i + 1] = prmt(v[2], v[3], 0x5410u);
        out[4 * i + 2] = prmt(v[0], v[1], 0x7632u);
        out[4 * i + 3] = prmt(v[2], v[3], 0x7632u);
    }
}

// Affine 8-bit: 8 words of bytes; w = bf16_rne(fmaf(scale, q, bias)), two
// weights per packed fp32x2 subtract and FMA.
BQ_DEVINL void deq_aff8_half(uint4 raw0, uint4 raw1, float s, float b, uint32_t (&out)[16])
{
    const uint32_t words[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
    const uint64_t s2 = f32x2_splat(s), b2 = f32x2_splat(b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        out[2 * i] = deq_aff8_pair<0>(words[i], s2, b2);
        out[2 * i + 1] = deq_aff8_pair<2>(words[i], s2, b2);
    }
}

struct DeqScale { uint32_t a, b; };

// Eight consecutive groups' scales (and biases) of one weight row: one 16-byte
// vector each.  A window spans group_size / 8 k-blocks (4 for group 32, 8 for 64,
// 16 for 128).
struct ScaleWindow {
    uint4 s, b;
};

BQ_DEVINL uint32_t halfword(const uint4& v, int k)
{
    const uint32_t w = (k < 2) ? v.x : (k < 4) ? v.y : (k < 6) ? v.z : v.w;
    return (w >> (16 * (k & 1))) & 0xFFFFu;
}

// Window `win` (groups 8 win .. 8 win + 7) of weight row `row`; zeros past the
// row's end and for rows past N.  With vec_scales every row is 16-byte aligned
// and holds whole windows, so one vector load per array suffices.
template <int MODE>
BQ_DEVINL ScaleWindow load_scale_window(const TcParams& p, int row, int win)
{
    ScaleWindow w;
    w.s = w.b = make_uint4(0, 0, 0, 0);
    const int per_row = p.K >> p.gs_shift;
    const int first = win * 8;
    if (row >= p.N || first >= per_row) return w;
    const uint16_t* srow = p.scales + (int64_t)row * per_row + first;
    const uint16_t* brow = p.biases + (int64_t)row * per_row + first;
    if (p.vec_scales) {
        w.s = __ldg(reinterpret_cast<const uint4*>(srow));
        if constexpr (MODE != kModeQ4_0) w.b = __ldg(reinterpret_cast<const uint4*>(brow));
    } else {
        uint32_t sv[8], bv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const bool in = first + k < per_row;
            sv[k] = in ? __ldg(srow + k) : 0u;
            bv[k] = (MODE != kModeQ4_0 && in) ? __ldg(brow + k) : 0u;
        }
        w.s = make_uint4(sv[0] | sv[1] << 16, sv[2] | sv[3] << 16, sv[4] | sv[5] << 16, sv[6] | sv[7] << 16);
        w.b = make_uint4(bv[0] | bv[1] << 16, bv[2] | bv[3] << 16, bv[4] | bv[5] << 16, bv[6] | bv[7] << 16);
    }
    return w;
}

// The packed bf16x2 operands of one 32-element half's dequantization from group
// k of a window.  Q4_0: d splits exactly into d_hi = bf16(d) and d_lo = d - d_hi
// (both representable in bf16), so that fma(q - 8, d_hi, (q - 8) * d_lo) rounds
// once to bf16((q - 8) * d).  Affine: the bf16 scale and bias bits.
template <int MODE>
BQ_DEVINL DeqScale window_scale(const ScaleWindow& w, int k)
{
    DeqScale r;
    if constexpr (MODE == kModeQ4_0) {
        const float d = f16_bits_to_f32(halfword(w.s, k));
        r.a = pack_bf16x2_rn(d, d);                                            // d_hi
        const float lo = __fsub_rn(d, __uint_as_float(r.a << 16));           // d - d_hi, exact
        r.b = pack_bf16x2_rn(lo, lo);
    } else {
        r.a = halfword(w.s, k);
        r.b = halfword(w.b, k);
    }
    return r;
}

// ONE_ACC: one TMEM accumulator (p.num_acc == 1), the next tile waiting for
// each drain; otherwise two, the drain overlapping the next tile.  A template
// argument, so that each kernel carries only its own epilogue.
template <int MODE, bool ONE_ACC>
__global__ void __launch_bounds__(TcCfg<MODE>::kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a, TcParams p)
{
    using C = TcCfg<MODE>;
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = (p.K + 63) / 64;
    const int S = p.stages;
    const uint32_t b_bytes = (uint32_t)p.bn * 128u;

    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t b_base = base;                                      // activation tiles (1024-aligned)
    const uint32_t a_base = b_base + (uint32_t)S * b_bytes;            // bf16 weight tiles (kModeBF16)
    const uint32_t c_base = a_base + (uint32_t)S * C::kABytes;         // packed code tiles (fused)
    const uint32_t bar_base = c_base + (uint32_t)S * C::kCBytes;
    // barriers per stage: landed (TMA), weight tile written (fused), free (MMA done);
    // per accumulator: ready, drained; and MMA done
    auto full_bar = [&](int s) { return bar_base + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (uint32_t)(S + s); };
    auto afull_bar = [&](int s) { return bar_base + 8u * (uint32_t)(2 * S + s); };
    auto tfull_bar = [&](int b) { return bar_base + 8u * (uint32_t)(3 * S + b); };      // accumulator b ready
    auto tempty_bar = [&](int b) { return bar_base + 8u * (uint32_t)(3 * S + 2 + b); };  // accumulator b drained
    const uint32_t mma_done_bar = bar_base + 8u * (uint32_t)(3 * S + 4);
    // TMEM columns: accumulators at 0 (and acc_stride); fused modes keep stage s of
    // the dequantized weight tile (128 lanes x 64 bf16 = 32 columns) after them.
    constexpr int kNumAcc = ONE_ACC ? 1 : 2;
    auto a_tmem_col = [&](int s) { return (uint32_t)(kNumAcc * p.acc_stride) + 32u * (uint32_t)s; };
    // Accumulator of the lt-th local tile and the parity of its use count.
    auto acc_of = [&](int lt) { return ONE_ACC ? 0 : (lt & 1); };
    auto acc_phase = [&](int lt) { return (uint32_t)(ONE_ACC ? lt : (lt >> 1)) & 1u; };
    const uint32_t tmem_slot = mma_done_bar + 8u;
    uint8_t* smem_gen = smem_raw + (base - smem_u32(smem_raw));
    volatile uint32_t* tmem_slot_ptr = reinterpret_cast<volatile uint32_t*>(smem_gen + (tmem_slot - base));
    auto tile_n0 = [&](int t) { return (t / p.m_tiles) * 128; };
    auto tile_m0 = [&](int t) { return (t % p.m_tiles) * p.bn; };
    // Work units: units [0, dp_tiles) are whole tiles.  Each later tile t is split
    // over K into p.splits units; unit dp_tiles + (t - dp_tiles) * splits + s takes
    // the k-blocks [kb_begin, kb_end) of split s.  With dp_tiles a whole number of
    // rounds of the grid, the split tiles fill the last round (dp_tiles == 0: every
    // tile is split; splits == 1: every tile is whole).
    const int units = p.dp_tiles + (p.tiles - p.dp_tiles) * p.splits;
    auto unit_tile = [&](int u) { return u < p.dp_tiles ? u : p.dp_tiles + (u - p.dp_tiles) / p.splits; };
    auto unit_split = [&](int u) { return u < p.dp_tiles ? 0 : (u - p.dp_tiles) % p.splits; };
    // (nk < 2^24 and splits <= 8: the products fit 32-bit arithmetic)
    auto kb_begin = [&](int u) { return u < p.dp_tiles ? 0 : unit_split(u) * nk / p.splits; };
    auto kb_end = [&](int u) { return u < p.dp_tiles ? nk : (unit_split(u) + 1) * nk / p.splits; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
            mbar_init(afull_bar(s), C::kDeqWarpsPerGroup);   // one group of dequant warps per k-block
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 128);
        }
        mbar_init(mma_done_bar, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(tmem_slot, 512u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot_ptr;

    if (warp == C::kTmaWarp) {
        // ---------------- producer ----------------
        // One lane runs the whole schedule; the stage index and phase advance
        // incrementally (no division in the loop).
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_a);
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const int t = unit_tile(u);
                const int n0 = tile_n0(t), m0 = tile_m0(t);
                const int kb1 = kb_end(u);
                for (int it = kb_begin(u); it < kb1; ++it) {
                    if (!mbar_wait(empty_bar(s), ph ^ 1u)) { ok = false; break; }
                    mbar_arrive_expect_tx(full_bar(s), b_bytes + (MODE == kModeBF16 ? C::kABytes : C::kCBytes));
                    tma_load_2d(b_base + (uint32_t)s * b_bytes, &tm_x, full_bar(s), it * 64, m0);
                    if constexpr (MODE == kModeBF16)
                        tma_load_2d(a_base + (uint32_t)s * C::kABytes, &tm_a, full_bar(s), it * 64, n0);
                    else
                        tma_load_2d(c_base + (uint32_t)s * C::kCBytes, &tm_a, full_bar(s), it * C::kCodeBytesPerRow, n0);
                    ++issued;
                    if (++s == S) { s = 0; ph ^= 1u; }
                }
            }
            // Drain: every issued copy has landed before this CTA may exit.  Walk the
            // last min(issued, S) stages backwards from the next stage to be used.
            for (int q = 0; q < S && q < issued; ++q) {
                if (--s < 0) { s = S - 1; ph ^= 1u; }
                mbar_wait(full_bar(s), ph);
            }
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ---------------- MMA issuer ----------------
        // One lane issues everything; its per-k-block path is kept short because
        // it shares an issue slot scheduler with busy dequant warps.  Descriptor
        // words, the A column and the barrier addresses of the current stage
        // advance incrementally.  Fused modes wait only for the dequant group's
        // barrier: the group arrives after it has itself waited for the stage's
        // TMA, so the activation tile has landed too.
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16_f32(128, p.bn);
            const uint64_t bd0 = umma_desc_k_sw128(b_base);
            const uint32_t b_lo0 = (uint32_t)bd0, desc_hi = (uint32_t)(bd0 >> 32);
            const uint32_t b_step = b_bytes >> 4;
            const uint32_t a_lo0 = (uint32_t)umma_desc_k_sw128(a_base);          // kModeBF16
            const uint32_t a_col0 = tmem_base + a_tmem_col(0);                    // fused modes
            const uint32_t a_step = (MODE == kModeBF16) ? (C::kABytes >> 4) : 32u;
            const uint32_t wait_off = 8u * (uint32_t)((MODE == kModeBF16) ? 0 : 2 * S);   // full / afull
            const uint32_t empty_off = 8u * (uint32_t)S;
            uint32_t b_lo = b_lo0, a_cur = (MODE == kModeBF16) ? a_lo0 : a_col0, bar_s = bar_base;
            int s = 0, lt = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++lt) {
                const int acc = acc_of(lt);
                const int kb0 = kb_begin(u), kb1 = kb_end(u);
                if (!mbar_wait(tempty_bar(acc), acc_phase(lt) ^ 1u)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.acc_stride);
                uint32_t accumulate = 0;
                for (int it = kb0; it < kb1; ++it) {
                    if (!mbar_wait(bar_s + wait_off, ph)) { ok = false; break; }
                    tc_fence_after();
                    if constexpr (MODE == kModeBF16)
                        umma_kblock_ss(d_tmem, a_cur, b_lo, desc_hi, idesc, accumulate);
                    else
                        umma_kblock_ts(d_tmem, a_cur, b_lo, desc_hi, idesc, accumulate);
                    accumulate = 1;
                    umma_commit(bar_s + empty_off);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                        b_lo = b_lo0;
                        a_cur = (MODE == kModeBF16) ? a_lo0 : a_col0;
                        bar_s = bar_base;
                    } else {
                        b_lo += b_step;
                        a_cur += a_step;
                        bar_s += 8u;
                    }
                }
                umma_commit(tfull_bar(acc));
            }
            umma_commit(mma_done_bar);   // nothing stays in flight past this point
            mbar_wait(mma_done_bar, 0);
        }
        __syncwarp();
    } else if (warp >= C::kEpiWarp0 && warp < C::kEpiWarp0 + 4) {
        // ---------------- epilogue ----------------
        const int q4 = warp & 3;                                       // TMEM lane quarter
        int lt = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++lt) {
            const int t = unit_tile(u);
            const int acc = acc_of(lt);
            if (!mbar_wait_warp(tfull_bar(acc), acc_phase(lt))) break;
            tc_fence_after();
            const int row = tile_n0(t) + 32 * q4 + lane;
            const int m0 = tile_m0(t);
            // a split unit's partial tile: [token of the tile][weight row of the tile]
            float* part = (p.splits > 1 && u >= p.dp_tiles)
                              ? p.ws + ((int64_t)unit_split(u) * (p.tiles - p.dp_tiles) + (t - p.dp_tiles)) *
                                           ((int64_t)p.bn * 128) + 32 * q4 + lane
                              : nullptr;
            const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * q4) << 16) + (uint32_t)(acc * p.acc_stride);
            // 16 columns (tokens) per TMEM load; the next load is in flight while
            // this chunk is converted and stored (wait::ld waits for all loads).
            auto drain = [&](auto&& store16) {
                uint32_t va[16], vb[16];
                tmem_ld_32x32b_x16(lane_addr, va);
                for (int c0 = 0; c0 < p.bn; c0 += 32) {
                    tmem_wait_ld();
                    const bool more = c0 + 16 < p.bn;
                    if (more) tmem_ld_32x32b_x16(lane_addr + (uint32_t)(c0 + 16), vb);
                    store16(va, m0 + c0);
                    if (!more) break;
                    tmem_wait_ld();
                    if (c0 + 32 < p.bn) tmem_ld_32x32b_x16(lane_addr + (uint32_t)(c0 + 32), va);
                    store16(vb, m0 + c0 + 16);
                }
                tmem_wait_ld();
            };
            // The branch is warp-uniform (part is per unit): the TMEM loads are
            // warp-collective, so every lane takes part; lanes past N only skip stores.
            const bool row_ok = row < p.N;
            if (part) {                                               // K split: fp32 partial sums
                // every token and row of the tile (the reduce skips those past M and N);
                // a warp's 32 rows of one token are one 128-byte line
                drain([&](const uint32_t (&v)[16], int mb) {
                    float* pt = part + (int64_t)(mb - m0) * 128;
#pragma unroll
                    for (int j = 0; j < 16; ++j) pt[j * 128] = __uint_as_float(v[j]);
                });
            } else if constexpr (ONE_ACC) {
                // One accumulator: the next tile waits for this drain, so it is kept
                // short -- two tokens per conversion, and a whole 16-token chunk
                // (the warp-uniform common case) stores without per-token checks.
                // (With two accumulators the drain overlaps the next tile, and the
                // per-token form below, which issues its stores more evenly,
                // measured faster.)
                const uint64_t ld_bytes = (uint64_t)p.N * 2u;
                drain([&](const uint32_t (&v)[16], int mb) {
                    if (!row_ok) return;
                    uint16_t* py = p.y + (int64_t)mb * p.N + row;
                    if (mb + 16 <= p.M) {
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            const uint32_t pk = pack_bf16x2_rn(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                            char* a = reinterpret_cast<char*>(py) + (uint64_t)j * ld_bytes;
                            *reinterpret_cast<uint16_t*>(a) = (uint16_t)(pk & 0xFFFFu);
                            *reinterpret_cast<uint16_t*>(a + ld_bytes) = (uint16_t)(pk >> 16);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (mb + j < p.M)
                                py[(int64_t)j * p.N] = (uint16_t)f32_to_bf16_bits(__uint_as_float(v[j]));
                    }
                });
            } else {
                drain([&](const uint32_t (&v)[16], int mb) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (row_ok && mb + j < p.M)
                            p.y[(int64_t)(mb + j) * p.N + row] = (uint16_t)f32_to_bf16_bits(__uint_as_float(v[j]));
                });
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
        }
    } else if (MODE != kModeBF16 && warp < C::kDeqWarps) {
        // ---------------- dequantization ----------------
        // Group grp takes the k-blocks whose position in this CTA's sequence (all
        // k-blocks of all its units, in order) is grp modulo the number of
        // groups; a warp walks only those, with a cursor over (unit, k-block).
        // Scales come in 8-group windows (one 16-byte load per array); the window
        // the group needs next is always in flight.
        constexpr int G = C::kDeqGroups;
        constexpr int kHalves = 8 / C::kDeqWarpsPerGroup;   // 32-element halves of a k-block per thread
        const int r = 32 * (warp & 3) + lane;                // weight row within the tile = TMEM lane
        const int h0 = (C::kDeqWarpsPerGroup == 8) ? ((warp >> 2) & 1) : 0;
        const int grp = warp / C::kDeqWarpsPerGroup;
        const int span_shift = p.gs_shift - 3;               // log2(k-blocks per window)
        const uint32_t lane_base = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16);
        struct Cur { int u, it, kb1, row; };                  // row: this thread's weight row in the unit's tile
        auto cur_at = [&](int u) {
            return u < units ? Cur{u, kb_begin(u), kb_end(u), tile_n0(unit_tile(u)) + r} : Cur{units, 0, 0, p.N};
        };
        auto step = [&](Cur c, int n) {                      // n positions further along the sequence
            c.it += n;
            while (c.u < units && c.it >= c.kb1) {
                const int carry = c.it - c.kb1;
                c = cur_at(c.u + (int)gridDim.x);
                c.it += carry;
            }
            return c;
        };
        Cur cur = step(cur_at(blockIdx.x), grp);            // first own k-block: position grp
        // Window in use (cu, cw) and the one in flight (nu, nw).
        int cu = -1, cw = -1, nu = cur.u, nw = cur.it >> span_shift;
        ScaleWindow win_cur, win_nxt = load_scale_window<MODE>(p, cur.row, nw);
        win_cur = win_nxt;
        int s = grp % S;
        uint32_t ph = (uint32_t)(grp / S) & 1u;
        bool ok = true;
        while (ok && cur.u < units) {
            const int w = cur.it >> span_shift;
            if (cur.u != cu || w != cw) {                    // entering a new window
                win_cur = (cur.u == nu && w == nw) ? win_nxt : load_scale_window<MODE>(p, cur.row, w);
                cu = cur.u;
                cw = w;
                Cur c = step(cur, G);                        // the group's first k-block past this window
                while (c.u == cu && (c.it >> span_shift) == cw) c = step(c, G);
                nu = c.u;
                nw = c.it >> span_shift;
                win_nxt = load_scale_window<MODE>(p, c.row, nw);   // rows past N / units past the end: zeros
            }
            if (!mbar_wait_warp(full_bar(s), ph)) { ok = false; break; }
            const uint32_t codes = c_base + (uint32_t)s * C::kCBytes + (uint32_t)(r * C::kCodeBytesPerRow);
#pragma unroll
            for (int hh = 0; hh < kHalves; ++hh) {
                const int h = h0 + hh;
                const DeqScale e = window_scale<MODE>(win_cur, ((cur.it * 64 + 32 * h) >> p.gs_shift) & 7);
                uint32_t wv[16];
                if constexpr (MODE == kModeQ4_0) {
                    deq_q4_0_half(ld_shared_v4(codes + 16u * h), e.a, e.b, wv);
                } else if constexpr (MODE == kModeAff4) {
                    deq_aff4_half(ld_shared_v4(codes + 16u * h), e.a | (e.a << 16), e.b | (e.b << 16), wv);
                } else {
                    deq_aff8_half(ld_shared_v4(codes + 32u * h), ld_shared_v4(codes + 32u * h + 16u),
                                  bf16_bits_to_f32(e.a), bf16_bits_to_f32(e.b), wv);
                }
                // These 32 weights = 16 TMEM columns of lane r in stage s.  The
                // stage's previous tile was consumed by the MMA S k-blocks back:
                // its smem stage was freed before this one was filled.
                tmem_st_32x32b_x16(lane_base + a_tmem_col(s) + 16u * h, wv);
            }
            cur = step(cur, G);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull_bar(s));
            s += G;
            if (s >= S) { s -= S; ph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::kMmaWarp) tmem_dealloc(tmem_base, 512u);
}

}  // namespace bq
