// gemv_stream.cuh -- decode path for 1..8 tokens: the packed weights stream
// once from HBM into per-warp shared-memory rings (16-byte asynchronous
// copies), and warp-level bf16 MMAs multiply the exact integer codes against
// the activations; each block's (or group's) scale is applied once to its fp32
// partial sum.
//
// The pages' decode kernels are prior art for this path: decode routes to a
// vector-dot kernel in "et-backend: Q4_0 matrix-engine GEMM rewrite for
// prefill" (Overview), and the SYCL page "2026-05-06 Q4 sync-after focused
// repro" runs MMVQ kernels over "reordered" Q4_0 (Important source touch
// points).  The operation is the MLX issue's quantized_matmul ("Repro"): y =
// x . dequant(W)^T, which is
//
//   y[m][n] = sum over blocks b of  d[n][b] * sum_{j in b} x[m][j] * (q[n][j] - 8)      (Q4_0)
//   y[m][n] = sum over groups g of  s[n][g] * sum_{j in g} x[m][j] * q[n][j]
//                                 + z[n][g] * sum_{j in g} x[m][j]                  (affine)
//
// computed in that order: the inner sums exactly in the tensor core (codes
// and activations are exact bf16, products exact, fp32 accumulation), the
// scale once per block.  The result differs from a product with the
// bf16-rounded dequantized weights only by those weights' roundings.
//
// Codes enter the MMA without arithmetic: OR-ing a nibble into the bf16
// pattern 0x4300 gives the value 128 + q exactly, so one LOP3 (plus a shift)
// turns two nibbles into an A-operand register.  The constant 128 (and Q4_0's
// -8) is removed through the activation sums: for Q4_0 the accumulator starts
// at C = -136 * sum_j x[j] (MMA addend), so it ends at sum_j x[j] (q[j] - 8).
// 8-bit codes are split into nibbles q = lo + 16 hi; the high nibbles multiply
// 16 x (exact in bf16), and the offset is 128 + 16 * 128 = 2176.
//
// Layout of the work: one CTA per SM walks a contiguous range of 16-row
// weight tiles (of one matrix, or of up to eight matrices that share x, as the
// fused pairs of one-token MMVQ nodes on the SYCL page; a tile is computed the
// same way whichever launch it is in, so the bits do not depend on it).  Each
// of the CTA's KW warps owns a fixed K slice of every tile and streams exactly
// that slice (codes and scales of its 16 rows) into its own ring of S stages
// with cp.async, so no warp waits for another and no registers hold data in
// flight.  Rows are padded by 16 bytes so that ldmatrix reads them without
// bank conflicts; ldmatrix hands each thread the 4-byte word of a 16-byte code
// unit that its MMA fragment needs.  The activations are staged once per CTA
// into a table permuted to the fragment order.  Per-warp partial sums of each
// tile are summed in warp order at the end, so the result is deterministic.
//
// Launch: with programmatic stream serialization the kernel's set-up overlaps
// the previous kernel; every global read of the data and every write of y
// happen after griddepcontrol.wait.
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

// D = A x B + C, m16n8k16, fp16 inputs, fp32 accumulate (a pure function of its operands).
BQ_DEVINL void mma_f16_16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                               uint32_t b1, float c0, float c1, float c2, float c3)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
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

// Right shift by 8 on the FMA pipe: the high word of w * 2^24.  The multiplier
// comes from the launch parameters, so the compiler cannot turn it back into a
// shift (which would load the ALU pipe that the LOP3s of the unpack need).
BQ_DEVINL uint32_t shr8_fma(uint32_t w, uint32_t mul24) { return __umulhi(w, mul24); }

// ------------------------------------------------------------------ formats
// The codes enter the MMA as exact fp16 values, made by OR-ing them into fp16
// patterns: a nibble in bits 0-3 under 0x6400 is 1024 + q, a nibble in bits
// 4-7 under 0x5400 is 64 + q (exponent 6, 1/16 per mantissa step), a byte
// under 0x64 (by a byte permute) is 1024 + q.  A 16-byte code unit of one row
// holds E elements; ldmatrix gives thread t of a quad word t of the unit.
//   Q4_0 (byte j: element j low nibble, j + 16 high): word t = bytes 4t..4t+3,
//     r0 = 1024 + (4t, 4t+2)  r1 = 1024 + (4t+1, 4t+3)  r2 = 64 + (16+4t, 18+4t)  r3 = 64 + (17+4t, 19+4t)
//   affine 4-bit (word i: elements 8i..8i+7, nibble n = element 8i+n)
//     r0 = 1024 + (8t, 8t+4)  r1 = 64 + (8t+1, 8t+5)  r2 = 1024 + (8t+2, 8t+6)  r3 = 64 + (8t+3, 8t+7)
//   affine 8-bit (word i: elements 4i..4i+3, one byte each)
//     r0 = 1024 + (4t, 4t+2)  r1 = 1024 + (4t+1, 4t+3)
// An MMA takes (r0, r1) as k-slots (2t, 2t+1) and (2t+8, 2t+9), a second one
// (r2, r3); the activation table holds the matching fp16 pairs.  The offsets
// (1024 or 64 per element) come out through per-unit activation sums.
template <Fmt F> struct SFmt;
template <> struct SFmt<Fmt::Q4_0> { static constexpr int E = 32, kBits = 4, kMmas = 2; };
template <> struct SFmt<Fmt::AFF4> { static constexpr int E = 32, kBits = 4, kMmas = 2; };
template <> struct SFmt<Fmt::AFF8> { static constexpr int E = 16, kBits = 8, kMmas = 1; };

template <Fmt F>
BQ_DEVINL void unpack_unit_word(uint32_t w, uint32_t (&r)[4], uint32_t mul24)
{
    if constexpr (F == Fmt::AFF8) {
        r[0] = prmt(w, 0x64646464u, 0x4240u);
        r[1] = prmt(w, 0x64646464u, 0x4341u);
    } else {
        const uint32_t w8 = shr8_fma(w, mul24);
        if constexpr (F == Fmt::Q4_0) {
            r[0] = and_or_i<0x000F000Fu, 0x64006400u>(w);
            r[1] = and_or_i<0x000F000Fu, 0x64006400u>(w8);
            r[2] = and_or_i<0x00F000F0u, 0x54005400u>(w);
            r[3] = and_or_i<0x00F000F0u, 0x54005400u>(w8);
        } else {
            r[0] = and_or_i<0x000F000Fu, 0x64006400u>(w);
            r[1] = and_or_i<0x00F000F0u, 0x54005400u>(w);
            r[2] = and_or_i<0x000F000Fu, 0x64006400u>(w8);
            r[3] = and_or_i<0x00F000F0u, 0x54005400u>(w8);
        }
    }
}

// ------------------------------------------------------------------ parameters
constexpr int kSgMaxTokens = 8;      // one n8 MMA column group
constexpr int kSgMaxMats = 8;        // matrices sharing x in one launch

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
    uint32_t x_row_bytes;     // activation table bytes per token (units x 4 entries + 64)
    uint32_t mul24;           // 2^24 (see shr8_fma)
    int red_cols;             // token columns of the partial-sum buffer (M rounded up to even)
    uint32_t off_x, off_c, off_red, off_ring;   // offsets into dynamic shared memory
};

// Activation-table entry bytes per (unit, quad position): the B registers of the unit's MMAs.
template <Fmt F> constexpr int sg_entry_bytes() { return F == Fmt::AFF8 ? 8 : 16; }
// C-table bytes per (group, token): Q4_0 the MMA addend C; affine (S, -T).
template <Fmt F> constexpr int sg_ctab_bytes() { return F == Fmt::Q4_0 ? 4 : 8; }

// ------------------------------------------------------------------ kernel pieces
// The MMAs of one warp's K slice of one stage, NU code units (compile-time
// count, fully unrolled) or nu_rt units (NU == 0).  ld: ldmatrix address of the
// slice's first unit pair; sc: this thread's row-g scale run (row g + 8 is
// 8 * pitch further, biases 16 rows further); xp: the slice's first
// activation-table entry of this thread; cp: its first C-table pair.
template <Fmt F, int GS, int NU>
BQ_DEVINL void slice_mma(float (&yv)[4], uint32_t ld, const uint8_t* sc, uint32_t pitch, const uint8_t* xp,
                         const uint8_t* cp, int nu_rt, uint32_t mul24)
{
    using T = SFmt<F>;
    constexpr int UPG = GS / T::E;
    constexpr int XU = 4 * sg_entry_bytes<F>();               // activation-table bytes per unit
    constexpr int CG = kSgMaxTokens * sg_ctab_bytes<F>();     // C-table bytes per group
    const int nu = NU > 0 ? NU : nu_rt;
    if constexpr (UPG == 1) {
        // Q4_0 or affine 4-bit with groups of 32: two groups per ldmatrix.x4
#pragma unroll (NU > 0 ? NU / 2 : 2)
        for (int s = 0; s < nu / 2; ++s) {
            uint32_t w[4];                                      // (g, u) (g+8, u) (g, u+1) (g+8, u+1)
            ldsm_x4(ld + (uint32_t)s * 32u, w[0], w[1], w[2], w[3]);
            const uint32_t sg = lds32(sc + 4 * s), sg8 = lds32(sc + 8 * pitch + 4 * s);
            [[maybe_unused]] uint32_t bg = 0u, bg8 = 0u;
            if constexpr (F != Fmt::Q4_0) {
                bg = lds32(sc + 16 * pitch + 4 * s);
                bg8 = lds32(sc + 24 * pitch + 4 * s);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t ra[4], rb[4];
                unpack_unit_word<F>(w[2 * h], ra, mul24);
                unpack_unit_word<F>(w[2 * h + 1], rb, mul24);
                const int u = 2 * s + h;
                const uint4 e = *reinterpret_cast<const uint4*>(xp + u * XU);
                float acc[4];
                if constexpr (F == Fmt::Q4_0) {
                    const float2 c = *reinterpret_cast<const float2*>(cp + u * CG);
                    mma_f16_16816_c(acc, ra[0], rb[0], ra[1], rb[1], e.x, e.y, c.x, c.y, c.x, c.y);
                    mma_f16_16816_c(acc, ra[2], rb[2], ra[3], rb[3], e.z, e.w, acc[0], acc[1], acc[2], acc[3]);
                    const float2 d2 = __half22float2(*reinterpret_cast<const __half2*>(&sg));
                    const float2 d28 = __half22float2(*reinterpret_cast<const __half2*>(&sg8));
                    const float dg = h ? d2.y : d2.x, dg8 = h ? d28.y : d28.x;
                    yv[0] = __fmaf_rn(dg, acc[0], yv[0]);
                    yv[1] = __fmaf_rn(dg, acc[1], yv[1]);
                    yv[2] = __fmaf_rn(dg8, acc[2], yv[2]);
                    yv[3] = __fmaf_rn(dg8, acc[3], yv[3]);
                } else {
                    const float4 c = *reinterpret_cast<const float4*>(cp + u * CG);   // (S, -T) of tokens 2t, 2t+1
                    mma_f16_16816_c(acc, ra[0], rb[0], ra[1], rb[1], e.x, e.y, c.y, c.w, c.y, c.w);
                    mma_f16_16816_c(acc, ra[2], rb[2], ra[3], rb[3], e.z, e.w, acc[0], acc[1], acc[2], acc[3]);
                    const float dg = __uint_as_float(h ? sg & 0xFFFF0000u : sg << 16);
                    const float dg8 = __uint_as_float(h ? sg8 & 0xFFFF0000u : sg8 << 16);
                    const float zg = __uint_as_float(h ? bg & 0xFFFF0000u : bg << 16);
                    const float zg8 = __uint_as_float(h ? bg8 & 0xFFFF0000u : bg8 << 16);
                    yv[0] = __fmaf_rn(dg, acc[0], __fmaf_rn(zg, c.x, yv[0]));
                    yv[1] = __fmaf_rn(dg, acc[1], __fmaf_rn(zg, c.z, yv[1]));
                    yv[2] = __fmaf_rn(dg8, acc[2], __fmaf_rn(zg8, c.x, yv[2]));
                    yv[3] = __fmaf_rn(dg8, acc[3], __fmaf_rn(zg8, c.z, yv[3]));
                }
            }
        }
    } else {
        // affine, one group of UPG >= 2 units per atom, every unit into the group's accumulator
#pragma unroll (NU > 0 ? NU / UPG : 1)
        for (int a = 0; a < nu / UPG; ++a) {
            const float4 c = *reinterpret_cast<const float4*>(cp + a * CG);   // (S, -T) of tokens 2t, 2t+1
            float gacc[4] = {c.y, c.w, c.y, c.w};
#pragma unroll
            for (int s = 0; s < UPG / 2; ++s) {
                const int u = a * UPG + 2 * s;
                uint32_t w[4];
                ldsm_x4(ld + (uint32_t)u * 16u, w[0], w[1], w[2], w[3]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t ra[4], rb[4];
                    unpack_unit_word<F>(w[2 * h], ra, mul24);
                    unpack_unit_word<F>(w[2 * h + 1], rb, mul24);
                    if constexpr (F == Fmt::AFF8) {
                        const uint2 e = *reinterpret_cast<const uint2*>(xp + (u + h) * XU);
                        mma_f16_16816_c(gacc, ra[0], rb[0], ra[1], rb[1], e.x, e.y, gacc[0], gacc[1], gacc[2],
                                        gacc[3]);
                    } else {
                        const uint4 e = *reinterpret_cast<const uint4*>(xp + (u + h) * XU);
                        mma_f16_16816_c(gacc, ra[0], rb[0], ra[1], rb[1], e.x, e.y, gacc[0], gacc[1], gacc[2],
                                        gacc[3]);
                        mma_f16_16816_c(gacc, ra[2], rb[2], ra[3], rb[3], e.z, e.w, gacc[0], gacc[1], gacc[2],
                                        gacc[3]);
                    }
                }
            }
            // group epilogue: y += s * acc + z * S
            const float dg = bf16_bits_to_f32(lds16(sc + 2 * a));
            const float dg8 = bf16_bits_to_f32(lds16(sc + 8 * pitch + 2 * a));
            const float zg = bf16_bits_to_f32(lds16(sc + 16 * pitch + 2 * a));
            const float zg8 = bf16_bits_to_f32(lds16(sc + 24 * pitch + 2 * a));
            yv[0] = __fmaf_rn(dg, gacc[0], __fmaf_rn(zg, c.x, yv[0]));
            yv[1] = __fmaf_rn(dg, gacc[1], __fmaf_rn(zg, c.z, yv[1]));
            yv[2] = __fmaf_rn(dg8, gacc[2], __fmaf_rn(zg8, c.x, yv[2]));
            yv[3] = __fmaf_rn(dg8, gacc[3], __fmaf_rn(zg8, c.z, yv[3]));
        }
    }
}

// Scaled fp16 pair of two bf16 activations (lo and hi halves of v), and the
// sum of the two fp16 values as the MMA sees them.
BQ_DEVINL uint32_t x_pair_f16(uint32_t lo_bits, uint32_t hi_bits, float scale, float& sum)
{
    const __half2 h = __floats2half2_rn(bf16_bits_to_f32(lo_bits) * scale, bf16_bits_to_f32(hi_bits) * scale);
    const float2 f = __half22float2(h);
    sum += f.x + f.y;
    return *reinterpret_cast<const uint32_t*>(&h);
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
    constexpr int XE = sg_entry_bytes<F>();
    constexpr int CB = sg_ctab_bytes<F>();
    static_assert(GS % E == 0, "group must hold whole code units");

    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float x_scale[kSgMaxTokens], x_unscale[kSgMaxTokens], warp_max[32][kSgMaxTokens];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    const int M = p.M, K = p.K, S = p.stages, nchunks = p.nchunks;
    const int t_begin = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
    const int t_end = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
    const int nt = t_end - t_begin;
    const int total = nt * nchunks;
    const int64_t row_bytes = (int64_t)K * T::kBits / 8;
    const int64_t srow = K / GS;                         // scale entries per row
    const int nu_all = K / E;                            // code units per row
    const int ng_all = K / GS;
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
    for (int i = 0; i < S - 1; ++i) issue_next(i);

    // ------------------------------------------------------------ activation tables
    // Each token is scaled by a power of two 2^e so that its largest magnitude
    // lies in [2^14, 2^15); the scaled bf16 values are then exact in fp16 (down to
    // 2^-24 of that magnitude), and y is multiplied by 2^-e at the end, exactly.
    const int nthreads = 32 * KW;
    {
        float mx[kSgMaxTokens];
#pragma unroll
        for (int m = 0; m < kSgMaxTokens; ++m) mx[m] = 0.0f;
        const int nv = K / 8;                                           // 16-byte vectors per token
#pragma unroll
        for (int m = 0; m < kSgMaxTokens; ++m) {
            if (m < M) {
                const uint4* xr = reinterpret_cast<const uint4*>(p.x + (int64_t)m * K);
#pragma unroll 4
                for (int i = tid; i < nv; i += nthreads) {
                    const uint4 v = xr[i];
                    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mx[m] = fmaxf(mx[m], fmaxf(fabsf(bf16_bits_to_f32(vv[j] & 0xFFFFu)),
                                                    fabsf(bf16_bits_to_f32(vv[j] >> 16))));
                }
            }
        }
#pragma unroll
        for (int m = 0; m < kSgMaxTokens; ++m) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[m] = fmaxf(mx[m], __shfl_xor_sync(0xFFFFFFFFu, mx[m], o));
            if (lane == 0) warp_max[warp][m] = mx[m];
        }
        __syncthreads();
        if (tid < kSgMaxTokens) {
            float a = 0.0f;
            for (int w = 0; w < KW; ++w) a = fmaxf(a, warp_max[w][tid]);
            // exponent of a (normal range), clamped so that both 2^e and 2^-e are normal fp32
            int e = 0;
            if (a > 0.0f && a < 3.0e38f) {
                const int ea = (int)((__float_as_uint(a) >> 23) & 0xFFu) - 127;
                e = max(-120, min(120, 14 - ea));
            }
            x_scale[tid] = __uint_as_float((uint32_t)(e + 127) << 23);
            x_unscale[tid] = __uint_as_float((uint32_t)(127 - e) << 23);
        }
        __syncthreads();
    }
    // Entry (m, unit u, quad position t): the B registers of the unit's MMAs for
    // token m, in the order unpack_unit_word produces the A registers.
    // U[m][u] = (sum of the class-A elements, sum of the class-B elements) of the
    // unit as fp16 values (class A: the 1024-offset codes, B: the 64-offset ones);
    // then per group the C table: Q4_0 -(1032 A + 72 B), the MMA addend that
    // leaves sum x (q - 8); affine (S, -T) with S = A + B and T = 1024 A + 64 B.
    const uint32_t xtab = sbase + p.off_x;
    float* usum = reinterpret_cast<float*>(smem + p.off_red);
    {
        const int entries = M * nu_all * 4;
#pragma unroll 4
        for (int base = warp * 32; base < entries; base += nthreads) {
            const int idx = base + lane;
            const bool valid = idx < entries;
            const int t = idx & 3, u = (idx >> 2) % nu_all, m = (idx >> 2) / nu_all;
            uint32_t e[4] = {0u, 0u, 0u, 0u};
            float sa = 0.0f, sb = 0.0f;
            if (valid) {
                const float xs = x_scale[m];
                const uint16_t* xr = p.x + (int64_t)m * K + (int64_t)u * E;
                if constexpr (F == Fmt::AFF4) {
                    const uint4 v = *reinterpret_cast<const uint4*>(xr + 8 * t);   // elements 8t .. 8t+7
                    e[0] = x_pair_f16(v.x & 0xFFFFu, v.z & 0xFFFFu, xs, sa);        // (8t, 8t+4)
                    e[1] = x_pair_f16(v.x >> 16, v.z >> 16, xs, sb);                // (8t+1, 8t+5)
                    e[2] = x_pair_f16(v.y & 0xFFFFu, v.w & 0xFFFFu, xs, sa);        // (8t+2, 8t+6)
                    e[3] = x_pair_f16(v.y >> 16, v.w >> 16, xs, sb);                // (8t+3, 8t+7)
                } else {
                    const uint2 a = *reinterpret_cast<const uint2*>(xr + 4 * t);    // elements 4t .. 4t+3
                    e[0] = x_pair_f16(a.x & 0xFFFFu, a.y & 0xFFFFu, xs, sa);        // (4t, 4t+2)
                    e[1] = x_pair_f16(a.x >> 16, a.y >> 16, xs, sa);                // (4t+1, 4t+3)
                    if constexpr (F == Fmt::Q4_0) {
                        const uint2 b = *reinterpret_cast<const uint2*>(xr + 16 + 4 * t);   // 16+4t .. 16+4t+3
                        e[2] = x_pair_f16(b.x & 0xFFFFu, b.y & 0xFFFFu, xs, sb);
                        e[3] = x_pair_f16(b.x >> 16, b.y >> 16, xs, sb);
                    }
                }
                const uint32_t at = xtab + (uint32_t)m * p.x_row_bytes + (uint32_t)(u * 4 + t) * (uint32_t)XE;
                if constexpr (XE == 16)
                    st_shared_v4(at, e[0], e[1], e[2], e[3]);
                else
                    *reinterpret_cast<uint2*>(smem + (at - sbase)) = make_uint2(e[0], e[1]);
            }
            sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
            sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 2);
            sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
            sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 2);
            if (valid && t == 0) *reinterpret_cast<float2*>(usum + 2 * (m * nu_all + u)) = make_float2(sa, sb);
        }
        __syncthreads();
        for (int i = tid; i < ng_all * kSgMaxTokens; i += nthreads) {
            const int gi = i / kSgMaxTokens, m = i % kSgMaxTokens;
            float a = 0.0f, b = 0.0f;
            if (m < M) {
#pragma unroll
                for (int j = 0; j < UPG; ++j) {
                    const float2 v = *reinterpret_cast<const float2*>(usum + 2 * (m * nu_all + gi * UPG + j));
                    a += v.x;
                    b += v.y;
                }
            }
            if constexpr (F == Fmt::Q4_0)
                reinterpret_cast<float*>(smem + p.off_c)[i] = -1032.0f * a - 72.0f * b;
            else
                reinterpret_cast<float2*>(smem + p.off_c)[i] = make_float2(a + b, -(1024.0f * a + 64.0f * b));
        }
        __syncthreads();
    }

    // ------------------------------------------------------------ main loop
    const int g = lane >> 2, t = lane & 3;
    // token column g of the MMA: columns g >= M read token M - 1 (their outputs are never stored)
    const uint8_t* x_lane = smem + p.off_x + (size_t)min(g, M - 1) * p.x_row_bytes + (size_t)t * XE;
    const uint8_t* c_lane = smem + p.off_c + (size_t)(2 * t) * CB;
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
        const uint8_t* xp = x_lane + (size_t)u_b * 4 * XE;
        const uint8_t* cp = c_lane + (size_t)g_b * kSgMaxTokens * CB;
        if (SU > 0 && !(last && nchunks > 1))
            slice_mma<F, GS, SU>(yv, st + ld_lane, sc, p.scale_pitch, xp, cp, SU, p.mul24);
        else
            slice_mma<F, GS, 0>(yv, st + ld_lane, sc, p.scale_pitch, xp, cp, sl.nu, p.mul24);
        if (last && 2 * t < M) {
            float* rp = red + ((tl * KW + warp) * 16 + g) * p.red_cols + 2 * t;
            *reinterpret_cast<float2*>(rp) = make_float2(yv[0], yv[1]);
            *reinterpret_cast<float2*>(rp + 8 * p.red_cols) = make_float2(yv[2], yv[3]);
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
    for (int o = tid; o < M * rows_cta; o += nthreads) {
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
        p.y[mat][(int64_t)m * p.N[mat] + row] = (uint16_t)f32_to_bf16_bits(sum * x_unscale[m]);
    }
}

}  // namespace bq
