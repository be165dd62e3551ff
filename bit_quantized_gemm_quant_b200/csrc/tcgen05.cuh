// tcgen05.cuh -- hand-written inline-PTX wrappers for sm_100a: mbarriers, TMA
// tensor loads, tcgen05 (TMEM allocation, MMA, commit, loads) and the UMMA
// shared-memory / instruction descriptors.
#pragma once

#include <cuda.h>   // CUtensorMap (type only)

#include "common.cuh"

namespace bq {

BQ_DEVINL uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ------------------------------------------------------------------ mbarrier
BQ_DEVINL void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

BQ_DEVINL void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

BQ_DEVINL void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

BQ_DEVINL void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

BQ_DEVINL void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// try_wait with a suspend-time hint: a warp whose phase is not complete sleeps in
// hardware (up to the hint, 10 ms) and is woken when the phase completes, so
// waiting warps do not take issue slots from working ones.
BQ_DEVINL bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 10000000;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait: about one second of clock cycles, then the device error word is
// set and false is returned so the caller can skip its remaining work.
constexpr long long kWaitLimitCycles = 2000000000LL;

BQ_DEVINL bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            raise_device_error(kErrWaitTimeout);
            return false;
        }
    }
    return true;
}

// Warp-level wait: every lane polls.  A poll is one warp instruction either way,
// all lanes see the same phase state from it (so they leave the loop together and
// each lane holds its own acquire), and no result has to be broadcast -- a lane-0
// poll followed by a shuffle measured 6-14% slower in the fused kernel.
BQ_DEVINL bool mbar_wait_warp(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    __syncwarp();
    return ok;
}

BQ_DEVINL uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

BQ_DEVINL void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// ------------------------------------------------------------------ TMA
BQ_DEVINL void tma_prefetch_desc(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2D tiled load (no multicast) into this CTA's shared memory; completes bytes on `bar`.
BQ_DEVINL void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x, int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(map), "r"(bar), "r"(x), "r"(y) : "memory");
}

// 3D tiled load (no multicast) into this CTA's shared memory; completes bytes on `bar`.
BQ_DEVINL void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x, int32_t y, int32_t z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z) : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory (16-byte aligned, a
// multiple of 16 bytes); completes bytes on `bar`.
BQ_DEVINL void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// ------------------------------------------------------------------ tcgen05
BQ_DEVINL void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

BQ_DEVINL void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

BQ_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

BQ_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
BQ_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// One 64-element k-block: four K = 16 MMAs into d_tmem.  The B descriptor of
// sub-step kk is the stage's descriptor with its start address advanced 32 bytes
// (2 in the descriptor's 16-byte units; the 14-bit field never carries).  The
// first MMA accumulates only when `accumulate` is nonzero; the other three always
// do.  A from TMEM (a_tmem: stage column, +8 columns per sub-step) or from shared
// memory (a_lo: the low word of its descriptor, same high word as B).
BQ_DEVINL void umma_kblock_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .b32 l1, l2, l3, a1, a2, a3;\n\t.reg .b64 d0, d1, d2, d3;\n\t"
        "setp.ne.b32 p, %5, 0;\n\tsetp.eq.b32 q, %5, %5;\n\t"
        "add.u32 l1, %2, 2;\n\tadd.u32 l2, %2, 4;\n\tadd.u32 l3, %2, 6;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "mov.b64 d0, {%2, %3};\n\tmov.b64 d1, {l1, %3};\n\tmov.b64 d2, {l2, %3};\n\tmov.b64 d3, {l3, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], d0, %4, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], d1, %4, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], d2, %4, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], d3, %4, q;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate) : "memory");
}

BQ_DEVINL void umma_kblock_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .b32 l1, l2, l3, m1, m2, m3;\n\t.reg .b64 a0, a1, a2, a3, d0, d1, d2, d3;\n\t"
        "setp.ne.b32 p, %5, 0;\n\tsetp.eq.b32 q, %5, %5;\n\t"
        "add.u32 l1, %2, 2;\n\tadd.u32 l2, %2, 4;\n\tadd.u32 l3, %2, 6;\n\t"
        "add.u32 m1, %1, 2;\n\tadd.u32 m2, %1, 4;\n\tadd.u32 m3, %1, 6;\n\t"
        "mov.b64 d0, {%2, %3};\n\tmov.b64 d1, {l1, %3};\n\tmov.b64 d2, {l2, %3};\n\tmov.b64 d3, {l3, %3};\n\t"
        "mov.b64 a0, {%1, %3};\n\tmov.b64 a1, {m1, %3};\n\tmov.b64 a2, {m2, %3};\n\tmov.b64 a3, {m3, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a0, d0, %4, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, d1, %4, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a2, d2, %4, q;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a3, d3, %4, q;\n\t}"
        ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05 ops of this thread complete.
BQ_DEVINL void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 32-bit, 16 consecutive columns: thread i of the warp gets lane
// (warp's lane quarter base + i), columns [col, col + 16).
BQ_DEVINL void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

BQ_DEVINL void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Thread i of the warp writes lane (warp's lane quarter base + i), columns [col, col + 16).
BQ_DEVINL void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

BQ_DEVINL void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// UMMA shared-memory descriptor: K-major operand, 128-byte swizzle, rows of
// 64 bf16 (128 B), 8-row (1024 B) swizzle atoms stacked along M/N.
//   bits  0-13 start address >> 4      bits 16-29 leading byte offset >> 4 (1)
//   bits 32-45 stride byte offset >> 4 (1024 B)   bits 46-47 version = 1
//   bits 49-51 base offset = 0         bits 61-63 layout = 2 (SWIZZLE_128B)
BQ_DEVINL uint64_t umma_desc_k_sw128(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
//   bits 4-5 D format (1 = f32)   bits 7-9 A format (1 = bf16)   bits 10-12 B format (1 = bf16)
//   bit 15 / 16 A / B major (0 = K)   bits 17-22 N >> 3   bits 24-28 M >> 4
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace bq
