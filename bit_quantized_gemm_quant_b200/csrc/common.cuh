// common.cuh -- small device helpers shared by the kernels of libbqgemm.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define BQ_DEVINL __device__ __forceinline__

namespace bq {

// Device error word: a kernel whose bounded wait runs out ORs a code here,
// skips its remaining work and exits.  Read and cleared by bq_device_status().
enum : int { kErrWaitTimeout = 1 };
__device__ int g_device_error = 0;

BQ_DEVINL void raise_device_error(int code) { atomicOr(&g_device_error, code); }

BQ_DEVINL uint32_t bf16_bits(__nv_bfloat16 h) { return (uint32_t)__bfloat16_as_ushort(h); }

// Round-to-nearest-even fp32 -> bf16, returned as raw bits.
BQ_DEVINL uint32_t f32_to_bf16_bits(float f) { return bf16_bits(__float2bfloat16_rn(f)); }

BQ_DEVINL float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

BQ_DEVINL float f16_bits_to_f32(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// Two fp32 -> packed bf16x2 (lo in bits 0..15), each rounded to nearest even.
BQ_DEVINL uint32_t pack_bf16x2_rn(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

BQ_DEVINL uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }

// Packed bf16x2 arithmetic on raw 32-bit registers.  fma.rn.bf16x2 rounds once.
BQ_DEVINL uint32_t hfma2_bf16(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

BQ_DEVINL uint32_t hmul2_bf16(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

BQ_DEVINL uint32_t hsub2_bf16(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Packed fp32x2 arithmetic (sm_100): two independent lanes in one 64-bit
// register, each rounded exactly as the scalar operation (sub.rn.f32x2 lane =
// __fsub_rn, fma.rn.f32x2 lane = __fmaf_rn), so results are bit-identical to
// the scalar forms at half the instruction count.
BQ_DEVINL uint64_t f32x2_pack(uint32_t lo, uint32_t hi)
{
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}

BQ_DEVINL uint64_t f32x2_splat(float v) { return f32x2_pack(__float_as_uint(v), __float_as_uint(v)); }

BQ_DEVINL void f32x2_unpack(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

BQ_DEVINL uint64_t sub_f32x2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

BQ_DEVINL uint64_t add_f32x2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

BQ_DEVINL float f32x2_sum(uint64_t v)
{
    float lo, hi;
    f32x2_unpack(v, lo, hi);
    return __fadd_rn(lo, hi);
}

BQ_DEVINL uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Affine 8-bit: bytes e and e+1 of a code word to bf16x2 (bf16_rne(fmaf(scale,
// q, bias)) per lane).  Each byte becomes the fp32 2^23 + q by a byte permute;
// subtracting 2^23 is exact.
template <int E>
BQ_DEVINL uint32_t deq_aff8_pair(uint32_t word, uint64_t s2, uint64_t b2)
{
    const uint64_t f = f32x2_pack(prmt(word, 0x4B000000u, 0x7650u | E), prmt(word, 0x4B000000u, 0x7650u | (E + 1)));
    float lo, hi;
    f32x2_unpack(fma_f32x2(s2, sub_f32x2(f, f32x2_splat(8388608.0f)), b2), lo, hi);
    return pack_bf16x2_rn(lo, hi);
}

// (a & mask) | magic in one LOP3.
BQ_DEVINL uint32_t and_or(uint32_t a, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

// Immediate-operand forms: the constants stay in the instruction stream instead
// of occupying registers (which the compiler would otherwise rematerialize).
template <uint32_t MASK, uint32_t MAGIC>
BQ_DEVINL uint32_t and_or_i(uint32_t a)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "n"(MAGIC));
    return d;
}

template <uint32_t C>
BQ_DEVINL uint32_t hsub2_bf16_i(uint32_t a)
{
    uint32_t d;
    asm("{\n\t.reg .b32 c;\n\tmov.b32 c, %2;\n\tsub.rn.bf16x2 %0, %1, c;\n\t}" : "=r"(d) : "r"(a), "n"(C));
    return d;
}

// 16-byte global loads that bypass L1 allocation for streamed weights.
BQ_DEVINL uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

BQ_DEVINL uint4 ldg_cached(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

}  // namespace bq
