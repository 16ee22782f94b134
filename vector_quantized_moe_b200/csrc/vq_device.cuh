// Device helpers shared by the sm_100a kernels of the VQ-MoE library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace vq {

// ---------------------------------------------------------------- loads

__device__ __forceinline__ uint32_t ldg_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ldg_u64(const uint32_t *p)
{
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_u128(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t *p)
{
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// 16 bytes of shared memory when pred holds, else zeros (a predicated load, no branch).
__device__ __forceinline__ uint4 lds128_if(const void *p, bool pred)
{
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"((int)pred));
    return v;
}

// ---------------------------------------------------------------- numbers

__device__ __forceinline__ float f16_to_f32(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b)
{
    return __uint_as_float((uint32_t)b << 16);
}

// Two bf16 values packed in a word -> fp16x2 (round to nearest; exact for
// magnitudes in [2^-14, 65504]).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w)
{
    float lo = __uint_as_float(w << 16);
    float hi = __uint_as_float(w & 0xFFFF0000u);
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v)
{
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

// ---------------------------------------------------------------- power-of-two operand scaling
//
// The tensor-core operands are fp16, whose range ([2^-24, 65504]) is far
// narrower than bf16's. Every 16-bit operand row (a token's activations, a
// slot's SwiGLU output) is therefore multiplied by 2^k before its fp16
// rounding, with k chosen so that the row's largest magnitude lands in
// [2^14, 2^15), and the fp32 results are multiplied by 2^-k. Both steps are
// exact (a power of two), so the only rounding is the fp16 rounding of the
// scaled operand, at fp16's full 11-bit precision for every element within
// 2^-28 of the row's largest.

// 2^e as an fp32 value, for e in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149));
}

// The scale exponent k for a row whose largest magnitude has the fp32 bit
// pattern `mag` (sign bit clear): 14 - floor(log2 max), capped at 127 so that
// 2^k and 2^-k are fp32 numbers, read off the exponent field (for a normal
// max with biased exponent E, floor(log2 max) = E - 127, so k = 141 - E; a
// zero or subnormal max has E = 0 and takes the cap: any scale leaves such a
// row's fp16 image within fp16's range). A row holding Inf or NaN (E = 255)
// gets 0 (no scaling). The result lies in [-113, 127].
__device__ __forceinline__ int scale_exp(uint32_t mag)
{
    const int E = (int)(mag >> 23);
    return E == 255 ? 0 : min(141 - E, 127);
}

// 2^e for e in [-126, 127] (a normal fp32 number), e.g. a scale_exp result.
__device__ __forceinline__ float pow2f_normal(int e)
{
    return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Two bf16 values packed in a word, times 2^k (as the fp32 value s = 2^k),
// -> fp16x2 (round to nearest even).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float s)
{
    const float lo = __uint_as_float(w << 16) * s;
    const float hi = __uint_as_float(w & 0xFFFF0000u) * s;
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Largest magnitude of the four bf16 pairs of a 16-byte load, as bf16
// magnitude bits in the low half (NaN patterns compare above Inf).
__device__ __forceinline__ uint32_t bf16x8_max_mag(uint4 v)
{
    uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16);
}

// ---------------------------------------------------------------- tensor cores

// D = A * B + C for one m16n8k16 tile, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- grid dependencies

// Programmatic dependent launch: wait until the previous kernel on the stream
// has completed and its memory is visible.
__device__ __forceinline__ void grid_dep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel on the stream to start its prologue (its own
// griddepcontrol.wait still waits for this kernel's completion and memory).
__device__ __forceinline__ void grid_dep_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- skipzero rows

// Packed-row index of row r of expert e, or -1 when the row is dead.
// bitmap/rank are [E, bm_words]; without a bitmap every row is live.
__device__ __forceinline__ long live_row(const uint32_t *bitmap, const uint32_t *rank, int bm_words,
                                         int rows, int e, int r)
{
    if (!bitmap)
        return (long)e * rows + r;
    const uint32_t w = bitmap[(long)e * bm_words + (r >> 5)];
    const uint32_t bit = 1u << (r & 31);
    if (!(w & bit))
        return -1;
    return (long)rank[(long)e * bm_words + (r >> 5)] + __popc(w & (bit - 1u));
}

}  // namespace vq
