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
