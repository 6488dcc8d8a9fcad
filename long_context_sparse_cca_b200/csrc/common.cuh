// Shared device helpers of the CUDA library: bf16 packing, vector loads,
// warp reductions, and the window / group arithmetic of CCA-Attention.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace cca {

constexpr float kLog2e = 1.4426950408889634f;

// Start of the local window of query t (section 局部保留模块 of the CCA
// write-up: at least w preceding raw tokens, window aligned to the group
// size g): the largest multiple of g not above max(t - w, 0).
__host__ __device__ __forceinline__ int64_t window_start(int64_t t, int64_t g,
                                                         int64_t w)
{
    const int64_t lo = t > w ? t - w : 0;
    return (lo / g) * g;
}

__device__ __forceinline__ float bf16_lo(uint32_t v)
{
    return __uint_as_float(v << 16);
}

__device__ __forceinline__ float bf16_hi(uint32_t v)
{
    return __uint_as_float(v & 0xFFFF0000u);
}

// Pack two floats into bf16x2 (round to nearest even); `lo` in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Pack two floats into f16x2 (round to nearest even); `lo` in bits 0..15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float f16_lo(uint32_t v)
{
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
}

__device__ __forceinline__ float f16_hi(uint32_t v)
{
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

// Largest finite fp16 value.  Core keys/values are stored in fp16; values
// beyond it are clamped and reported (status bit kStatusRange).
constexpr float kF16Max = 65504.0f;
constexpr unsigned int kStatusTimeout = 1u;  // a bounded wait ran out
constexpr unsigned int kStatusRange = 2u;    // a value exceeded the fp16 range
constexpr unsigned int kStatusCapacity = 4u; // a row's length exceeded the cache

__device__ __forceinline__ float clamp_f16(float x, bool &over)
{
    over |= !(fabsf(x) <= kF16Max);
    return fminf(fmaxf(x, -kF16Max), kF16Max);
}

__device__ __forceinline__ uint16_t bf16_bits(float x)
{
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

// 16-byte global load that skips L1 allocation (streamed data).
__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace cca
