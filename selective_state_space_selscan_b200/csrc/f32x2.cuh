// f32x2.cuh -- packed fp32 pairs (one 64-bit register, two lanes of the
// FMA pipe per instruction) and bf16 packing helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace selscan {

__device__ __forceinline__ uint64_t pk2(float lo, float hi)
{
    return (uint64_t(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}

__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(uint32_t(v)); }

__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float(uint32_t(v >> 32)); }

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// bf16 pair (lo, hi halves of a 32-bit word) -> packed fp32 pair
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w)
{
    return pk2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ void unpack8_bf16(uint4 v, float (&f)[8])
{
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace selscan
