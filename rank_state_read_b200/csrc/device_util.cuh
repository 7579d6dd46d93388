// Small device helpers shared by the decode and flush kernels.
#pragma once

#include <cuda_runtime.h>

namespace sk {

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// read-only (non-coherent) 16-byte global load
__device__ __forceinline__ float4 ldg4(const float *p)
{
    return __ldg(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ float4 lds4(const float *p)
{
    return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ void st4(float *p, float4 v)
{
    *reinterpret_cast<float4 *>(p) = v;
}

__device__ __forceinline__ float dot4(float4 a, float4 b)
{
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

__device__ __forceinline__ void fma4(float4 &acc, float c, float4 x)
{
    acc.x = fmaf(c, x.x, acc.x);
    acc.y = fmaf(c, x.y, acc.y);
    acc.z = fmaf(c, x.z, acc.z);
    acc.w = fmaf(c, x.w, acc.w);
}

__device__ __forceinline__ float4 zero4()
{
    return make_float4(0.f, 0.f, 0.f, 0.f);
}

// sum of a float4 over the lanes whose index differs only in bits 0..2
__device__ __forceinline__ float4 sum8_xor(float4 d)
{
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        d.x += __shfl_xor_sync(0xffffffffu, d.x, o);
        d.y += __shfl_xor_sync(0xffffffffu, d.y, o);
        d.z += __shfl_xor_sync(0xffffffffu, d.z, o);
        d.w += __shfl_xor_sync(0xffffffffu, d.w, o);
    }
    return d;
}

}  // namespace sk
