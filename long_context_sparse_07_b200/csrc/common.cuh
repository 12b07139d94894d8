// common.cuh -- shared device helpers of the CSA / HCA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// Device error word: [0] = -status of the first failure (0 = none),
// [1] = kernel id, [2], [3] = kernel-specific detail (row, index).
enum KernelId : unsigned {
    K_COMPRESS = 1, K_INDEXER = 2, K_TOPK = 3, K_ATTEND = 4, K_ATTEND_TC = 5,
    K_INDEXER_TC = 6, K_COMBINE = 7, K_PROBE = 8, K_GEMM = 9
};

__device__ __forceinline__ void report(unsigned *err, csa_status code, unsigned kernel,
                                       unsigned a, unsigned b)
{
    if (atomicCAS(err, 0u, (unsigned)(-(int)code)) == 0u) {
        err[1] = kernel;
        err[2] = a;
        err[3] = b;
    }
}

// Entries visible to a query at absolute position t (entry i covers tokens
// m*i .. m*i+m-1 and becomes visible when its last token is at or before t).
__host__ __device__ __forceinline__ int64_t visible(int64_t t, int m, int64_t E)
{
    int64_t v = (t + 1) / m;
    if (v < 0) v = 0;
    return v < E ? v : E;
}

// ---- loads of 16 bytes converted to float ---------------------------------

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *v)
{
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ void load4(const float *p, float *v)
{
    float4 f = *reinterpret_cast<const float4 *>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float *p, float *v) { load4(p, v); }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float *v) { load8(p, v); }
};

__device__ __forceinline__ float e4m3_to_float(uint8_t code)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(h));
}

// Two floats to two e4m3 codes: round to nearest even, saturate to +-448.
__device__ __forceinline__ uint16_t float2_to_e4m3x2(float a, float b)
{
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float scalar_to_float(float x) { return x; }
__device__ __forceinline__ float scalar_to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// Order-preserving unsigned key of a float (larger float -> larger key);
// -0 is folded onto +0 so that the two compare equal.
__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace csa
