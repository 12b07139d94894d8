// rope.cu -- Q/KV RMSNorm and partial RoPE before the core attention, and the
// rotation of its output back by the query position (Module D: "Q/KV
// normalisation", "partial RoPE").
//
// In place on rows x heads vectors of c values (bf16 or f32): for each vector
//   x <- x / sqrt(mean_j x_j^2 + eps) * gamma          (when normalise)
// then the last R dims turn in adjacent pairs (c-R+2p, c-R+2p+1) by the angle
//   phi_p = P * base^(-2p/R),  P = pos_mul * (pos ? pos[row] : row) + pos_add.
// One warp per row: lane l owns c/32 consecutive values of a vector, so a
// rotated pair never straddles two lanes; the angles of a row are worked out
// once (in double precision: positions reach 2^20 and beyond, where a float
// angle would be off by a large fraction of a radian) and serve all its heads.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kRopeWarps = 8;

template <typename T, int EPL>
__global__ void __launch_bounds__(32 * kRopeWarps)
norm_rope_kernel(T *__restrict__ x, const float *__restrict__ gamma, int64_t rows, int heads,
                 int R, const int64_t *__restrict__ pos, int64_t pos_mul, int64_t pos_add,
                 int normalise, float eps, float base)
{
    constexpr int C = 32 * EPL;
    const int lane = threadIdx.x & 31;
    const int j0 = lane * EPL;                        // this lane's first channel
    float g[EPL];
#pragma unroll
    for (int e = 0; e < EPL; e++)
        g[e] = gamma ? gamma[j0 + e] : 1.f;
    // inverse frequencies of this lane's rotated pairs (double)
    const int r0 = C - R;                             // first rotated channel
    double inv[EPL / 2];
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
        const int p = (j0 + e - r0) / 2;
        inv[e / 2] = (j0 + e >= r0) ? pow((double)base, -2.0 * p / R) : 0.0;
    }
    const bool rot = j0 + EPL > r0 && R > 0;
    for (int64_t row = (int64_t)blockIdx.x * kRopeWarps + (threadIdx.x >> 5); row < rows;
         row += (int64_t)gridDim.x * kRopeWarps) {
        float cs[EPL / 2], sn[EPL / 2];
        if (rot) {
            const int64_t P = pos_mul * (pos ? pos[row] : row) + pos_add;
#pragma unroll
            for (int e = 0; e < EPL / 2; e++) {
                double s, c;
                sincos((double)P * inv[e], &s, &c);
                cs[e] = (float)c;
                sn[e] = (float)s;
            }
        }
        T *xr = x + row * (int64_t)heads * C;
#pragma unroll 1
        for (int h = 0; h < heads; h++) {
            T *v = xr + (int64_t)h * C + j0;
            // this lane's EPL values as 32-bit words, in 16-, 8- or 4-byte loads
            constexpr int NW = EPL * (int)sizeof(T) / 4;
            uint32_t wd[NW];
            if constexpr (NW % 4 == 0) {
#pragma unroll
                for (int i = 0; i < NW / 4; i++)
                    *(uint4 *)&wd[4 * i] = ((const uint4 *)v)[i];
            } else if constexpr (NW % 2 == 0) {
#pragma unroll
                for (int i = 0; i < NW / 2; i++)
                    *(uint2 *)&wd[2 * i] = ((const uint2 *)v)[i];
            } else {
                wd[0] = *(const uint32_t *)v;
            }
            float f[EPL];
#pragma unroll
            for (int e = 0; e < EPL; e++) {
                if constexpr (sizeof(T) == 2)
                    f[e] = __uint_as_float((e & 1) ? (wd[e / 2] & 0xffff0000u) : (wd[e / 2] << 16));
                else
                    f[e] = __uint_as_float(wd[e]);
            }
            if (normalise) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; e++)
                    ss += f[e] * f[e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv_rms = 1.f / sqrtf(ss / C + eps);
#pragma unroll
                for (int e = 0; e < EPL; e++)
                    f[e] = f[e] * inv_rms * g[e];
            }
            if (rot) {
#pragma unroll
                for (int e = 0; e < EPL; e += 2) {
                    if (j0 + e >= r0) {
                        const float a = f[e], b = f[e + 1];
                        f[e] = a * cs[e / 2] - b * sn[e / 2];
                        f[e + 1] = a * sn[e / 2] + b * cs[e / 2];
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < EPL; e++) {
                if constexpr (sizeof(T) == 2) {
                    if (e & 1) {
                        const __nv_bfloat162 pr = __floats2bfloat162_rn(f[e - 1], f[e]);
                        wd[e / 2] = *(const uint32_t *)&pr;
                    }
                } else {
                    wd[e] = __float_as_uint(f[e]);
                }
            }
            if constexpr (NW % 4 == 0) {
#pragma unroll
                for (int i = 0; i < NW / 4; i++)
                    ((uint4 *)v)[i] = *(const uint4 *)&wd[4 * i];
            } else if constexpr (NW % 2 == 0) {
#pragma unroll
                for (int i = 0; i < NW / 2; i++)
                    ((uint2 *)v)[i] = *(const uint2 *)&wd[2 * i];
            } else {
                *(uint32_t *)v = wd[0];
            }
        }
    }
}

template <typename T>
cudaError_t launch_t(const NormRopeArgs &a, cudaStream_t s)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (a.rows + kRopeWarps - 1) / kRopeWarps;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap)
        blocks = cap;
    T *x = (T *)a.x;
#define CSA_ROPE_CASE(EPL)                                                                      \
    case EPL * 32:                                                                              \
        norm_rope_kernel<T, EPL><<<(unsigned)blocks, 32 * kRopeWarps, 0, s>>>(                   \
            x, a.gamma, a.rows, a.heads, a.rope_dims, a.pos, a.pos_mul, a.pos_add, a.normalise, \
            a.eps, a.base);                                                                      \
        break;
    switch (a.c) {
        CSA_ROPE_CASE(2)
        CSA_ROPE_CASE(4)
        CSA_ROPE_CASE(8)
        CSA_ROPE_CASE(16)
        CSA_ROPE_CASE(32)
    default:
        return cudaErrorInvalidValue;
    }
#undef CSA_ROPE_CASE
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs &a, cudaStream_t s)
{
    if (a.rows == 0 || a.heads == 0)
        return cudaSuccess;
    return a.dt == CSA_BF16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<float>(a, s);
}

}  // namespace csa
