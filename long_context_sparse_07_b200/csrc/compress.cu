// compress.cu -- token-level KV compressor (CSA Eq. 9-12, HCA Eq. 20-23).
//
// HBM-streaming kernel. Each thread owns VEC consecutive channels (16-byte
// vector loads of C and Z rows, coalesced across the threads of an entry) and
// keeps, per channel, an online softmax (running max, running sum, running
// weighted sum) over the rows it reads. The softmax is over token positions
// and independent per channel, so no cross-lane reduction is needed inside a
// slice. For long windows (HCA, m' = 128) the rows of one entry are split
// into `split` interleaved slices handled by different warps; the slices are
// merged through shared memory with the usual max-rescaled combination.
// Each row of Ca / Za / Cb / Zb is read exactly once from HBM.
#include <cuda_fp4.h>
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 256;

struct OutDesc {
    void *body;
    float *scale;
    void *rope;
    int c, body_c, rope_dims, group;
    csa_dtype dt;
};

// 16 bytes of T (8 bf16 or 4 f32) as floats.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &u, float *v);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4 &u, float *v)
{
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &u, float *v)
{
    const __nv_bfloat162 *h = (const __nv_bfloat162 *)&u;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const float2 f = __bfloat1622float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
compress_kernel(const T *__restrict__ Ca, const T *__restrict__ Cb, const T *__restrict__ Za,
                const T *__restrict__ Zb, const float *__restrict__ Ba,
                const float *__restrict__ Bb, int64_t E, int c, int m, int overlap, int split,
                OutDesc out)
{
    constexpr int VEC = Vec<T>::N;
    extern __shared__ float smem[];

    const int tpe = c / VEC;                 // threads per entry slice
    const int lane_e = threadIdx.x % tpe;
    const int rest = threadIdx.x / tpe;
    const int slice = rest % split;
    const int e_local = rest / split;
    const int epb = kThreads / (tpe * split);
    const int64_t i = (int64_t)blockIdx.x * epb + e_local;
    const int ch = lane_e * VEC;
    const bool live = (e_local < epb) && (i < E);

    float mx[VEC], sum[VEC], acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; v++) {
        mx[v] = -INFINITY;
        sum[v] = 0.f;
        acc[v] = 0.f;
    }
    if (live) {
        const int rows = (overlap && i > 0) ? 2 * m : m;
        // UNR rows of this slice are loaded before any is folded in, so their
        // memory latencies overlap (16 bytes of C, of Z and VEC bias values each)
        constexpr int UNR = 4;
        for (int r0 = slice; r0 < rows; r0 += split * UNR) {
            uint4 craw[UNR], zraw[UNR];
            float bv[UNR][VEC];
#pragma unroll
            for (int q = 0; q < UNR; q++) {
                const int r = r0 + q * split;
                if (r < rows) {
                    const T *cp, *zp;
                    const float *bp;
                    if (r < m) {
                        const int64_t row = (int64_t)m * i + r;
                        cp = Ca + row * c + ch;
                        zp = Za + row * c + ch;
                        bp = Ba + (int64_t)r * c + ch;
                    } else {
                        const int64_t row = (int64_t)m * (i - 1) + (r - m);
                        cp = Cb + row * c + ch;
                        zp = Zb + row * c + ch;
                        bp = Bb + (int64_t)(r - m) * c + ch;
                    }
                    craw[q] = __ldg((const uint4 *)cp);
                    zraw[q] = __ldg((const uint4 *)zp);
#pragma unroll
                    for (int v = 0; v < VEC; v += 4)
                        load4(bp + v, bv[q] + v);
                }
            }
#pragma unroll
            for (int q = 0; q < UNR; q++) {
                if (r0 + q * split >= rows)
                    break;
                float cv[VEC], zv[VEC];
                unpack16<T>(craw[q], cv);
                unpack16<T>(zraw[q], zv);
#pragma unroll
                for (int v = 0; v < VEC; v++) {
                    const float l = zv[v] + bv[q][v];
                    if (l > mx[v]) {
                        const float f = expf(mx[v] - l);
                        sum[v] = sum[v] * f + 1.f;
                        acc[v] = acc[v] * f + cv[v];
                        mx[v] = l;
                    } else {
                        const float pr = expf(l - mx[v]);
                        sum[v] += pr;
                        acc[v] += pr * cv[v];
                    }
                }
            }
        }
    }

    float res[VEC];
    if (split > 1) {
        // merge the slices: smem[(e_local*split + slice)*tpe + lane][3][VEC]
        float *mine = smem + ((size_t)(e_local * split + slice) * tpe + lane_e) * 3 * VEC;
#pragma unroll
        for (int v = 0; v < VEC; v++) {
            mine[v] = mx[v];
            mine[VEC + v] = sum[v];
            mine[2 * VEC + v] = acc[v];
        }
        __syncthreads();
#pragma unroll
        for (int v = 0; v < VEC; v++) {
            float M = -INFINITY;
            for (int s = 0; s < split; s++) {
                const float *o = smem + ((size_t)(e_local * split + s) * tpe + lane_e) * 3 * VEC;
                M = fmaxf(M, o[v]);
            }
            float S = 0.f, A = 0.f;
            for (int s = 0; s < split; s++) {
                const float *o = smem + ((size_t)(e_local * split + s) * tpe + lane_e) * 3 * VEC;
                const float f = (o[v] == -INFINITY) ? 0.f : expf(o[v] - M);
                S += o[VEC + v] * f;
                A += o[2 * VEC + v] * f;
            }
            res[v] = A / S;
        }
    } else {
#pragma unroll
        for (int v = 0; v < VEC; v++)
            res[v] = acc[v] / sum[v];
    }

    const bool writer = live && slice == 0;
    if (out.dt == CSA_E2M1) {
        // fp4 indexer keys: per block of 32 channels (32 / VEC lanes) the
        // smallest 2^E with 6 * 2^E >= the block's largest magnitude, raised
        // to the row's largest E - 8 when below it (the row's lanes are the
        // entry's tpe consecutive lanes); an all-zero row takes E = 0
        float amax = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; v++)
            amax = fmaxf(amax, fabsf(res[v]));
        const int glanes = 32 / VEC;
        for (int off = 1; off < glanes; off <<= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        constexpr int kNone = -100000;
        int e = kNone;
        if (amax > 0.f) {
            int x;
            const float f = frexpf(amax, &x);       // amax = f 2^x, f in [0.5, 1)
            e = f <= 0.75f ? x - 3 : x - 2;
        }
        int emax = e;
        for (int off = glanes; off < tpe; off <<= 1)
            emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, off));
        if (!writer)
            return;
        e = emax == kNone ? 0 : max(e, emax - 8);
        e = min(max(e, -127), 128);
        uint32_t packed = 0;                          // channel ch + v at byte v / 2
#pragma unroll
        for (int v = 0; v < VEC; v += 2)
            packed |= (uint32_t)(uint8_t)__nv_cvt_float2_to_fp4x2(
                          make_float2(ldexpf(res[v], -e), ldexpf(res[v + 1], -e)), __NV_E2M1,
                          cudaRoundNearest)
                      << (4 * v);
        uint8_t *dst = (uint8_t *)out.body + i * (c / 2) + ch / 2;
        if (VEC == 8)
            *reinterpret_cast<uint32_t *>(dst) = packed;
        else
            *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
        if (ch % 32 == 0)
            ((uint8_t *)out.scale)[i * (c / 32) + ch / 32] = (uint8_t)(e + 127);
        return;
    }
    if (out.dt == CSA_E4M3) {
        // group amax across the group's lanes (aligned, power-of-two lanes);
        // every thread takes part in the shuffles, only slice 0 writes.
        const bool in_body = ch < out.body_c;
        float amax = 0.f;
        if (in_body) {
#pragma unroll
            for (int v = 0; v < VEC; v++)
                amax = fmaxf(amax, fabsf(res[v]));
        }
        const int glanes = out.group / VEC;
        for (int off = 1; off < glanes; off <<= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (!writer)
            return;
        if (in_body) {
            float s = amax / 448.0f;
            if (s < FLT_MIN)
                s = FLT_MIN;
            uint8_t *dst = (uint8_t *)out.body + i * out.body_c + ch;
            uint16_t codes[VEC / 2];
#pragma unroll
            for (int v = 0; v < VEC; v += 2)
                codes[v / 2] = float2_to_e4m3x2(res[v] / s, res[v + 1] / s);
            if (VEC == 8)
                *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<uint2 *>(codes);
            else
                *reinterpret_cast<uint32_t *>(dst) = *reinterpret_cast<uint32_t *>(codes);
            if ((ch % out.group) == 0)
                out.scale[i * (out.body_c / out.group) + ch / out.group] = s;
        } else {
            __nv_bfloat16 *dst = (__nv_bfloat16 *)out.rope + i * out.rope_dims + (ch - out.body_c);
#pragma unroll
            for (int v = 0; v < VEC; v++)
                dst[v] = __float2bfloat16_rn(res[v]);
        }
        return;
    }
    if (!writer)
        return;
    if (out.dt == CSA_F32) {
        float *dst = (float *)out.body + i * c + ch;
#pragma unroll
        for (int v = 0; v < VEC; v += 4)
            *reinterpret_cast<float4 *>(dst + v) = make_float4(res[v], res[v + 1], res[v + 2], res[v + 3]);
    } else {
        __nv_bfloat16 *dst = (__nv_bfloat16 *)out.body + i * c + ch;
        __nv_bfloat162 h[VEC / 2];
#pragma unroll
        for (int v = 0; v < VEC; v += 2)
            h[v / 2] = __floats2bfloat162_rn(res[v], res[v + 1]);
        if (VEC == 8)
            *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<uint4 *>(h);
        else
            *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<uint2 *>(h);
    }
}

}  // namespace

cudaError_t launch_compress(const CompressArgs &a, unsigned *err, cudaStream_t s)
{
    (void)err;
    const int VEC = a.in_dt == CSA_BF16 ? 8 : 4;
    const int tpe = a.c / VEC;
    const int64_t E = a.n / a.m;
    // Rows of an entry are split over `split` slices when the window is long
    // (>= 8 rows per slice), or, for narrow rows, when there are too few
    // entries to keep the GPU busy (>= 2 rows per slice).
    const int rows = a.overlap ? 2 * a.m : a.m;
    const int64_t target_threads = 148 * 1024;
    int split = 1;
    while (split * 2 * tpe <= kThreads &&
           (rows / (split * 2) >= 8 ||
            (tpe <= 32 && rows / (split * 2) >= 2 && E * tpe * split < target_threads)))
        split *= 2;
    const int epb = kThreads / (tpe * split);
    OutDesc o;
    o.body = a.out.body;
    o.scale = a.out.scale;
    o.rope = a.out.rope;
    o.c = a.c;
    o.rope_dims = a.out.dt == CSA_E4M3 ? a.out.rope_dims : 0;
    o.body_c = a.c - o.rope_dims;
    o.group = a.out.dt == CSA_E4M3 ? a.out.scale_group : 1;
    o.dt = a.out.dt;
    const size_t smem = split > 1 ? (size_t)kThreads * 3 * VEC * sizeof(float) : 0;
    const int64_t blocks = (E + epb - 1) / epb;
    if (blocks == 0)
        return cudaSuccess;
    if (a.in_dt == CSA_BF16)
        compress_kernel<__nv_bfloat16><<<(unsigned)blocks, kThreads, smem, s>>>(
            (const __nv_bfloat16 *)a.Ca, (const __nv_bfloat16 *)a.Cb,
            (const __nv_bfloat16 *)a.Za, (const __nv_bfloat16 *)a.Zb, a.Ba, a.Bb, E, a.c,
            a.m, a.overlap, split, o);
    else
        compress_kernel<float><<<(unsigned)blocks, kThreads, smem, s>>>(
            (const float *)a.Ca, (const float *)a.Cb, (const float *)a.Za,
            (const float *)a.Zb, a.Ba, a.Bb, E, a.c, a.m, a.overlap, split, o);
    return cudaGetLastError();
}

}  // namespace csa
