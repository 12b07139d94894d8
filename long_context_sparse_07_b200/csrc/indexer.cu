// indexer.cu -- lightning-indexer scores (Eq. 16), CUDA-core path.
//
// I[b][t][s] = sum_h wI[b][t][h] * ReLU(qI[b][t][h] . kI[b][s]) for s < V_t.
// One block scores a tile of TQ queries x TS keys of one batch. The key tile
// (dequantised to float) stays in shared memory for all heads; each head's
// query tile is staged in turn. Key tiles past the causal bound of every
// query of the tile are skipped; score entries s >= V_t are not written.
// This path serves float32 operands and any shape; the tensor-core path in
// indexer_tc.cu takes bf16 / e4m3 operands of the supported shapes. FP4 keys
// (e2m1 codes with a power-of-two scale per 32 channels) are decoded here
// to float.
#include <cuda_fp4.h>

#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int TQ = 16;
constexpr int TS = 64;
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float ld_val(const T *p, int64_t i);
template <> __device__ __forceinline__ float ld_val<float>(const float *p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float ld_val<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i)
{
    return __bfloat162float(p[i]);
}
template <> __device__ __forceinline__ float ld_val<uint8_t>(const uint8_t *p, int64_t i)
{
    return e4m3_to_float(p[i]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
indexer_kernel(const T *__restrict__ qI, const float *__restrict__ qI_scale,
               const float *__restrict__ wI, const T *__restrict__ kI,
               const float *__restrict__ kI_scale, const uint8_t *__restrict__ kI_exp,
               const int64_t *__restrict__ q_pos, int64_t n_q, int64_t E, int hI, int cI, int m,
               float *__restrict__ scores, int64_t ld)
{
    extern __shared__ float sm[];
    float *ks = sm;                       // [TS][cI + 1]
    float *qs = ks + TS * (cI + 1);       // [TQ][cI + 1]
    __shared__ int64_t vis[TQ];
    __shared__ int any_work;

    const int b = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.x * TQ;
    const int64_t s0 = (int64_t)blockIdx.y * TS;

    if (threadIdx.x == 0)
        any_work = 0;
    __syncthreads();
    if (threadIdx.x < TQ) {
        const int64_t t = t0 + threadIdx.x;
        int64_t V = 0;
        if (t < n_q)
            V = visible(q_pos[(int64_t)b * n_q + t], m, E);
        vis[threadIdx.x] = V;
        if (V > s0)
            atomicOr(&any_work, 1);
    }
    __syncthreads();
    if (!any_work)
        return;

    // key tile, dequantised
    for (int e = threadIdx.x; e < TS * cI; e += kThreads) {
        const int r = e / cI, x = e % cI;
        const int64_t s = s0 + r;
        float v = 0.f;
        if (s < E) {
            const int64_t row = (int64_t)b * E + s;
            if (kI_exp) {
                // fp4 key: nibble x % 2 of byte x / 2, scaled by 2^(e - 127)
                const uint8_t byte = ((const uint8_t *)kI)[row * (cI / 2) + x / 2];
                const __half_raw h = __nv_cvt_fp4_to_halfraw(
                    (__nv_fp4_storage_t)((x & 1) ? byte >> 4 : byte & 15), __NV_E2M1);
                v = ldexpf(__half2float(__half(h)), (int)kI_exp[row * (cI / 32) + x / 32] - 127);
            } else {
                v = ld_val<T>(kI, row * cI + x);
                if (kI_scale)
                    v *= kI_scale[row];
            }
        }
        ks[r * (cI + 1) + x] = v;
    }

    // thread -> (query row tq, 4 keys)
    const int tq = threadIdx.x / (TS / 4);
    const int sk = (threadIdx.x % (TS / 4)) * 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int hh = 0; hh < hI; hh++) {
        __syncthreads();
        for (int e = threadIdx.x; e < TQ * cI; e += kThreads) {
            const int r = e / cI, x = e % cI;
            const int64_t t = t0 + r;
            float v = 0.f;
            if (t < n_q) {
                const int64_t row = ((int64_t)b * n_q + t) * hI + hh;
                v = ld_val<T>(qI, row * cI + x);
                if (qI_scale)
                    v *= qI_scale[row];
            }
            qs[r * (cI + 1) + x] = v;
        }
        __syncthreads();
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        for (int x = 0; x < cI; x++) {
            const float qv = qs[tq * (cI + 1) + x];
#pragma unroll
            for (int j = 0; j < 4; j++)
                d[j] += qv * ks[(sk + j) * (cI + 1) + x];
        }
        const int64_t t = t0 + tq;
        const float w = (t < n_q) ? wI[((int64_t)b * n_q + t) * hI + hh] : 0.f;
#pragma unroll
        for (int j = 0; j < 4; j++)
            acc[j] += w * fmaxf(d[j], 0.f);
    }
    const int64_t t = t0 + tq;
    if (t < n_q) {
        float *row = scores + ((int64_t)b * n_q + t) * ld;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int64_t s = s0 + sk + j;
            if (s < vis[tq])
                row[s] = acc[j];
        }
    }
}

}  // namespace

cudaError_t launch_indexer_tc(const IndexerArgs &a, unsigned *err, cudaStream_t s, bool *taken);

cudaError_t launch_indexer(const IndexerArgs &a, unsigned *err, cudaStream_t s)
{
    bool taken = false;
    cudaError_t e = launch_indexer_tc(a, err, s, &taken);
    if (taken || e != cudaSuccess)
        return e;
    dim3 grid((unsigned)((a.n_q + TQ - 1) / TQ), (unsigned)((a.E + TS - 1) / TS), (unsigned)a.B);
    if (grid.x == 0 || grid.y == 0 || grid.z == 0)
        return cudaSuccess;
    const size_t smem = (size_t)(TS + TQ) * (a.cI + 1) * sizeof(float);
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(indexer_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        cudaFuncSetAttribute(indexer_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        cudaFuncSetAttribute(indexer_kernel<uint8_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        attr_set = true;
    }
    const float *ksc = a.kI.dt == CSA_E4M3 ? a.kI.scale : nullptr;
    const uint8_t *kex = a.kI.dt == CSA_E2M1 ? (const uint8_t *)a.kI.scale : nullptr;
    const float *qsc = a.dt == CSA_E4M3 ? a.qI_scale : nullptr;
    switch (a.dt) {
    case CSA_F32:
        indexer_kernel<float><<<grid, kThreads, smem, s>>>(
            (const float *)a.qI, qsc, a.wI, (const float *)a.kI.body, ksc, kex, a.q_pos, a.n_q, a.E,
            a.hI, a.cI, a.m, a.scores, a.ld);
        break;
    case CSA_BF16:
        indexer_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
            (const __nv_bfloat16 *)a.qI, qsc, a.wI, (const __nv_bfloat16 *)a.kI.body, ksc,
            kex, a.q_pos, a.n_q, a.E, a.hI, a.cI, a.m, a.scores, a.ld);
        break;
    case CSA_E4M3:
        indexer_kernel<uint8_t><<<grid, kThreads, smem, s>>>(
            (const uint8_t *)a.qI, qsc, a.wI, (const uint8_t *)a.kI.body, ksc, kex, a.q_pos, a.n_q,
            a.E, a.hI, a.cI, a.m, a.scores, a.ld);
        break;
    }
    return cudaGetLastError();
}

}  // namespace csa
