// attend.cu -- shared-KV multi-query attention with sliding window and sink
// (CSA Eq. 18-19, HCA Eq. 24-26, window and sink of Module D), CUDA-core path.
//
// One block serves one query and a group of HG heads. Keys (selected or
// visible compressed entries, then the window rows) are staged KC at a time
// in shared memory as float (the fp8 layout is dequantised on the way in);
// each warp computes whole dot products for a share of the (head, key)
// pairs, and the online softmax (running max and sum per head) rescales the
// output accumulators, which live in registers spread over the block.
// This path serves float32 operands, head dims other than 512 and the split
// decode layout; the tensor-core path (attend_tc.cu) takes bf16 prefill.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int KC = 8;          // keys per chunk
constexpr int kElems = 4096;   // HG * c

struct Dev {
    const void *q;
    csa_dtype q_dt;
    const void *body;
    const float *scale;
    const void *rope;
    int c, body_c, rope_dims, group;
    csa_dtype kv_dt;
    int64_t E;
    const int32_t *idx;
    int dense;
    int k, m;
    const void *kwin;
    int64_t win_rows;
    const int64_t *win_pos0;
    int n_win;
    const int64_t *q_pos;
    const float *sink;
    int64_t n_q;
    int h, HG;
    float scale_qk;
    void *out;
    float *lse;
    unsigned *err;
};

__device__ __forceinline__ float load_plain(const void *p, csa_dtype dt, int64_t i)
{
    return dt == CSA_F32 ? ((const float *)p)[i] : __bfloat162float(((const __nv_bfloat16 *)p)[i]);
}

__device__ __forceinline__ float load_entry(const Dev &d, int64_t row, int x)
{
    if (d.kv_dt != CSA_E4M3)
        return load_plain(d.body, d.kv_dt, row * d.c + x);
    if (x < d.body_c)
        return e4m3_to_float(((const uint8_t *)d.body)[row * d.body_c + x]) *
               d.scale[row * (d.body_c / d.group) + x / d.group];
    return __bfloat162float(((const __nv_bfloat16 *)d.rope)[row * d.rope_dims + (x - d.body_c)]);
}

__global__ void __launch_bounds__(kThreads) attend_kernel(Dev d)
{
    extern __shared__ float sm[];
    const int c = d.c, HG = d.HG;
    float *qs = sm;                          // [HG][c]
    float *ks = qs + HG * c;                 // [KC][c]
    float *z = ks + KC * c;                  // [HG][KC]
    float *mrun = z + HG * KC;               // [HG]
    float *lrun = mrun + HG;                 // [HG]
    float *alpha = lrun + HG;                // [HG]
    __shared__ int64_t key_row[KC];          // >= 0 entry row, or -(window row) - 2; -1 skip
    __shared__ int key_src[KC];              // 0 entry, 1 window

    const int64_t bt = blockIdx.x;
    const int64_t b = bt / d.n_q;
    const int h0 = blockIdx.y * HG;
    const int64_t t = d.q_pos[bt];
    const int64_t V = visible(t, d.m, d.E);
    const int64_t nsel = d.dense ? V : d.k;
    const int64_t w0 = t - d.n_win + 1 < 0 ? 0 : t - d.n_win + 1;
    const int64_t nwin = d.n_win > 0 ? t - w0 + 1 : 0;
    const int64_t NK = nsel + nwin;
    const int64_t wp0 = d.win_pos0 ? d.win_pos0[b] : 0;

    for (int e = threadIdx.x; e < HG * c; e += kThreads) {
        const int hh = e / c, x = e % c;
        float v = 0.f;
        if (h0 + hh < d.h)
            v = load_plain(d.q, d.q_dt, (bt * d.h + h0 + hh) * c + x);
        qs[e] = v;
    }
    for (int hh = threadIdx.x; hh < HG; hh += kThreads) {
        mrun[hh] = -INFINITY;
        lrun[hh] = 0.f;
    }
    constexpr int PER = kElems / kThreads;   // accumulators per thread (max)
    float acc[PER];
#pragma unroll
    for (int r = 0; r < PER; r++)
        acc[r] = 0.f;
    const int nacc = HG * c / kThreads;

    for (int64_t j0 = 0; j0 < NK; j0 += KC) {
        __syncthreads();
        if (threadIdx.x < KC) {
            const int64_t j = j0 + threadIdx.x;
            int64_t r = -1;
            int src = 0;
            if (j < NK) {
                if (j < nsel) {
                    const int64_t s = d.dense ? j : (int64_t)d.idx[bt * d.k + j];
                    if (s >= 0) {
                        if (s < V)
                            r = b * d.E + s;
                        else
                            report(d.err, CSA_ERR_BOUNDS, K_ATTEND, (unsigned)bt, (unsigned)s);
                    }
                } else {
                    const int64_t p = w0 + (j - nsel);
                    const int64_t wr = p - wp0;
                    if (wr >= 0 && wr < d.win_rows) {
                        r = b * d.win_rows + wr;
                        src = 1;
                    } else {
                        report(d.err, CSA_ERR_BOUNDS, K_ATTEND, (unsigned)bt, (unsigned)p);
                    }
                }
            }
            key_row[threadIdx.x] = r;
            key_src[threadIdx.x] = src;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < KC * c; e += kThreads) {
            const int jj = e / c, x = e % c;
            const int64_t r = key_row[jj];
            float v = 0.f;
            if (r >= 0)
                v = key_src[jj] ? load_plain(d.kwin, d.q_dt, r * c + x) : load_entry(d, r, x);
            ks[e] = v;
        }
        __syncthreads();
        // z[hh][jj] = scale * q_hh . key_jj  (one warp per pair)
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        for (int pr = warp; pr < HG * KC; pr += kWarps) {
            const int hh = pr / KC, jj = pr % KC;
            float s = 0.f;
            for (int x = lane; x < c; x += 32)
                s += qs[hh * c + x] * ks[jj * c + x];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0)
                z[hh * KC + jj] = key_row[jj] >= 0 ? d.scale_qk * s : -INFINITY;
        }
        __syncthreads();
        for (int hh = threadIdx.x; hh < HG; hh += kThreads) {
            float zm = -INFINITY;
            for (int jj = 0; jj < KC; jj++)
                zm = fmaxf(zm, z[hh * KC + jj]);
            const float mo = mrun[hh];
            const float mn = fmaxf(mo, zm);
            if (mn == -INFINITY) {
                alpha[hh] = 1.f;
                for (int jj = 0; jj < KC; jj++)
                    z[hh * KC + jj] = 0.f;
            } else {
                const float al = expf(mo - mn);
                float l = lrun[hh] * al;
                for (int jj = 0; jj < KC; jj++) {
                    const float p = expf(z[hh * KC + jj] - mn);
                    z[hh * KC + jj] = p;
                    l += p;
                }
                alpha[hh] = al;
                mrun[hh] = mn;
                lrun[hh] = l;
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; r++) {
            if (r < nacc) {
                const int e = threadIdx.x + r * kThreads;
                const int hh = e / c, x = e % c;
                float a = acc[r] * alpha[hh];
#pragma unroll
                for (int jj = 0; jj < KC; jj++)
                    a += z[hh * KC + jj] * ks[jj * c + x];
                acc[r] = a;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < PER; r++) {
        if (r < nacc) {
            const int e = threadIdx.x + r * kThreads;
            const int hh = e / c, x = e % c;
            const int head = h0 + hh;
            if (head >= d.h)
                continue;
            const float zs = d.sink[head];
            const float mo = mrun[hh];
            float o, l;
            if (zs == INFINITY) {
                o = 0.f;
                l = INFINITY;
            } else {
                const float M = fmaxf(mo, zs);
                if (M == -INFINITY) {
                    o = 0.f;
                    l = -INFINITY;
                } else {
                    const float f = expf(mo - M);
                    const float den = lrun[hh] * f + expf(zs - M);
                    o = acc[r] * f / den;
                    l = M + logf(den);
                }
            }
            const int64_t oi = (bt * d.h + head) * c + x;
            if (d.q_dt == CSA_F32)
                ((float *)d.out)[oi] = o;
            else
                ((__nv_bfloat16 *)d.out)[oi] = __float2bfloat16_rn(o);
            if (x == 0 && d.lse)
                d.lse[bt * d.h + head] = l;
        }
    }
}

}  // namespace

size_t attend_tc_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys);

// Scratch of the tensor-core path (split-key partial results); the CUDA-core
// path needs none.
size_t attend_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys)
{
    return attend_tc_workspace_size(B, n_q, h, c, max_keys);
}

cudaError_t launch_attend_tc(const AttendArgs &a, unsigned *err, cudaStream_t s, bool *taken);

cudaError_t launch_attend(const AttendArgs &a, unsigned *err, cudaStream_t s)
{
    bool taken = false;
    cudaError_t e = launch_attend_tc(a, err, s, &taken);
    if (taken || e != cudaSuccess)
        return e;
    Dev d;
    d.q = a.q;
    d.q_dt = a.q_dt;
    d.body = a.kv.body;
    d.scale = a.kv.scale;
    d.rope = a.kv.rope;
    d.c = a.kv.c;
    d.kv_dt = a.kv.dt;
    d.rope_dims = a.kv.dt == CSA_E4M3 ? a.kv.rope_dims : 0;
    d.body_c = d.c - d.rope_dims;
    d.group = a.kv.dt == CSA_E4M3 ? a.kv.scale_group : 1;
    d.E = a.E;
    d.idx = a.idx;
    d.dense = a.dense;
    d.k = a.k;
    d.m = a.m;
    d.kwin = a.kwin;
    d.win_rows = a.win_rows;
    d.win_pos0 = a.win_pos0;
    d.n_win = a.n_win;
    d.q_pos = a.q_pos;
    d.sink = a.sink;
    d.n_q = a.n_q;
    d.h = a.h;
    d.HG = kElems / d.c;
    if (d.HG > a.h) {
        d.HG = 1;
        while (d.HG < a.h)
            d.HG *= 2;
        while (d.HG * d.c < kThreads)
            d.HG *= 2;
    }
    d.scale_qk = a.scale;
    d.out = a.out;
    d.lse = a.lse;
    d.err = err;
    const int64_t rows = (int64_t)a.B * a.n_q;
    if (rows == 0)
        return cudaSuccess;
    dim3 grid((unsigned)rows, (unsigned)((a.h + d.HG - 1) / d.HG));
    const size_t smem = ((size_t)d.HG * d.c + (size_t)KC * d.c + (size_t)d.HG * KC + 3 * d.HG) *
                        sizeof(float);
    cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
    attend_kernel<<<grid, kThreads, smem, s>>>(d);
    return cudaGetLastError();
}

}  // namespace csa
