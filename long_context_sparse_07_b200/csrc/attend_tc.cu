// attend_tc.cu -- shared-KV multi-query attention with window and sink on the
// 5th-generation tensor cores (CSA Eq. 18-19, HCA Eq. 24-26, Module D).
//
// All H heads of a query share one key set, and every key is also its own
// value. Keys therefore go on the M axis of both contractions:
//   S^T[key][head]  = sum_d K[key][d] * Q[head][d]        (M = 128 keys, N = H)
//   O^T[dim][head] += sum_key K[key][dim] * P^T[key][head] (M = 4 x 128 dims, N = H)
// so one 128 x 512 bf16 key tile staged in shared memory (128-byte swizzled,
// gathered row by row with cp.async from the selection list or the window)
// serves as the K-major A operand of the first product and, read along the
// other axis, as the M/N-major A operand of the second. S^T and O^T live in
// tensor memory (H + 4H columns).
//
// Softmax: the thread that owns a key lane holds that key's logits for every
// head. The per-head offset m_h is updated lazily: only when some logit of a
// tile exceeds m_h + 8 are the tile's maxima reduced across the block, the O^T
// accumulators rescaled in tensor memory and the partial sums rescaled; the
// first tile of a query always takes that path. Probabilities are rounded to
// bf16 for the second product and summed from the rounded values, so the
// numerator and the denominator agree. The sink joins only the final
// normalisation: out = O * e^{m-M} / (l * e^{m-M} + e^{z'-M}), M = max(m, z').
//
// One persistent block per SM loops over queries; four warps gather, run the
// softmax and the epilogue, thread 0 issues the MMAs. Every wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kThreads = 128;
constexpr int DIM = 512;
constexpr int KT = 128;
constexpr float kLazy = 8.f;

struct TcAttn {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *ent;
    const int32_t *idx;
    int dense, k, m;
    int64_t E;
    const __nv_bfloat16 *kwin;
    int64_t win_rows;
    const int64_t *win_pos0;
    int n_win;
    const int64_t *q_pos;
    const float *sink;
    int64_t n_q, nqueries;
    float scale;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *err;
};

template <int H>
struct Lay {
    static constexpr size_t K_OFF = 0;                              // 8 x 16 KB
    static constexpr size_t Q_OFF = 8 * 16384;                      // 8 x H x 128
    static constexpr size_t P_OFF = Q_OFF + 8 * H * 128;            // 2 x H x 128
    static constexpr size_t PTR_OFF = P_OFF + 2 * H * 128;          // 128 pointers
    static constexpr size_t F_OFF = PTR_OFF + KT * 8;               // floats: m, red[4], alpha, fin, lsum
    static constexpr size_t BAR_OFF = F_OFF + ((8 * H * 4 + 63) / 64) * 64;
    static constexpr size_t TOTAL = BAR_OFF + 64;
    static constexpr uint32_t TMEM_COLS = (5 * H <= 128) ? 128 : (5 * H <= 256 ? 256 : 512);
    static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, H, 0, 0);
    static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, H, 1, 0);
};

// Loads the H columns starting at `taddr` of this thread's TMEM lane.
template <int H>
__device__ __forceinline__ void load_cols(uint32_t taddr, float (&v)[H])
{
    if constexpr (H >= 32) {
#pragma unroll
        for (int c = 0; c < H / 32; c++) {
            uint32_t r[32];
            tc::tmem_ld32(taddr + c * 32, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j++)
                v[c * 32 + j] = __uint_as_float(r[j]);
        }
    } else {
        uint32_t r[16];
        tc::tmem_ld16(taddr, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; j++)
            v[j] = __uint_as_float(r[j]);
    }
}

// Multiplies the H columns starting at `taddr` of this thread's lane by
// f[column], in place (16 columns at a time).
template <int H>
__device__ __forceinline__ void scale_cols(uint32_t taddr, const float *f)
{
#pragma unroll 1
    for (int c = 0; c < H / 16; c++) {
        uint32_t r[16];
        tc::tmem_ld16(taddr + c * 16, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; j++)
            r[j] = __float_as_uint(__uint_as_float(r[j]) * f[c * 16 + j]);
        tc::tmem_st16(taddr + c * 16, r);
    }
    tc::tmem_st_wait();
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const TcAttn a)
{
    using L = Lay<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sK = sm + L::K_OFF;
    uint8_t *sQ = sm + L::Q_OFF;
    uint8_t *sP = sm + L::P_OFF;
    const __nv_bfloat16 **kptr = (const __nv_bfloat16 **)(sm + L::PTR_OFF);
    float *m_run = (float *)(sm + L::F_OFF);     // [H]
    float *red = m_run + H;                      // [4][H]
    float *alpha = red + 4 * H;                  // [H]
    float *fin = alpha + H;                      // [H]
    uint64_t *bars = (uint64_t *)(sm + L::BAR_OFF);
    uint64_t *sbar = bars, *obar = bars + 1, *done = bars + 2;
    uint32_t *tmem_slot = (uint32_t *)(bars + 3);
    int *abort_flag = (int *)(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        tc::mbar_init(sbar, 1);
        tc::mbar_init(obar, 1);
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, L::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_tm = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t sK_a = tc::smem_u32(sK), sQ_a = tc::smem_u32(sQ), sP_a = tc::smem_u32(sP);

    uint32_t g = 0;                     // tiles issued by this block (barrier phases)
    bool ok = true;

    for (int64_t bt = blockIdx.x; bt < a.nqueries && ok; bt += gridDim.x) {
        const int64_t b = bt / a.n_q;
        const int64_t t = a.q_pos[bt];
        const int64_t V = visible(t, a.m, a.E);
        const int64_t nsel = a.dense ? V : a.k;
        const int64_t w0 = t - a.n_win + 1 < 0 ? 0 : t - a.n_win + 1;
        const int64_t nwin = a.n_win > 0 ? t - w0 + 1 : 0;
        const int64_t NK = nsel + nwin;
        const int64_t wp0 = a.win_pos0 ? a.win_pos0[b] : 0;
        const int ntiles = (int)((NK + KT - 1) / KT);

        // queries of this token -> sQ (K-major, 128-byte swizzle, 8 blocks of 64 dims)
        for (int ch = tid; ch < H * 64; ch += kThreads) {
            const int hh = ch >> 6, c16 = ch & 63;
            uint8_t *dst = sQ + (c16 >> 3) * (H * 128) + hh * 128 + (((c16 & 7) ^ (hh & 7)) << 4);
            tc::cp_async16(dst, a.q + (bt * H + hh) * DIM + c16 * 8, 16);
        }
        for (int hh = tid; hh < H; hh += kThreads)
            m_run[hh] = -INFINITY;
        float lpart[H];
#pragma unroll
        for (int hh = 0; hh < H; hh++)
            lpart[hh] = 0.f;

        for (int it = 0; it < ntiles; ++it, ++g) {
            // the previous tile's products must be done with sK / sP; every
            // thread takes the same decision, so a timeout never splits the block
            const bool prev_done = g == 0 || tc::mbar_wait(obar, (g - 1) & 1, abort_flag);
            if (!__syncthreads_and(prev_done)) {
                ok = false;
                break;
            }
            const int64_t j = (int64_t)it * KT + tid;
            const __nv_bfloat16 *src = nullptr;
            if (j < NK) {
                if (j < nsel) {
                    const int64_t s = a.dense ? j : (int64_t)a.idx[bt * a.k + j];
                    if (s >= 0) {
                        if (s < V)
                            src = a.ent + (b * a.E + s) * DIM;
                        else
                            report(a.err, CSA_ERR_BOUNDS, K_ATTEND_TC, (unsigned)bt, (unsigned)s);
                    }
                } else {
                    const int64_t p = w0 + (j - nsel);
                    const int64_t wr = p - wp0;
                    if (wr >= 0 && wr < a.win_rows)
                        src = a.kwin + (b * a.win_rows + wr) * DIM;
                    else
                        report(a.err, CSA_ERR_BOUNDS, K_ATTEND_TC, (unsigned)bt, (unsigned)p);
                }
            }
            const bool valid = src != nullptr;
            kptr[tid] = src;
            __syncthreads();
            // gather the 128 keys: rows of 64 16-byte chunks, coalesced per row
#pragma unroll 4
            for (int itc = 0; itc < 64; ++itc) {
                const int lin = itc * kThreads + tid;
                const int r = lin >> 6, c16 = lin & 63;
                const __nv_bfloat16 *sp = kptr[r];
                uint8_t *dst = sK + (c16 >> 3) * 16384 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
                tc::cp_async16(dst, sp ? (const void *)(sp + c16 * 8) : (const void *)a.ent,
                               sp ? 16u : 0u);
            }
            tc::cp_async_wait_all();
            tc::fence_async_shared();
            __syncthreads();

            // S^T = K Q^T
            if (tid == 0) {
                tc::fence_after();
#pragma unroll 1
                for (int kb = 0; kb < 8; kb++) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint64_t ad = tc::sdesc_sw128(sK_a + kb * 16384 + kk * 32);
                        const uint64_t bd = tc::sdesc_sw128(sQ_a + kb * (H * 128) + kk * 32);
                        tc::mma_f16(tmem, ad, bd, L::IDESC_S, (kb | kk) != 0);
                    }
                }
                tc::mma_commit(sbar);
            }
            if (!__syncthreads_and(tc::mbar_wait(sbar, g & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc::fence_after();
            float z[H];
            load_cols<H>(lane_tm, z);
            int need = 0;
#pragma unroll
            for (int hh = 0; hh < H; hh++) {
                z[hh] = valid ? z[hh] * a.scale : -INFINITY;
                need |= z[hh] > m_run[hh] + kLazy;
            }
            if (__syncthreads_or(need)) {
                // exact per-head maxima of this tile, then rescale what came before
#pragma unroll
                for (int hh = 0; hh < H; hh++) {
                    float v = z[hh];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                    if (lane == 0)
                        red[warp * H + hh] = v;
                }
                __syncthreads();
                for (int hh = tid; hh < H; hh += kThreads) {
                    const float tmax = fmaxf(fmaxf(red[hh], red[H + hh]),
                                             fmaxf(red[2 * H + hh], red[3 * H + hh]));
                    const float mo = m_run[hh];
                    const float mn = fmaxf(mo, tmax);
                    alpha[hh] = (mn == -INFINITY) ? 1.f : __expf(mo - mn);
                    m_run[hh] = mn;
                }
                __syncthreads();
                if (it > 0) {
                    // every earlier product has completed (waited above)
#pragma unroll 1
                    for (int jt = 0; jt < 4; jt++)
                        scale_cols<H>(lane_tm + H + jt * H, alpha);
                }
#pragma unroll
                for (int hh = 0; hh < H; hh++)
                    lpart[hh] *= alpha[hh];
            }
            // probabilities -> P^T (K-major rows = heads, 2 blocks of 64 keys)
            {
                uint8_t *prow = sP + (tid >> 6) * (H * 128) + (tid & 7) * 2;
                const int chunk = (tid & 63) >> 3;
#pragma unroll
                for (int hh = 0; hh < H; hh++) {
                    const float p = valid ? __expf(z[hh] - m_run[hh]) : 0.f;
                    const __nv_bfloat16 pb = __float2bfloat16_rn(p);
                    lpart[hh] += __bfloat162float(pb);
                    *(__nv_bfloat16 *)(prow + hh * 128 + ((chunk ^ (hh & 7)) << 4)) = pb;
                }
            }
            tc::fence_async_shared();
            tc::fence_before();
            __syncthreads();

            // O^T += K^T P^T
            if (tid == 0) {
                tc::fence_after();
#pragma unroll 1
                for (int jt = 0; jt < 4; jt++) {
#pragma unroll
                    for (int kk = 0; kk < 8; kk++) {
                        const uint64_t ad =
                            tc::sdesc_sw128_mn(sK_a + (2 * jt) * 16384 + kk * 2048, 16384, 1024);
                        const uint64_t bd =
                            tc::sdesc_sw128(sP_a + (kk >> 2) * (H * 128) + (kk & 3) * 32);
                        tc::mma_f16(tmem + H + jt * H, ad, bd, L::IDESC_O, (it > 0) || (kk > 0));
                    }
                }
                tc::mma_commit(obar);
            }
        }
        if (!ok)
            break;

        // ---- end of the query: normaliser, sink, output
        const bool last_done = ntiles == 0 || tc::mbar_wait(obar, (g - 1) & 1, abort_flag);
        if (!__syncthreads_and(last_done)) {
            ok = false;
            break;
        }
        tc::fence_after();
#pragma unroll
        for (int hh = 0; hh < H; hh++) {
            float v = lpart[hh];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0)
                red[warp * H + hh] = v;
        }
        __syncthreads();
        for (int hh = tid; hh < H; hh += kThreads) {
            const float l = red[hh] + red[H + hh] + red[2 * H + hh] + red[3 * H + hh];
            const float mo = m_run[hh];
            const float zs = a.sink[hh];
            float f, lse;
            if (zs == INFINITY) {
                f = 0.f;
                lse = INFINITY;
            } else {
                const float M = fmaxf(mo, zs);
                if (M == -INFINITY) {
                    f = 0.f;
                    lse = -INFINITY;
                } else {
                    const float e = __expf(mo - M);
                    const float den = l * e + __expf(zs - M);
                    f = e / den;
                    lse = M + __logf(den);
                }
            }
            if (ntiles == 0)
                f = 0.f;
            fin[hh] = f;
            if (a.lse)
                a.lse[bt * H + hh] = lse;
        }
        __syncthreads();
        // O^T (lane = dim within a 128-dim block) -> sK as [H][512] bf16 -> out
        __nv_bfloat16 *so = (__nv_bfloat16 *)sK;
#pragma unroll 1
        for (int jt = 0; jt < 4; jt++) {
#pragma unroll 1
            for (int c = 0; c < H / 16; c++) {
                uint32_t r[16];
                if (ntiles > 0) {
                    tc::tmem_ld16(lane_tm + H + jt * H + c * 16, r);
                    tc::tmem_ld_wait();
                }
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int hh = c * 16 + j;
                    const float o = ntiles > 0 ? __uint_as_float(r[j]) * fin[hh] : 0.f;
                    so[hh * DIM + jt * 128 + tid] = __float2bfloat16_rn(o);
                }
            }
        }
        tc::fence_before();
        __syncthreads();
        const uint4 *vs = (const uint4 *)so;
        uint4 *vd = (uint4 *)(a.out + bt * H * DIM);
        for (int v = tid; v < H * DIM / 8; v += kThreads)
            vd[v] = vs[v];
        __syncthreads();
    }

    tc::cp_async_wait_all();
    if (!ok) {
        *abort_flag = 1;
        report(a.err, CSA_ERR_TIMEOUT, K_ATTEND_TC, blockIdx.x, g);
    }
    if (tid == 0) {
        // every product issued above has completed once `done` flips
        tc::mma_commit(done);
        volatile int never = 0;
        static_cast<void>(tc::mbar_wait(done, 0, &never, 200000000ull));
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int H>
cudaError_t launch_h(const AttendArgs &a, unsigned *err, cudaStream_t s)
{
    TcAttn t;
    t.q = (const __nv_bfloat16 *)a.q;
    t.ent = (const __nv_bfloat16 *)a.kv.body;
    t.idx = a.idx;
    t.dense = a.dense;
    t.k = a.k;
    t.m = a.m;
    t.E = a.E;
    t.kwin = (const __nv_bfloat16 *)a.kwin;
    t.win_rows = a.win_rows;
    t.win_pos0 = a.win_pos0;
    t.n_win = a.n_win;
    t.q_pos = a.q_pos;
    t.sink = a.sink;
    t.n_q = a.n_q;
    t.nqueries = (int64_t)a.B * a.n_q;
    t.scale = a.scale;
    t.out = (__nv_bfloat16 *)a.out;
    t.lse = a.lse;
    t.err = err;
    const size_t smem = Lay<H>::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = t.nqueries < sms ? t.nqueries : sms;
    attend_tc_kernel<H><<<(unsigned)grid, kThreads, smem, s>>>(t);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const AttendArgs &a, unsigned *err, cudaStream_t s, bool *taken)
{
    *taken = false;
    if (a.q_dt != CSA_BF16 || a.kv.dt != CSA_BF16 || a.kv.c != DIM)
        return cudaSuccess;
    if (a.h != 16 && a.h != 32 && a.h != 64)
        return cudaSuccess;
    if (a.n_win > 0 && !a.kwin)
        return cudaSuccess;
    *taken = true;
    switch (a.h) {
    case 16: return launch_h<16>(a, err, s);
    case 32: return launch_h<32>(a, err, s);
    default: return launch_h<64>(a, err, s);
    }
}

}  // namespace csa
