// attend_tc.cu -- shared-KV multi-query attention with window and sink on the
// 5th-generation tensor cores (CSA Eq. 18-19, HCA Eq. 24-26, Module D).
//
// All H heads of a query share one key set, and every key is also its own
// value. Keys therefore go on the M axis of both contractions:
//   S^T[key][head]  = sum_d K[key][d] * Q[head][d]        (M = 128 keys, N = H)
//   O^T[dim][head] += sum_key K[key][dim] * P^T[key][head] (M = 4 x 128 dims, N = H)
// One 128 x 512 bf16 key tile in shared memory (8 blocks of 64 dims, 128-byte
// swizzle) is the K-major A operand of the first product and, read along the
// other axis, the M/N-major A operand of the second. S^T and O^T live in
// tensor memory (H + 4H columns).
//
// Warp roles (one persistent block per SM looping over queries):
//  * warps 0-3 gather the key rows of each tile (selected entries, or window
//    rows) with 16-byte cp.async, block by block, keeping up to four 16 KB
//    blocks in flight per thread; block pair (2j, 2j+1) of the next tile is
//    refetched as soon as the O^T product of M-tile j has consumed it. One
//    thread also loads each query's Q with a tiled TMA copy.
//  * warp 4 allocates tensor memory and issues the MMAs (S^T block by block
//    as blocks land, then O^T per M-tile), committing to the barriers the
//    other roles wait on.
//  * warps 5.. (four per group of 16 heads) own the TMEM lanes (one key, then
//    one dim, per thread): softmax of each tile into P^T for their heads, and
//    the normalisation and output of each query.
// Softmax: the per-head offset m_h is updated lazily -- only when some logit
// of a tile exceeds m_h + 8 are the tile's maxima of that head group reduced,
// its O^T columns rescaled in tensor memory and its partial sums rescaled (the
// first tile always takes this path). Probabilities are rounded to bf16 for
// the second product and the normaliser sums the rounded values. The sink
// joins the final normalisation only.
// Every wait is bounded; on expiry the block records CSA_ERR_TIMEOUT, lets its
// own copies and products land, frees its tensor memory and returns.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma_host.h"

namespace csa {

namespace {

constexpr int DIM = 512;
constexpr int KT = 128;
constexpr float kLazy2 = 11.5f;     // lazy-rescale margin, base-2 units (about e^8)
constexpr int kMmaWarp = 4;
constexpr int kSoftWarp0 = 5;
constexpr int kGatherBar = 5;        // named barrier of the 4 gather warps (1..4: head groups)
constexpr int kInFlight = 3;         // 16 KB blocks a gather thread may leave in flight

struct TcAttn {
    const __nv_bfloat16 *ent, *kwin;
    const uint8_t *ent8;             // fp8 layout: e4m3 body [rows, 448]
    const float *ent_scale;          //   one scale per 64 body dims [rows, 7]
    const __nv_bfloat16 *ent_rope;   //   bf16 RoPE dims [rows, 64]
    int nchunks, tpc;                // split of each query's key tiles over work items
    float *ws_o, *ws_ml;             // partial O [item][H][512] and (m, l) [item][H][2]
    const int32_t *idx;
    int dense, k, m;
    int tma_ent, tma_win;            // whole-tile TMA boxes available per source
    int64_t E;
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

// 2^x and log2(x) from the special-function unit (approximate, about 2 ulp).
__device__ __forceinline__ float fast_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float fast_lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int H>
struct Lay {
    static constexpr int NG = H / 16;                               // head groups
    static constexpr int THREADS = 32 * (kSoftWarp0 + 4 * NG);
    static constexpr size_t K_OFF = 0;                              // 8 x 16 KB
    static constexpr size_t Q_OFF = 8 * 16384;                      // 8 x H x 128
    static constexpr size_t P_OFF = Q_OFF + 8 * H * 128;            // 2 x H x 128
    static constexpr size_t PTR_OFF = P_OFF + 2 * H * 128;          // 128 row pointers
    static constexpr size_t ROW_OFF = PTR_OFF + KT * 8;             // 128 fp8 entry rows
    static constexpr size_t F_OFF = ROW_OFF + KT * 8;               // m, red[4], fin
    static constexpr size_t BAR_OFF = F_OFF + ((8 * H * 4 + 63) / 64) * 64;
    static constexpr size_t TOTAL = BAR_OFF + 256;
    static constexpr uint32_t TMEM_COLS = (5 * H <= 128) ? 128 : (5 * H <= 256 ? 256 : 512);
    static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, H, 0, 0);
    static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, H, 1, 0);
};

// Per-work-item quantities (a query, or one chunk of a query's key tiles),
// computed identically by every role.
struct QInfo {
    int64_t b, t, V, nsel, nwin, w0, wp0, nk;
    int64_t wbeg;     // first window slot: nsel rounded up to 8 (8-slot groups never mix)
    int ntiles;       // tiles of this item
    int tile0;        // first key tile of this item
};

__device__ __forceinline__ QInfo query_info(const TcAttn &a, int64_t bt, int chunk)
{
    QInfo q;
    q.b = bt / a.n_q;
    q.t = a.q_pos[bt];
    q.V = visible(q.t, a.m, a.E);
    q.nsel = a.dense ? q.V : a.k;
    q.w0 = q.t - a.n_win + 1 < 0 ? 0 : q.t - a.n_win + 1;
    q.nwin = a.n_win > 0 ? q.t - q.w0 + 1 : 0;
    q.wp0 = a.win_pos0 ? a.win_pos0[q.b] : 0;
    q.wbeg = (q.nsel + 7) & ~(int64_t)7;
    q.nk = q.wbeg + q.nwin;
    const int all = (int)((q.nk + KT - 1) / KT);
    q.tile0 = chunk * a.tpc;
    int end = q.tile0 + a.tpc;
    if (end > all)
        end = all;
    q.ntiles = end > q.tile0 ? end - q.tile0 : 0;
    return q;
}

// Source row of key slot j of a query (NULL: empty slot or out of range).
// `report_bad` records a selection index or window position out of range.
// With the fp8 entry layout, an entry comes back as *entry_row >= 0 (its row
// in the cache) and a NULL pointer stands for "not a bf16 row".
template <bool KV8>
__device__ __forceinline__ const __nv_bfloat16 *key_row(const TcAttn &a, const QInfo &q,
                                                        int64_t bt, int64_t j, bool report_bad,
                                                        int64_t *entry_row)
{
    *entry_row = -1;
    if (j < q.nsel) {
        const int64_t s = a.dense ? j : (int64_t)a.idx[bt * a.k + j];
        if (s < 0)
            return nullptr;
        if (s < q.V) {
            if (KV8) {
                *entry_row = q.b * a.E + s;
                return nullptr;
            }
            return a.ent + (q.b * a.E + s) * DIM;
        }
        if (report_bad)
            report(a.err, CSA_ERR_BOUNDS, K_ATTEND_TC, (unsigned)bt, (unsigned)s);
        return nullptr;
    }
    if (j >= q.wbeg && j < q.nk) {
        const int64_t p = q.w0 + (j - q.wbeg);
        const int64_t wr = p - q.wp0;
        if (wr >= 0 && wr < a.win_rows)
            return a.kwin + (q.b * a.win_rows + wr) * DIM;
        if (report_bad)
            report(a.err, CSA_ERR_BOUNDS, K_ATTEND_TC, (unsigned)bt, (unsigned)p);
    }
    return nullptr;
}

template <int H, bool KV8>
__global__ void __launch_bounds__(Lay<H>::THREADS, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ent,
                 const __grid_constant__ CUtensorMap tm_win, const TcAttn a)
{
    using L = Lay<H>;
    constexpr int NG = L::NG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sK = sm + L::K_OFF;
    uint8_t *sQ = sm + L::Q_OFF;
    uint8_t *sP = sm + L::P_OFF;
    const __nv_bfloat16 **kptr = (const __nv_bfloat16 **)(sm + L::PTR_OFF);
    int64_t *krow = (int64_t *)(sm + L::ROW_OFF);
    float *m_run = (float *)(sm + L::F_OFF);     // [H]
    float *red = m_run + H;                      // [4][H]
    float *sink2 = red + 4 * H;                  // [H] sink logits, base-2 units
    float *m_new = sink2 + H;                    // [H] offsets after a rescale
    float *alpha_s = m_new + H;                  // [H] rescale factors
    uint64_t *bars = (uint64_t *)(sm + L::BAR_OFF);
    uint64_t *kfull = bars;          // [8] key block landed (128 gather arrivals)
    uint64_t *kfree = bars + 8;      // [4] block pair consumed by O^T M-tile j
    uint64_t *qfull = bars + 12, *qfree = bars + 13, *sfull = bars + 14, *pfull = bars + 15;
    uint64_t *ofull = bars + 16, *ofree = bars + 17, *done = bars + 18;
    uint32_t *tmem_slot = (uint32_t *)(bars + 19);
    int *abort_flag = (int *)(tmem_slot + 1);
    const int64_t nitems = a.nqueries * a.nchunks;
    const bool split = a.nchunks > 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 8; i++)
            tc::mbar_init(&kfull[i], 128);
        for (int i = 0; i < 4; i++)
            tc::mbar_init(&kfree[i], 1);
        tc::mbar_init(qfull, 1);
        tc::mbar_init(qfree, 1);
        tc::mbar_init(sfull, 1);
        tc::mbar_init(pfull, 128 * NG);
        tc::mbar_init(ofull, 1);
        tc::mbar_init(ofree, 128 * NG);
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
        tc::tma_prefetch_desc(&tm_q);
        tc::tma_prefetch_desc(&tm_ent);
        tc::tma_prefetch_desc(&tm_win);
    }
    for (int hh = tid; hh < H; hh += blockDim.x) {
        sink2[hh] = a.sink[hh] * 1.4426950408889634f;
        m_run[hh] = -INFINITY;
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(tmem_slot, L::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int *abortv = abort_flag;

    if (warp < 4) {
        // ------------------------------------------------------------ gather
        const int gt = tid;                          // 0..127
        const void *zero_src = KV8 ? (a.kwin ? (const void *)a.kwin : (const void *)a.ent8)
                                   : (a.E > 0 ? (const void *)a.ent : (const void *)a.kwin);
        uint32_t tctr = 0, qctr = 0, issued = 0, arrived = 0;
        bool ok = true;
        // announce every block still in flight: required before any wait on
        // a barrier that the products of those blocks release
        auto flush = [&]() {
            tc::cp_async_wait_group<0>();
            tc::fence_async_shared();
            for (; arrived < issued; ++arrived)
                tc::mbar_arrive(&kfull[arrived & 7]);
        };
        for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
            const int64_t bt = w / a.nchunks;
            const QInfo q = query_info(a, bt, (int)(w % a.nchunks));
            flush();
            const bool qf = qctr == 0 || tc::mbar_wait(qfree, (qctr - 1) & 1, abortv);
            if (tc::named_bar_or(kGatherBar, 128, !qf)) {
                ok = false;
                break;
            }
            if (gt == 0) {
                tc::mbar_arrive_expect_tx(qfull, (uint32_t)(H * 1024));
                for (int kb = 0; kb < 8; kb++)
                    tc::tma_load_2d(sQ + kb * (H * 128), &tm_q, qfull, kb * 64, (int)(bt * H));
            }
            for (int i = 0; i < q.ntiles && ok; ++i, ++tctr) {
                flush();
                int64_t er;
                const int64_t jt0 = (int64_t)(q.tile0 + i) * KT;
                const __nv_bfloat16 *kp = key_row<KV8>(a, q, bt, jt0 + gt, false, &er);
                kptr[gt] = kp;
                krow[gt] = er;
                // A tile whose 128 rows are consecutive rows of one bf16 source
                // (dense entries, a selection that is a run, window positions)
                // goes by one tiled TMA box per 64-dim slice; any other tile by
                // per-thread 16-byte copies.
                int tma_src = 0, tma_row = 0;
                {
                    int64_t er0;
                    const __nv_bfloat16 *p0 = key_row<KV8>(a, q, bt, jt0, false, &er0);
                    const bool src_ent = jt0 < q.nsel, src_win = jt0 >= q.wbeg;
                    const bool same = (jt0 + gt < q.nsel) == src_ent && (jt0 + gt >= q.wbeg) == src_win;
                    bool run = p0 != nullptr && same && kp == p0 + (int64_t)gt * DIM;
                    const __nv_bfloat16 *base = src_ent ? a.ent : a.kwin;
                    const int64_t row0 = p0 ? (p0 - base) / DIM : 0;
                    run = run && row0 <= 0x7fffffff - KT && (src_ent ? a.tma_ent : a.tma_win);
                    const bool all_run = !tc::named_bar_or(kGatherBar, 128, !run);
                    if (all_run) {
                        tma_src = src_ent ? 1 : 2;
                        tma_row = (int)row0;
                    }
                }
                for (int kb = 0; kb < 8; kb++) {
                    if ((kb & 1) == 0 && tctr > 0) {
                        const bool fr = tc::mbar_wait(&kfree[kb >> 1], (tctr - 1) & 1, abortv);
                        if (tc::named_bar_or(kGatherBar, 128, !fr)) {
                            ok = false;
                            break;
                        }
                    }
                    if (tma_src != 0) {
                        if (gt == 0) {
                            tc::mbar_expect_tx(&kfull[kb], 16384u);
                            tc::tma_load_2d(sK + kb * 16384, tma_src == 1 ? &tm_ent : &tm_win,
                                            &kfull[kb], kb * 64, tma_row);
                        }
                        tc::cp_async_commit();
                        ++issued;
                        if (issued - arrived > kInFlight) {
                            tc::cp_async_wait_group<kInFlight>();
                            tc::fence_async_shared();
                            tc::mbar_arrive(&kfull[arrived & 7]);
                            ++arrived;
                        }
                        continue;
                    }
                    // fp8 entries: all eight code loads of this block go out
                    // before any is converted, so their latencies overlap
                    int64_t er8[8];
                    uint2 cw[8];
                    float sc8[8];
#pragma unroll
                    for (int u = 0; u < 8; u++) {
                        const int r = (u * 128 + gt) >> 3, c = gt & 7;
                        er8[u] = KV8 ? krow[r] : -1;
                        if (KV8 && kb < 7 && er8[u] >= 0) {
                            cw[u] = __ldg((const uint2 *)(a.ent8 + er8[u] * 448 + kb * 64 + c * 8));
                            sc8[u] = __ldg(a.ent_scale + er8[u] * 7 + kb);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 8; u++) {
                        const int lin = u * 128 + gt;
                        const int r = lin >> 3, c = lin & 7;
                        uint8_t *dst = sK + kb * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
                        if (KV8 && er8[u] >= 0) {
                            if (kb < 7) {
                                // 8 e4m3 codes of one 64-dim scale group -> 8 bf16
                                const uint16_t *c2 = (const uint16_t *)&cw[u];
                                __nv_bfloat162 o[4];
#pragma unroll
                                for (int e = 0; e < 4; e++) {
                                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                                        (__nv_fp8x2_storage_t)c2[e], __NV_E4M3);
                                    const float2 f = __half22float2(__half2(hr));
                                    o[e] = __floats2bfloat162_rn(f.x * sc8[u], f.y * sc8[u]);
                                }
                                *(uint4 *)dst = *(const uint4 *)o;
                            } else {
                                tc::cp_async16(dst, a.ent_rope + er8[u] * 64 + c * 8, 16u);
                            }
                        } else {
                            const __nv_bfloat16 *sp = kptr[r];
                            tc::cp_async16(dst, sp ? (const void *)(sp + kb * 64 + c * 8) : zero_src,
                                           sp ? 16u : 0u);
                        }
                    }
                    tc::cp_async_commit();
                    ++issued;
                    if (issued - arrived > kInFlight) {
                        tc::cp_async_wait_group<kInFlight>();
                        tc::fence_async_shared();
                        tc::mbar_arrive(&kfull[arrived & 7]);
                        ++arrived;
                    }
                }
                tc::named_bar_sync(kGatherBar, 128);     // kptr / krow rewritten next tile
            }
        }
        flush();
        if (!ok) {
            *abort_flag = 1;
            report(a.err, CSA_ERR_TIMEOUT, K_ATTEND_TC, blockIdx.x, 0);
        }
        if (gt == 0 && qctr > 0) {
            volatile int never = 0;
            static_cast<void>(tc::mbar_wait(qfull, (qctr - 1) & 1, &never, 200000000ull));
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            uint32_t tctr = 0, qctr = 0;
            bool ok = true;
            const uint32_t sK_a = tc::smem_u32(sK), sQ_a = tc::smem_u32(sQ), sP_a = tc::smem_u32(sP);
            const uint64_t adS = tc::sdesc_sw128(sK_a), bdS = tc::sdesc_sw128(sQ_a);
            const uint64_t adO = tc::sdesc_sw128_mn(sK_a, 16384, 1024), bdO = tc::sdesc_sw128(sP_a);
            for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
                const QInfo q = query_info(a, w / a.nchunks, (int)(w % a.nchunks));
                bool ofree_done = qctr == 0;
                if (!tc::mbar_wait(qfull, qctr & 1, abortv)) {
                    ok = false;
                    break;
                }
                for (int i = 0; i < q.ntiles; ++i, ++tctr) {
                    // descriptors advance by constants: 16 KB per key block and
                    // H x 128 B per Q block (>> 4), 32 B per 16-dim step (>> 4)
#pragma unroll 1
                    for (int kb = 0; kb < 8; kb++) {
                        if (!tc::mbar_wait(&kfull[kb], tctr & 1, abortv)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
                        const uint64_t ad = adS + (uint64_t)(kb * 1024), bd = bdS + (uint64_t)(kb * (H * 8));
                        tc::mma_f16(tmem, ad, bd, L::IDESC_S, kb != 0);
#pragma unroll
                        for (int kk = 1; kk < 4; kk++)
                            tc::mma_f16(tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), L::IDESC_S, 1u);
                    }
                    if (!ok)
                        break;
                    tc::mma_commit(sfull);
                    if (i == q.ntiles - 1)
                        tc::mma_commit(qfree);
                    if (!ofree_done) {
                        if (!tc::mbar_wait(ofree, (qctr - 1) & 1, abortv)) {
                            ok = false;
                            break;
                        }
                        ofree_done = true;
                    }
                    if (!tc::mbar_wait(pfull, tctr & 1, abortv)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t acc0 = i > 0;
#pragma unroll 1
                    for (int jt = 0; jt < 4; jt++) {
                        const uint64_t ad = adO + (uint64_t)(jt * 2048);
                        const uint32_t d = tmem + H + jt * H;
                        tc::mma_f16(d, ad, bdO, L::IDESC_O, acc0);
#pragma unroll
                        for (int kk = 1; kk < 8; kk++)
                            tc::mma_f16(d, ad + (uint64_t)(kk * 128),
                                        bdO + (uint64_t)((kk >> 2) * (H * 8) + (kk & 3) * 2),
                                        L::IDESC_O, 1u);
                        tc::mma_commit(&kfree[jt]);
                    }
                }
                if (!ok)
                    break;
                if (q.ntiles == 0) {
                    tc::mma_commit(qfree);
                    if (!ofree_done && !tc::mbar_wait(ofree, (qctr - 1) & 1, abortv)) {
                        ok = false;
                        break;
                    }
                }
                tc::mma_commit(ofull);
            }
            if (!ok) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_ATTEND_TC, blockIdx.x, 1);
            }
            tc::mma_commit(done);
            volatile int never = 0;
            static_cast<void>(tc::mbar_wait(done, 0, &never, 200000000ull));
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        // Logits are kept in base-2 units, z2 = (q . k) * scale * log2(e), so
        // every probability is one ex2 of a difference; offsets m2 live in
        // registers, replicated in every thread of the head group.
        const float scale2 = a.scale * 1.4426950408889634f;
        const int g = (warp - kSoftWarp0) >> 2;         // head group: heads h0 .. h0+15
        const int h0 = 16 * g;
        const int gbar = 1 + g;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;                   // key (then dim) of this TMEM lane
        const int et = (warp - kSoftWarp0 - 4 * g) * 32 + lane;   // 0..127 inside the group
        const uint32_t lane_tm = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t tctr = 0, qctr = 0;
        bool ok = true;
        for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
            const int64_t bt = w / a.nchunks;
            const QInfo q = query_info(a, bt, (int)(w % a.nchunks));
            // running offsets m_run[h0..h0+15] (base 2) start at -inf for every item
            float lpart[16];
#pragma unroll
            for (int u = 0; u < 16; u++)
                lpart[u] = 0.f;
            for (int i = 0; i < q.ntiles; ++i, ++tctr) {
                int64_t er;
                const bool valid =
                    key_row<KV8>(a, q, bt, (int64_t)(q.tile0 + i) * KT + r, g == 0, &er) != nullptr ||
                    er >= 0;
                const bool got = tc::mbar_wait(sfull, tctr & 1, abortv);
                if (tc::named_bar_or(gbar, 128, !got)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                float z[16];
                {
                    uint32_t rr[16];
                    tc::tmem_ld16(lane_tm + h0, rr);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        z[u] = valid ? __uint_as_float(rr[u]) * scale2 : -INFINITY;
                }
                float m2[16];
#pragma unroll
                for (int u = 0; u < 16; u += 4) {
                    const float4 mv = *(const float4 *)(m_run + h0 + u);
                    m2[u] = mv.x;
                    m2[u + 1] = mv.y;
                    m2[u + 2] = mv.z;
                    m2[u + 3] = mv.w;
                }
                bool need = false;
#pragma unroll
                for (int u = 0; u < 16; u++)
                    need |= z[u] > m2[u] + kLazy2;
                if (tc::named_bar_or(gbar, 128, need)) {
#pragma unroll
                    for (int u = 0; u < 16; u++) {
                        float v = z[u];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1)
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                        if (lane == 0)
                            red[q4 * H + h0 + u] = v;
                    }
                    tc::named_bar_sync(gbar, 128);
                    // one thread per head: new offset and the factor for what is summed
                    float mn = 0.f;
                    if (et < 16) {
                        const int hh = h0 + et;
                        const float tmax = fmaxf(fmaxf(red[hh], red[H + hh]),
                                                 fmaxf(red[2 * H + hh], red[3 * H + hh]));
                        const float mo = m_run[hh];
                        mn = fmaxf(mo, tmax);
                        m_new[hh] = mn;
                        alpha_s[hh] = (mn == -INFINITY) ? 1.f : fast_ex2(mo - mn);
                    }
                    tc::named_bar_sync(gbar, 128);
                    if (et < 16)
                        m_run[h0 + et] = mn;
#pragma unroll
                    for (int u = 0; u < 16; u += 4) {
                        const float4 mv = *(const float4 *)(m_new + h0 + u);
                        m2[u] = mv.x;
                        m2[u + 1] = mv.y;
                        m2[u + 2] = mv.z;
                        m2[u + 3] = mv.w;
                    }
                    if (i > 0) {
                        // O^T of the earlier tiles is complete (S of this tile came after it)
#pragma unroll 1
                        for (int jt = 0; jt < 4; jt++) {
                            uint32_t rr[16];
                            const uint32_t ad = lane_tm + H + jt * H + h0;
                            tc::tmem_ld16(ad, rr);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int u = 0; u < 16; u++)
                                rr[u] = __float_as_uint(__uint_as_float(rr[u]) * alpha_s[h0 + u]);
                            tc::tmem_st16(ad, rr);
                        }
                        tc::tmem_st_wait();
                    }
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        lpart[u] *= alpha_s[h0 + u];
                }
                // P^T rows h0..h0+15: 2 blocks of 64 keys, 128-byte swizzle
                {
                    uint8_t *prow = sP + (r >> 6) * (H * 128) + (r & 7) * 2;
                    const int chunk = (r & 63) >> 3;
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const float p0 = valid ? fast_ex2(z[u] - m2[u]) : 0.f;
                        const float p1 = valid ? fast_ex2(z[u + 1] - m2[u + 1]) : 0.f;
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        const float2 pr = __bfloat1622float2(pb);
                        lpart[u] += pr.x;
                        lpart[u + 1] += pr.y;
                        const int hh = h0 + u;
                        *(__nv_bfloat16 *)(prow + hh * 128 + ((chunk ^ (hh & 7)) << 4)) = pb.x;
                        *(__nv_bfloat16 *)(prow + (hh + 1) * 128 + ((chunk ^ ((hh + 1) & 7)) << 4)) = pb.y;
                    }
                }
                tc::fence_async_shared();
                tc::fence_before();
                tc::mbar_arrive(pfull);
            }
            if (!ok)
                break;
            // ---- end of the item: normaliser, sink, output for heads h0..h0+15
#pragma unroll
            for (int u = 0; u < 16; u++) {
                float v = lpart[u];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0)
                    red[q4 * H + h0 + u] = v;
            }
            tc::named_bar_sync(gbar, 128);
            float f[16];
#pragma unroll
            for (int u = 0; u < 16; u++) {
                const int hh = h0 + u;
                const float l = red[hh] + red[H + hh] + red[2 * H + hh] + red[3 * H + hh];
                if (split) {
                    // partial of this key chunk: raw accumulator, offset (natural units), sum
                    f[u] = 1.f;
                    if (et == u) {
                        a.ws_ml[(w * H + hh) * 2] = m_run[hh] * 0.6931471805599453f;
                        a.ws_ml[(w * H + hh) * 2 + 1] = l;
                    }
                    continue;
                }
                const float zs2 = sink2[hh];
                float fu, lse;
                if (zs2 == INFINITY) {
                    fu = 0.f;
                    lse = INFINITY;
                } else {
                    const float mh = m_run[hh];
                    const float M2 = fmaxf(mh, zs2);
                    if (M2 == -INFINITY) {
                        fu = 0.f;
                        lse = -INFINITY;
                    } else {
                        const float e = fast_ex2(mh - M2);
                        const float den = l * e + fast_ex2(zs2 - M2);
                        fu = e / den;
                        lse = (M2 + fast_lg2(den)) * 0.6931471805599453f;
                    }
                }
                f[u] = q.ntiles > 0 ? fu : 0.f;
                if (et == u && a.lse)
                    a.lse[bt * H + hh] = lse;
            }
            const bool got = tc::mbar_wait(ofull, qctr & 1, abortv);
            if (tc::named_bar_or(gbar, 128, !got)) {
                ok = false;
                break;
            }
            tc::fence_after();
#pragma unroll 1
            for (int jt = 0; jt < 4; jt++) {
                float o[16];
                if (q.ntiles > 0) {
                    uint32_t rr[16];
                    tc::tmem_ld16(lane_tm + H + jt * H + h0, rr);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        o[u] = __uint_as_float(rr[u]) * f[u];
                } else {
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        o[u] = 0.f;
                }
                if (split) {
                    float *orow = a.ws_o + (w * H) * DIM + jt * 128 + r;
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        orow[(h0 + u) * DIM] = o[u];
                } else {
                    // lanes r and r^1 swap halves so that each stores bf16 pairs of
                    // adjacent dims: even lanes heads h0..h0+7, odd lanes h0+8..h0+15
                    const bool odd = lane & 1;
                    __nv_bfloat162 *orow = (__nv_bfloat162 *)(a.out + bt * H * DIM + jt * 128 + (r & ~1));
#pragma unroll
                    for (int u = 0; u < 8; u++) {
                        const float mine = odd ? o[u + 8] : o[u];
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? o[u] : o[u + 8], 1);
                        const int hh = h0 + (odd ? u + 8 : u);
                        orow[hh * (DIM / 2)] = odd ? __floats2bfloat162_rn(other, mine)
                                                   : __floats2bfloat162_rn(mine, other);
                    }
                }
            }
            tc::fence_before();
            tc::mbar_arrive(ofree);
            tc::named_bar_sync(gbar, 128);     // red and m_run reused next item
            if (et < 16)
                m_run[h0 + et] = -INFINITY;
        }
        if (!ok) {
            *abort_flag = 1;
            report(a.err, CSA_ERR_TIMEOUT, K_ATTEND_TC, blockIdx.x, 2);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// Joins the key chunks of each (query, head): out = sum_c O_c e^{m_c - M} /
// (sum_c l_c e^{m_c - M} + e^{z' - M}), M = max(max_c m_c, z'), the sink z'
// entering once here.
__global__ void __launch_bounds__(128)
combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_ml, int nchunks, int H,
               const float *__restrict__ sink, __nv_bfloat16 *__restrict__ out,
               float *__restrict__ lse)
{
    const int64_t bt = blockIdx.x;
    const int hh = blockIdx.y;
    const float zs = sink[hh];
    float M = zs;
    for (int c = 0; c < nchunks; c++)
        M = fmaxf(M, ws_ml[((bt * nchunks + c) * H + hh) * 2]);
    float den = 0.f, l_out;
    const bool zero = zs == INFINITY || M == -INFINITY;
    if (!zero) {
        den = __expf(zs - M);
        for (int c = 0; c < nchunks; c++) {
            const float *ml = ws_ml + ((bt * nchunks + c) * H + hh) * 2;
            if (ml[0] != -INFINITY)
                den += ml[1] * __expf(ml[0] - M);
        }
        l_out = M + __logf(den);
    } else {
        l_out = zs == INFINITY ? INFINITY : -INFINITY;
    }
    for (int d = threadIdx.x; d < DIM; d += blockDim.x) {
        float o = 0.f;
        if (!zero) {
            for (int c = 0; c < nchunks; c++) {
                const float mc = ws_ml[((bt * nchunks + c) * H + hh) * 2];
                if (mc != -INFINITY)
                    o += ws_o[((bt * nchunks + c) * H + hh) * DIM + d] * __expf(mc - M);
            }
            o /= den;
        }
        out[(bt * H + hh) * DIM + d] = __float2bfloat16_rn(o);
    }
    if (threadIdx.x == 0 && lse)
        lse[bt * H + hh] = l_out;
}

// Split of each query's key tiles over work items when there are too few
// queries to fill the GPU: about two items per SM.
void split_plan(int64_t nq, int64_t max_keys, int *nchunks, int *tpc)
{
    const int64_t tiles = (max_keys + KT - 1) / KT;
    *nchunks = 1;
    *tpc = 1 << 28;
    if (nq <= 0 || nq >= 74 || tiles <= 1)
        return;
    int64_t want = (296 + nq - 1) / nq;
    if (want > tiles)
        want = tiles;
    const int64_t t = (tiles + want - 1) / want;
    *tpc = (int)t;
    *nchunks = (int)((tiles + t - 1) / t);
}

template <int H, bool KV8>
cudaError_t launch_h(const AttendArgs &a, unsigned *err, cudaStream_t s)
{
    CUtensorMap tm_q;
    if (!make_tmap_2d(&tm_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.n_q * H,
                      DIM, H))
        return cudaErrorInvalidValue;
    // whole-tile boxes (KT rows) of the bf16 entries and of the window rows,
    // for tiles that are one run of consecutive rows
    CUtensorMap tm_ent, tm_win;
    const uint64_t ent_rows = (uint64_t)a.B * a.E, win_rows = (uint64_t)a.B * a.win_rows;
    const bool have_ent = !KV8 && ent_rows >= (uint64_t)KT;
    const bool have_win = a.n_win > 0 && win_rows >= (uint64_t)KT;
    if (have_ent && !make_tmap_2d(&tm_ent, a.kv.body, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ent_rows,
                                  DIM, KT))
        return cudaErrorInvalidValue;
    if (have_win && !make_tmap_2d(&tm_win, a.kwin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, win_rows,
                                  DIM, KT))
        return cudaErrorInvalidValue;
    if (!have_ent)
        tm_ent = have_win ? tm_win : tm_q;
    if (!have_win)
        tm_win = tm_ent;
    TcAttn t;
    t.ent = KV8 ? nullptr : (const __nv_bfloat16 *)a.kv.body;
    t.ent8 = KV8 ? (const uint8_t *)a.kv.body : nullptr;
    t.ent_scale = KV8 ? a.kv.scale : nullptr;
    t.ent_rope = KV8 ? (const __nv_bfloat16 *)a.kv.rope : nullptr;
    t.kwin = (const __nv_bfloat16 *)a.kwin;
    t.idx = a.idx;
    t.dense = a.dense;
    t.tma_ent = have_ent;
    t.tma_win = have_win;
    t.k = a.k;
    t.m = a.m;
    t.E = a.E;
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
    split_plan(t.nqueries, (a.dense ? a.E : a.k) + a.n_win, &t.nchunks, &t.tpc);
    t.ws_o = (float *)a.ws;
    t.ws_ml = t.nchunks > 1 ? t.ws_o + (size_t)t.nqueries * t.nchunks * H * DIM : nullptr;
    if (t.nchunks > 1 && !a.ws)
        return cudaErrorInvalidValue;
    const size_t smem = Lay<H>::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<H, KV8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = t.nqueries * t.nchunks;
    const int64_t grid = items < sms ? items : sms;
    attend_tc_kernel<H, KV8><<<(unsigned)grid, Lay<H>::THREADS, smem, s>>>(tm_q, tm_ent, tm_win, t);
    e = cudaGetLastError();
    if (e != cudaSuccess || t.nchunks == 1)
        return e;
    combine_kernel<<<dim3((unsigned)t.nqueries, H), 128, 0, s>>>(t.ws_o, t.ws_ml, t.nchunks, H,
                                                                   a.sink, t.out, a.lse);
    return cudaGetLastError();
}

bool takes_fp8(const AttendArgs &a)
{
    return a.kv.dt == CSA_E4M3 && a.kv.rope_dims == 64 && a.kv.scale_group == 64 &&
           a.kv.rope != nullptr;
}

}  // namespace

size_t attend_tc_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys)
{
    if (c != DIM || (h != 16 && h != 32 && h != 64))
        return 0;
    int nchunks, tpc;
    split_plan((int64_t)B * n_q, max_keys, &nchunks, &tpc);
    if (nchunks <= 1)
        return 0;
    return (size_t)B * n_q * nchunks * h * (DIM + 2) * sizeof(float);
}

cudaError_t launch_attend_tc(const AttendArgs &a, unsigned *err, cudaStream_t s, bool *taken)
{
    *taken = false;
    if (a.q_dt != CSA_BF16 || a.kv.c != DIM)
        return cudaSuccess;
    const bool fp8 = takes_fp8(a);
    if (a.kv.dt != CSA_BF16 && !fp8)
        return cudaSuccess;
    if (a.h != 16 && a.h != 32 && a.h != 64)
        return cudaSuccess;
    if (a.E <= 0 && (a.n_win == 0 || a.win_rows <= 0))
        return cudaSuccess;
    if ((int64_t)a.B * a.n_q * a.h >= INT32_MAX)     // TMA row coordinate of Q
        return cudaSuccess;
    *taken = true;
    if (fp8) {
        switch (a.h) {
        case 16: return launch_h<16, true>(a, err, s);
        case 32: return launch_h<32, true>(a, err, s);
        default: return launch_h<64, true>(a, err, s);
        }
    }
    switch (a.h) {
    case 16: return launch_h<16, false>(a, err, s);
    case 32: return launch_h<32, false>(a, err, s);
    default: return launch_h<64, false>(a, err, s);
    }
}

}  // namespace csa
