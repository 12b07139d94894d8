// attend_tc.cu -- shared-KV multi-query attention with window and sink on the
// 5th-generation tensor cores (CSA Eq. 18-19, HCA Eq. 24-26, Module D).
//
// All H heads of a query share one key set, and every key is also its own
// value. Keys are taken in tiles of 64, double-buffered in shared memory, and
// go on the M axis of both contractions:
//   S^T  M = 128 rows: the tile's 64 keys twice, rows 0-63 with dims 0-255 and
//        rows 64-127 with dims 256-511; N = 2H columns: Q dims 0-255 for heads
//        0..H-1, Q dims 256-511 for heads H..2H-1. Row r < 64 of the first H
//        columns plus row r + 64 of the last H columns is the logit of key r;
//        the other two quarters are not used. (M stays 128, and the tile is
//        half the size of a 128-key one, so two fit beside Q.)
//   O^T[dim][head] += sum_key K[key][dim] P^T[key][head]: M = 128 dims (the
//        64-dim blocks j and j + 4), N = H, four M-tiles.
// A tile is 8 slots of 8 KB (64 rows x 128 bytes, 128-byte swizzle); slot 2p
// holds dims 64p.., slot 2p+1 dims 256 + 64p.., so the 16 KB slot pair p is
// the K-major A operand of the S^T product for dims {64p.., 256 + 64p..} and,
// read along the other axis, the M/N-major A operand of O^T M-tile p.
//
// Warp roles (one persistent block per SM looping over queries):
//  * warps 0-3 gather each tile into the free buffer: one tiled TMA box per
//    slot when the 64 keys are consecutive rows of one source, else 16-byte
//    cp.async per thread (fp8 entries are decoded to bf16 on the way). One
//    thread also loads each query's Q with tiled TMA copies.
//  * warp 4 allocates tensor memory and issues the MMAs: the S^T product of a
//    tile as soon as it has landed and the O^T product of the tile before it
//    as soon as its probabilities are written, whichever is ready first.
//  * warps 5.. (four per group of 16 heads) own the TMEM lanes: they add the
//    two halves of each logit (through shared memory), take the softmax into
//    P^T for their heads, and normalise and write each query's output.
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
constexpr int KT = 64;               // keys per tile
constexpr float kLazy2 = 11.5f;      // lazy-rescale margin, base-2 units (about e^8)
constexpr int kMmaWarp = 4;
constexpr int kSoftWarp0 = 5;
constexpr int kGatherBar = 5;        // named barrier of the 4 gather warps (1..4: head groups;
                                     // 6, 7: the two gather groups)

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

// slot of 64-dim block kb inside a tile (pairs {p, p + 4} side by side)
__host__ __device__ constexpr int slot_of(int kb) { return (kb & 3) * 2 + (kb >> 2); }

template <int H>
struct Lay {
    static constexpr int NG = H / 16;                               // head groups
    static constexpr int THREADS = 32 * (kSoftWarp0 + 4 * NG);
    static constexpr size_t K_OFF = 0;                              // 2 x 64 KB tiles
    static constexpr size_t Q_OFF = 2 * 65536;                      // 4 pairs x 2H x 128
    static constexpr size_t P_OFF = Q_OFF + 8 * H * 128;            // H x 128 (64 keys)
    static constexpr size_t X_OFF = P_OFF + H * 128;                // NG x 8 x 128 floats
    static constexpr size_t PTR_OFF = X_OFF + NG * 8 * 128 * 4;     // 2 x 64 row pointers
    static constexpr size_t ROW_OFF = PTR_OFF + 2 * KT * 8;         // 64 fp8 entry rows
    static constexpr size_t F_OFF = ROW_OFF + KT * 8;               // 8 x H floats
    static constexpr size_t BAR_OFF = F_OFF + ((8 * H * 4 + 63) / 64) * 64;
    static constexpr size_t TOTAL = BAR_OFF + 256;
    static constexpr uint32_t S_COLS = 2 * H;                       // per S^T buffer
    static constexpr uint32_t O_COL = 4 * H;                        // after 2 S^T buffers
    static constexpr uint32_t TMEM_COLS = (8 * H <= 128) ? 128 : (8 * H <= 256 ? 256 : 512);
    static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 2 * H, 0, 0);
    static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, H, 1, 0);
};

// Per-work-item quantities (a query, or one chunk of a query's key tiles),
// computed identically by every role.
struct QInfo {
    int64_t b, t, V, nsel, nwin, w0, wp0, nk;
    int64_t wbeg;     // first window slot: nsel rounded up to 8
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

// key_row with the selection index of slot j already loaded (slot_index).
template <bool KV8>
__device__ __forceinline__ const __nv_bfloat16 *key_row_s(const TcAttn &a, const QInfo &q,
                                                          int64_t bt, int64_t j, int32_t sidx,
                                                          bool report_bad, int64_t *entry_row)
{
    *entry_row = -1;
    if (j < q.nsel) {
        const int64_t s = a.dense ? j : (int64_t)sidx;
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

// The selection index read by key slot j (only slots j < nsel of a sparse
// selection read one), and whether slot j holds a key, given that index: the
// same decision as key_row, split so that the load can be issued early.
__device__ __forceinline__ int32_t slot_index(const TcAttn &a, const QInfo &q, int64_t bt,
                                              int64_t j)
{
    return (!a.dense && j < q.nsel) ? __ldg(a.idx + bt * a.k + j) : 0;
}

__device__ __forceinline__ bool slot_valid(const TcAttn &a, const QInfo &q, int64_t j, int32_t s)
{
    if (j < q.nsel) {
        const int64_t e = a.dense ? j : (int64_t)s;
        return e >= 0 && e < q.V;
    }
    if (j >= q.wbeg && j < q.nk) {
        const int64_t wr = q.w0 + (j - q.wbeg) - q.wp0;
        return wr >= 0 && wr < a.win_rows;
    }
    return false;
}

// 16 e4m3 codes times one scale -> 16 bf16 in two 16-byte chunks.
__device__ __forceinline__ void decode16(const uint4 &cw, float sc, uint4 *lo, uint4 *hi)
{
    const uint16_t *c2 = (const uint16_t *)&cw;
    __nv_bfloat162 o[8];
#pragma unroll
    for (int e = 0; e < 8; e++) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)c2[e], __NV_E4M3);
        const float2 f = __half22float2(__half2(hr));
        o[e] = __floats2bfloat162_rn(f.x * sc, f.y * sc);
    }
    *lo = *(const uint4 *)&o[0];
    *hi = *(const uint4 *)&o[4];
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
    float *sX = (float *)(sm + L::X_OFF);
    const __nv_bfloat16 **kptr = (const __nv_bfloat16 **)(sm + L::PTR_OFF);
    int64_t *krow = (int64_t *)(sm + L::ROW_OFF);
    float *m_run = (float *)(sm + L::F_OFF);     // [H] running offsets, base 2
    float *red = m_run + H;                      // [4][H] per-warp maxima / sums
    float *sink2 = red + 4 * H;                  // [H] sink logits, base-2 units
    float *m_new = sink2 + H;                    // [H] offsets after a rescale
    float *alpha_s = m_new + H;                  // [H] rescale factors
    uint64_t *bars = (uint64_t *)(sm + L::BAR_OFF);
    uint64_t *kfull = bars;          // [2] tile landed (128 gather arrivals + TMA bytes)
    uint64_t *kfree = bars + 2;      // [2] tile consumed by its O^T product
    uint64_t *sfull = bars + 4;      // [2] S^T product done
    uint64_t *pfull = bars + 6;      // P^T written (all head groups)
    uint64_t *odone = bars + 7;      // O^T product of a tile done (one phase per tile)
    uint64_t *qfull = bars + 8, *qfree = bars + 9;
    uint64_t *ofull = bars + 10, *ofree = bars + 11, *done = bars + 12;
    uint32_t *tmem_slot = (uint32_t *)(bars + 13);
    int *abort_flag = (int *)(tmem_slot + 1);
    const int64_t nitems = a.nqueries * a.nchunks;
    const bool split = a.nchunks > 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&kfull[i], KV8 ? 128 : 64);    // one arrival per gather thread of the group
            tc::mbar_init(&kfree[i], 1);
            tc::mbar_init(&sfull[i], 1);
        }
        tc::mbar_init(pfull, 128 * NG);
        tc::mbar_init(odone, 1);
        tc::mbar_init(qfull, 1);
        tc::mbar_init(qfree, 1);
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
        // bf16 entries: two groups of two warps take alternate tiles (group g
        // fills buffer g), so that one group's copies are in flight while the
        // other waits for its buffer; fp8 entries: one group of four warps.
        // The selection indices of a group's next tile are loaded while its
        // current tile is copied.
        constexpr int NGRP = KV8 ? 1 : 2;
        constexpr int GT = 128 / NGRP;               // threads of a group
        const int gt = tid;                          // 0..127
        const int grp = gt / GT, lt = gt % GT;
        const int gbar = kGatherBar + 1 + grp;       // the group's own named barrier
        const __nv_bfloat16 **gptr = kptr + grp * KT;
        const void *zero_src = KV8 ? (a.kwin ? (const void *)a.kwin : (const void *)a.ent8)
                                   : (a.E > 0 ? (const void *)a.ent : (const void *)a.kwin);
        uint32_t t = 0, qctr = 0;
        bool ok = true;
        for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
            const int64_t bt = w / a.nchunks;
            const QInfo q = query_info(a, bt, (int)(w % a.nchunks));
            // Q buffer free once the previous item's last S^T product is done
            const bool qf = qctr == 0 || tc::mbar_wait(qfree, (qctr - 1) & 1, abortv);
            if (tc::named_bar_or(kGatherBar, 128, !qf)) {
                ok = false;
                break;
            }
            if (gt == 0) {
                tc::mbar_arrive_expect_tx(qfull, (uint32_t)(H * 1024));
                for (int kb = 0; kb < 8; kb++)
                    tc::tma_load_2d(sQ + (kb & 3) * (2 * H * 128) + (kb >> 2) * (H * 128), &tm_q,
                                    qfull, kb * 64, (int)(bt * H));
            }
            const uint32_t t_item = t;
            // this group's first tile of the item
            int i = (int)((grp - (int)(t_item % NGRP) + NGRP) % NGRP);
            int32_t s_own = 0, s_first = 0;
            if (i < q.ntiles && lt < KT) {
                const int64_t j0 = (int64_t)(q.tile0 + i) * KT;
                s_own = slot_index(a, q, bt, j0 + lt);
                s_first = slot_index(a, q, bt, j0);
            }
            for (; i < q.ntiles; i += NGRP) {
                const uint32_t tt = t_item + (uint32_t)i;
                const int b = tt & 1;
                uint8_t *kbuf = sK + b * 65536;
                const int64_t jt0 = (int64_t)(q.tile0 + i) * KT;
                // A tile whose 64 rows are consecutive rows of one bf16 source
                // (dense entries, a selection that is a run, window positions)
                // goes by one tiled TMA box per slot; any other tile by
                // per-thread copies.
                bool run = true;
                int64_t row0 = 0;
                const bool src_ent = jt0 < q.nsel;
                if (lt < KT) {
                    int64_t er, er0;
                    const __nv_bfloat16 *kp = key_row_s<KV8>(a, q, bt, jt0 + lt, s_own, true, &er);
                    gptr[lt] = kp;
                    if (KV8)
                        krow[lt] = er;
                    const __nv_bfloat16 *p0 = key_row_s<KV8>(a, q, bt, jt0, s_first, false, &er0);
                    const bool src_win = jt0 >= q.wbeg;
                    const bool same = (jt0 + lt < q.nsel) == src_ent && (jt0 + lt >= q.wbeg) == src_win;
                    run = p0 != nullptr && same && kp == p0 + (int64_t)lt * DIM;
                    const __nv_bfloat16 *base = src_ent ? a.ent : a.kwin;
                    row0 = p0 ? (p0 - base) / DIM : 0;
                    run = run && row0 <= 0x7fffffff - KT && (src_ent ? a.tma_ent : a.tma_win);
                }
                const bool all_run = !tc::named_bar_or(gbar, GT, !run);
                // the group's next tile: its indices are requested now
                if (i + NGRP < q.ntiles && lt < KT) {
                    const int64_t jn = jt0 + (int64_t)NGRP * KT;
                    s_own = slot_index(a, q, bt, jn + lt);
                    s_first = slot_index(a, q, bt, jn);
                }
                // buffer b is free once the O^T product of tile tt - 2 is done
                if (tt >= 2) {
                    const bool fr = tc::mbar_wait(&kfree[b], ((tt - 2) >> 1) & 1, abortv);
                    if (tc::named_bar_or(gbar, GT, !fr)) {
                        ok = false;
                        break;
                    }
                }
                if (all_run) {
                    if (lt == 0) {
                        tc::mbar_expect_tx(&kfull[b], 65536u);
#pragma unroll 1
                        for (int kb = 0; kb < 8; kb++)
                            tc::tma_load_2d(kbuf + slot_of(kb) * 8192, src_ent ? &tm_ent : &tm_win,
                                            &kfull[b], kb * 64, (int)row0);
                    }
                } else if (KV8) {
                    // two threads per row: body bytes [224 * half, +224) as 14
                    // pieces of 16 codes (each inside one 64-dim scale group),
                    // decoded to bf16; RoPE dims and bf16 window rows by cp.async
                    const int row = lt >> 1, half = lt & 1;
                    const int64_t er = krow[row];
                    uint8_t *rbase = kbuf + row * 128;
                    if (er >= 0) {
                        // RoPE dims first (asynchronous), and both batches'
                        // lines requested from HBM at once
#pragma unroll
                        for (int c = half * 4; c < half * 4 + 4; c++)
                            tc::cp_async16(rbase + slot_of(7) * 8192 + ((c ^ (row & 7)) << 4),
                                           a.ent_rope + er * 64 + c * 8, 16u);
                        const uint8_t *rp = a.ent8 + er * 448 + half * 224;
#pragma unroll
                        for (int off = 0; off < 224; off += 64)
                            tc::prefetch_l2(rp + off);
#pragma unroll 1
                        for (int bat = 0; bat < 2; bat++) {
                            uint4 cw[7];
                            float sc[7];
#pragma unroll
                            for (int j = 0; j < 7; j++) {
                                const int byte = (half * 14 + bat * 7 + j) * 16;
                                cw[j] = __ldg((const uint4 *)(a.ent8 + er * 448 + byte));
                                sc[j] = __ldg(a.ent_scale + er * 7 + (byte >> 6));
                            }
#pragma unroll
                            for (int j = 0; j < 7; j++) {
                                const int byte = (half * 14 + bat * 7 + j) * 16;
                                const int kb = byte >> 6, c0 = (byte & 63) >> 3;
                                uint8_t *sb = rbase + slot_of(kb) * 8192;
                                uint4 lo, hi;
                                decode16(cw[j], sc[j], &lo, &hi);
                                *(uint4 *)(sb + ((c0 ^ (row & 7)) << 4)) = lo;
                                *(uint4 *)(sb + (((c0 + 1) ^ (row & 7)) << 4)) = hi;
                            }
                        }
                    } else {
                        const __nv_bfloat16 *sp = gptr[row];
#pragma unroll 1
                        for (int kb = half * 4; kb < half * 4 + 4; kb++)
#pragma unroll
                            for (int c = 0; c < 8; c++)
                                tc::cp_async16(rbase + slot_of(kb) * 8192 + ((c ^ (row & 7)) << 4),
                                               sp ? (const void *)(sp + kb * 64 + c * 8) : zero_src,
                                               sp ? 16u : 0u);
                    }
                } else {
                    // this thread's KT * 8 / GT rows, read once (a pointer re-read
                    // from shared memory before every copy would serialise the issue)
                    // (destinations as 32-bit shared addresses: row r of a slot
                    // at r * 128, its 16-byte chunk c at (c ^ (r & 7)) * 16)
                    constexpr int RPT = KT * 8 / GT;           // rows per thread
                    const __nv_bfloat16 *sp[RPT];
                    const int c = lt & 7;
                    const uint32_t d0 = tc::smem_u32(kbuf) + (uint32_t)(lt >> 3) * 128u;
#pragma unroll
                    for (int u = 0; u < RPT; u++) {
                        const int row = u * (GT / 8) + (lt >> 3);
                        const __nv_bfloat16 *p = gptr[row];
                        sp[u] = p ? p + c * 8 : nullptr;
                    }
#pragma unroll
                    for (int kb = 0; kb < 8; kb++)
#pragma unroll
                        for (int u = 0; u < RPT; u++) {
                            const int row = u * (GT / 8) + (lt >> 3);
                            tc::cp_async16_s(d0 + (uint32_t)(u * (GT / 8) * 128 + slot_of(kb) * 8192 +
                                                             ((c ^ (row & 7)) << 4)),
                                             sp[u] ? (const void *)(sp[u] + kb * 64) : zero_src,
                                             sp[u] ? 16u : 0u);
                        }
                }
                tc::cp_async_commit();
                tc::cp_async_wait_all();
                tc::fence_async_shared();
                tc::mbar_arrive(&kfull[b]);
                tc::named_bar_sync(gbar, GT);     // the group's row pointers rewritten next tile
            }
            t = t_item + (uint32_t)q.ntiles;
        }
        tc::cp_async_wait_all();
        if (!ok) {
            *abort_flag = 1;
            report(a.err, CSA_ERR_TIMEOUT, K_ATTEND_TC, blockIdx.x, 0);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t sK_a = tc::smem_u32(sK), sQ_a = tc::smem_u32(sQ), sP_a = tc::smem_u32(sP);
            // descriptors advance by constants (byte offsets >> 4)
            const uint64_t adS = tc::sdesc_sw128(sK_a), bdS = tc::sdesc_sw128(sQ_a);
            const uint64_t adO = tc::sdesc_sw128_mn(sK_a, 8192, 1024), bdO = tc::sdesc_sw128(sP_a);
            uint32_t t = 0, qctr = 0;
            bool ok = true;
            // the tile whose O^T product is still to be issued
            bool pend = false, pend_first = false, pend_last = false;
            uint32_t pend_t = 0, pend_q = 0;
            auto issue_s = [&](uint32_t ts) {
                const int b = ts & 1;
#pragma unroll 1
                for (int p = 0; p < 4; p++) {
                    const uint64_t ad = adS + (uint64_t)(b * 4096 + p * 1024);
                    const uint64_t bd = bdS + (uint64_t)(p * (H * 16));
                    tc::mma_f16(tmem + b * L::S_COLS, ad, bd, L::IDESC_S, p != 0);
#pragma unroll
                    for (int kk = 1; kk < 4; kk++)
                        tc::mma_f16(tmem + b * L::S_COLS, ad + (uint64_t)(kk * 2),
                                    bd + (uint64_t)(kk * 2), L::IDESC_S, 1u);
                }
                tc::mma_commit(&sfull[b]);
            };
            auto issue_o = [&]() {
                const int b = pend_t & 1;
                const uint32_t acc0 = pend_first ? 0u : 1u;
#pragma unroll 1
                for (int jt = 0; jt < 4; jt++) {
                    const uint64_t ad = adO + (uint64_t)(b * 4096 + jt * 1024);
                    const uint32_t d = tmem + L::O_COL + jt * H;
                    tc::mma_f16(d, ad, bdO, L::IDESC_O, acc0);
#pragma unroll
                    for (int kk = 1; kk < 4; kk++)
                        tc::mma_f16(d, ad + (uint64_t)(kk * 128), bdO + (uint64_t)(kk * 2),
                                    L::IDESC_O, 1u);
                }
                tc::mma_commit(&kfree[b]);
                tc::mma_commit(odone);
                if (pend_last)
                    tc::mma_commit(ofull);
                pend = false;
            };
            // O^T of the first tile of item pend_q overwrites the accumulator:
            // the epilogue of item pend_q - 1 must have read it
            auto o_ready = [&]() {
                if (!tc::mbar_test_wait(pfull, pend_t & 1))
                    return false;
                return !pend_first || pend_q == 0 || tc::mbar_test_wait(ofree, (pend_q - 1) & 1);
            };
            // Issues S^T of tile ts (when wanted) and the pending O^T product,
            // each as soon as its inputs are ready. Bounded in time.
            auto advance = [&](bool want_s, uint32_t ts) -> bool {
                const uint64_t t0 = tc::global_ns();
                for (uint32_t it = 1;; ++it) {
                    if (want_s && tc::mbar_test_wait(&kfull[ts & 1], (ts >> 1) & 1)) {
                        tc::fence_after();
                        issue_s(ts);
                        want_s = false;
                    }
                    if (pend && o_ready()) {
                        tc::fence_after();
                        issue_o();
                    }
                    if (!want_s && !pend)
                        return true;
                    if ((it & 255u) == 0u && (*abortv || tc::global_ns() - t0 > 2000000000ull))
                        return false;
                }
            };
            for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
                const QInfo q = query_info(a, w / a.nchunks, (int)(w % a.nchunks));
                if (!tc::mbar_wait(qfull, qctr & 1, abortv)) {
                    ok = false;
                    break;
                }
                if (q.ntiles == 0) {
                    // no keys: finish the pending product, then hand an (unused)
                    // O^T to this item's epilogue once the previous one has read it
                    if (pend && !advance(false, 0)) {
                        ok = false;
                        break;
                    }
                    if (qctr > 0 && !tc::mbar_wait(ofree, (qctr - 1) & 1, abortv)) {
                        ok = false;
                        break;
                    }
                    tc::mma_commit(qfree);
                    tc::mma_commit(ofull);
                    continue;
                }
                for (int i = 0; i < q.ntiles; ++i, ++t) {
                    // S^T of tile t (its Q is resident) and O^T of tile t - 1
                    if (!advance(true, t)) {
                        ok = false;
                        break;
                    }
                    if (i == q.ntiles - 1)
                        tc::mma_commit(qfree);
                    pend = true;
                    pend_t = t;
                    pend_first = i == 0;
                    pend_last = i == q.ntiles - 1;
                    pend_q = qctr;
                }
            }
            if (ok && pend && !advance(false, 0))
                ok = false;
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
        // every probability is one ex2 of a difference.
        const float scale2 = a.scale * 1.4426950408889634f;
        const int g = (warp - kSoftWarp0) >> 2;         // head group: heads h0 .. h0+15
        const int h0 = 16 * g;
        const int gbar = 1 + g;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;                   // TMEM lane of this thread
        const int half = r >> 6;                        // S^T half: dims 0-255 / 256-511
        const int kidx = r & 63;                        // key of the tile
        const int hk = h0 + 8 * half;                   // first of the 8 heads kept here
        const int et = (warp - kSoftWarp0 - 4 * g) * 32 + lane;   // 0..127 inside the group
        const uint32_t lane_tm = tmem + ((uint32_t)(q4 * 32) << 16);
        float *xg = sX + g * (8 * 128);                 // [8][128] partial logits handed over
        uint32_t t = 0, qctr = 0;
        bool ok = true, stale = false;
        for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++qctr) {
            const int64_t bt = w / a.nchunks;
            const QInfo q = query_info(a, bt, (int)(w % a.nchunks));
            float lpart[8];
#pragma unroll
            for (int u = 0; u < 8; u++)
                lpart[u] = 0.f;
            // the selection index of this thread's key slot, loaded one tile
            // ahead so that its latency overlaps the softmax of the tile before
            int32_t s_next =
                q.ntiles > 0 ? slot_index(a, q, bt, (int64_t)q.tile0 * KT + kidx) : 0;
            for (int i = 0; i < q.ntiles; ++i, ++t) {
                const int64_t jslot = (int64_t)(q.tile0 + i) * KT + kidx;
                const int32_t s_cur = s_next;
                if (i + 1 < q.ntiles)
                    s_next = slot_index(a, q, bt, jslot + KT);
                const bool valid = slot_valid(a, q, jslot, s_cur);
                // a wait that gives up marks this thread stale; the group agrees
                // on it at its next barrier (the exchange below, or the end of
                // the item), so no barrier is spent on the waits themselves
                stale |= !tc::mbar_wait(&sfull[t & 1], (t >> 1) & 1, abortv);
                tc::fence_after();
                float z[8];
                {
                    uint32_t rr[16];
                    tc::tmem_ld16(lane_tm + (t & 1) * L::S_COLS + half * H + h0, rr);
                    tc::tmem_ld_wait();
                    // hand the other half's 8 heads to the partner lane r ^ 64
#pragma unroll
                    for (int j = 0; j < 8; j++)
                        xg[j * 128 + r] = __uint_as_float(half ? rr[j] : rr[8 + j]);
                    if (tc::named_bar_or(gbar, 128, stale)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const float mine = __uint_as_float(half ? rr[8 + j] : rr[j]);
                        z[j] = valid ? (mine + xg[j * 128 + (r ^ 64)]) * scale2 : -INFINITY;
                    }
                }
                float m8[8];
                {
                    const float4 m0 = *(const float4 *)(m_run + hk);
                    const float4 m1 = *(const float4 *)(m_run + hk + 4);
                    m8[0] = m0.x; m8[1] = m0.y; m8[2] = m0.z; m8[3] = m0.w;
                    m8[4] = m1.x; m8[5] = m1.y; m8[6] = m1.z; m8[7] = m1.w;
                }
                bool need = false;
#pragma unroll
                for (int j = 0; j < 8; j++)
                    need |= z[j] > m8[j] + kLazy2;
                bool o_waited = false;
                if (tc::named_bar_or(gbar, 128, need)) {
                    // maxima of this tile: warps 0,1 of the group hold heads
                    // h0..h0+7, warps 2,3 heads h0+8..h0+15
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        float v = z[j];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1)
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                        if (lane == 0)
                            red[q4 * H + hk + j] = v;
                    }
                    tc::named_bar_sync(gbar, 128);
                    // one thread per head: new offset and the factor for what is summed
                    float mn = 0.f;
                    if (et < 16) {
                        const int hh = h0 + et;
                        const int qa = et < 8 ? 0 : 2;
                        const float tmax = fmaxf(red[qa * H + hh], red[(qa + 1) * H + hh]);
                        const float mo = m_run[hh];
                        mn = fmaxf(mo, tmax);
                        m_new[hh] = mn;
                        alpha_s[hh] = (mn == -INFINITY) ? 1.f : fast_ex2(mo - mn);
                    }
                    tc::named_bar_sync(gbar, 128);
                    if (et < 16)
                        m_run[h0 + et] = mn;
                    {
                        const float4 m0 = *(const float4 *)(m_new + hk);
                        const float4 m1 = *(const float4 *)(m_new + hk + 4);
                        m8[0] = m0.x; m8[1] = m0.y; m8[2] = m0.z; m8[3] = m0.w;
                        m8[4] = m1.x; m8[5] = m1.y; m8[6] = m1.z; m8[7] = m1.w;
                    }
                    if (i > 0) {
                        // O^T of the tiles before must be complete before rescaling
                        const bool od = tc::mbar_wait(odone, (t - 1) & 1, abortv);
                        if (tc::named_bar_or(gbar, 128, !od)) {
                            ok = false;
                            break;
                        }
                        o_waited = true;
                        tc::fence_after();
#pragma unroll 1
                        for (int jt = 0; jt < 4; jt++) {
                            uint32_t rr[16];
                            const uint32_t ad = lane_tm + L::O_COL + jt * H + h0;
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
                    for (int j = 0; j < 8; j++)
                        lpart[j] *= alpha_s[hk + j];
                }
                __nv_bfloat162 pb[4];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const float p0 = valid ? fast_ex2(z[j] - m8[j]) : 0.f;
                    const float p1 = valid ? fast_ex2(z[j + 1] - m8[j + 1]) : 0.f;
                    pb[j / 2] = __floats2bfloat162_rn(p0, p1);
                    const float2 pr = __bfloat1622float2(pb[j / 2]);
                    lpart[j] += pr.x;
                    lpart[j + 1] += pr.y;
                }
                // P^T is free once the O^T product of the previous tile is done
                if (t > 0 && !o_waited)
                    stale |= !tc::mbar_wait(odone, (t - 1) & 1, abortv);
                {
                    // P^T rows hk..hk+7 (one per head, 64 keys, 128-byte swizzle)
                    uint8_t *pbase = sP + (kidx & 7) * 2;
                    const int chunk = kidx >> 3;
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const int hh = hk + j;
                        const __nv_bfloat16 v = (j & 1) ? pb[j / 2].y : pb[j / 2].x;
                        *(__nv_bfloat16 *)(pbase + hh * 128 + ((chunk ^ (hh & 7)) << 4)) = v;
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
            for (int j = 0; j < 8; j++) {
                float v = lpart[j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0)
                    red[q4 * H + hk + j] = v;
            }
            if (tc::named_bar_or(gbar, 128, stale)) {
                ok = false;
                break;
            }
            // one thread per head: the output factor (alpha_s is free here)
            if (et < 16) {
                const int hh = h0 + et;
                const int qa = et < 8 ? 0 : 2;
                const float l = red[qa * H + hh] + red[(qa + 1) * H + hh];
                float fh;
                if (split) {
                    // partial of this key chunk: raw accumulator, offset (natural units), sum
                    fh = 1.f;
                    a.ws_ml[(w * H + hh) * 2] = m_run[hh] * 0.6931471805599453f;
                    a.ws_ml[(w * H + hh) * 2 + 1] = l;
                } else {
                    const float zs2 = sink2[hh];
                    float lse;
                    if (zs2 == INFINITY) {
                        fh = 0.f;
                        lse = INFINITY;
                    } else {
                        const float mh = m_run[hh];
                        const float M2 = fmaxf(mh, zs2);
                        if (M2 == -INFINITY) {
                            fh = 0.f;
                            lse = -INFINITY;
                        } else {
                            const float e = fast_ex2(mh - M2);
                            const float den = l * e + fast_ex2(zs2 - M2);
                            fh = e / den;
                            lse = (M2 + fast_lg2(den)) * 0.6931471805599453f;
                        }
                    }
                    if (q.ntiles == 0)
                        fh = 0.f;
                    if (a.lse)
                        a.lse[bt * H + hh] = lse;
                }
                alpha_s[hh] = fh;
            }
            tc::named_bar_sync(gbar, 128);
            float f[16];
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const float4 fv = *(const float4 *)(alpha_s + h0 + u);
                f[u] = fv.x;
                f[u + 1] = fv.y;
                f[u + 2] = fv.z;
                f[u + 3] = fv.w;
            }
            const bool got = tc::mbar_wait(ofull, qctr & 1, abortv);
            if (tc::named_bar_or(gbar, 128, !got)) {
                ok = false;
                break;
            }
            tc::fence_after();
            // O^T M-tile jt: lanes 0-63 dims 64 jt.., lanes 64-127 dims 256 + 64 jt..
#pragma unroll 1
            for (int jt = 0; jt < 4; jt++) {
                const int d = (half ? 256 : 0) + 64 * jt + kidx;
                float o[16];
                if (q.ntiles > 0) {
                    uint32_t rr[16];
                    tc::tmem_ld16(lane_tm + L::O_COL + jt * H + h0, rr);
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
                    float *orow = a.ws_o + (w * H) * DIM + d;
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        orow[(h0 + u) * DIM] = o[u];
                } else {
                    // this warp's 32 dims x 16 heads go through its 1 KB of the
                    // group's exchange area as [head][dim], then out as 16-byte
                    // runs of 8 dims of one head
                    __nv_bfloat16 *xs = (__nv_bfloat16 *)xg + (et >> 5) * 512;
#pragma unroll
                    for (int u = 0; u < 16; u++)
                        xs[u * 32 + lane] = __float2bfloat16_rn(o[u]);
                    __syncwarp();
                    const int dbase = d - lane;
#pragma unroll
                    for (int c2 = 0; c2 < 2; c2++) {
                        const int c = lane + 32 * c2, head = c >> 2, part = c & 3;
                        const uint4 v = *(const uint4 *)(xs + head * 32 + part * 8);
                        *(uint4 *)(a.out + (bt * H + h0 + head) * DIM + dbase + part * 8) = v;
                    }
                    __syncwarp();
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
// entering once here. The per-chunk weights are worked out once per block;
// each thread then owns 4 dims and keeps several chunk loads in flight.
constexpr int kMaxChunks = 512;

__global__ void __launch_bounds__(128)
combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_ml, int nchunks, int H,
               const float *__restrict__ sink, __nv_bfloat16 *__restrict__ out,
               float *__restrict__ lse)
{
    __shared__ float wt[kMaxChunks];
    __shared__ float red[4];
    __shared__ float s_den;
    const int64_t bt = blockIdx.x;
    const int hh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *ml = ws_ml + (bt * nchunks * H + hh) * 2;     // chunk c at + c * H * 2
    const float zs = sink[hh];
    float M = -INFINITY;
    for (int c = tid; c < nchunks; c += 128)
        M = fmaxf(M, ml[(int64_t)c * H * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0)
        red[warp] = M;
    __syncthreads();
    M = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])), zs);
    const bool zero = zs == INFINITY || M == -INFINITY;
    float part = 0.f;
    for (int c = tid; c < nchunks; c += 128) {
        const float mc = ml[(int64_t)c * H * 2];
        const float wc = (zero || mc == -INFINITY) ? 0.f : __expf(mc - M);
        wt[c] = wc;
        part += ml[(int64_t)c * H * 2 + 1] * wc;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        part += __shfl_xor_sync(0xffffffffu, part, o);
    __syncthreads();                       // red reused, wt complete
    if (lane == 0)
        red[warp] = part;
    __syncthreads();
    if (tid == 0) {
        const float den = zero ? 0.f : red[0] + red[1] + red[2] + red[3] + __expf(zs - M);
        s_den = den;
        if (lse)
            lse[bt * H + hh] = zero ? (zs == INFINITY ? INFINITY : -INFINITY) : M + __logf(den);
    }
    __syncthreads();
    const float inv = zero ? 0.f : 1.f / s_den;
    const float *op = ws_o + (bt * nchunks * H + hh) * (int64_t)DIM + tid * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int c = zero ? nchunks : 0;
    for (; c + 8 <= nchunks; c += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; j++)
            v[j] = __ldg((const float4 *)(op + (int64_t)(c + j) * H * DIM));
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float wc = wt[c + j];
            acc.x += v[j].x * wc;
            acc.y += v[j].y * wc;
            acc.z += v[j].z * wc;
            acc.w += v[j].w * wc;
        }
    }
    for (; c < nchunks; c++) {
        const float4 v = __ldg((const float4 *)(op + (int64_t)c * H * DIM));
        const float wc = wt[c];
        acc.x += v.x * wc;
        acc.y += v.y * wc;
        acc.z += v.z * wc;
        acc.w += v.w * wc;
    }
    __nv_bfloat162 o2[2] = {__floats2bfloat162_rn(acc.x * inv, acc.y * inv),
                            __floats2bfloat162_rn(acc.z * inv, acc.w * inv)};
    *(uint2 *)(out + (bt * H + hh) * DIM + tid * 4) = *(const uint2 *)o2;
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
