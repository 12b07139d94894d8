// topk.cu -- top-k selector (Eq. 17): radix select over the visible scores.
//
// Scores are mapped to order-preserving 32-bit keys (larger float -> larger
// key, -0 folded onto +0). Radix digits, most significant first, find the key
// T of the k-th largest element and how many elements equal to T must be
// taken (ties prefer lower indices). A final pass in index order writes every
// element with key > T and the first `need` elements with key == T, so each
// row comes out in ascending index order. Three layouts of the work:
//  * short rows (<= 2048 visible): one warp per row, keys in registers;
//  * rows up to 64 K: one block per row; for k <= 1024 the row's candidates
//    (entries at or above a lower bound taken from a sample of the row) are
//    kept in shared memory and selected exactly with 8-bit digits; for larger
//    k the keys are staged once in shared memory when they fit (re-read from
//    L2 otherwise) and selected with 12 + 12 + 8-bit digits;
//  * longer rows (decode): rows of up to 256 K entries in one launch, a
//    cluster of 8 blocks per row exchanging digit counts through distributed
//    shared memory; past that, chunks of the row over many blocks, then one
//    block per row over the candidates of the threshold bin.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kResident = 40960;   // keys staged in shared memory (160 KB)

constexpr int kCand = 4096;          // keys of the first threshold bin kept aside

struct Shared {
    unsigned hist[4096];                 // digit histogram (12 or 8 bits)
    uint32_t cand[kCand];                // keys of the first threshold bin
    unsigned warp_tot[kWarps];
    unsigned warp_cnt[2][kWarps];
    unsigned bin, need, ncand;
};

// Source of one row: order-preserving key and the index it reports.
struct RowScores {
    const float *src;
    __device__ __forceinline__ uint32_t key(int64_t p) const { return float_key(src[p]); }
    __device__ __forceinline__ int32_t index(int64_t p) const { return (int32_t)p; }
    // keys of [0, V) into shared memory with 16-byte loads, 4 in flight per
    // thread (a row is read from HBM once; one scalar load at a time would
    // pay the memory latency for every 2 KB of the row), counted into the
    // histogram of their top 12 bits on the way
    __device__ __forceinline__ void stage(uint32_t *keys, int V, unsigned *hist) const
    {
        int head = 0;
        if (((uintptr_t)src & 15u) != 0)
            head = V < 4 - (int)(((uintptr_t)src & 15u) >> 2) ? V
                                                                : 4 - (int)(((uintptr_t)src & 15u) >> 2);
        for (int s = threadIdx.x; s < head; s += kThreads) {
            keys[s] = key(s);
            atomicAdd(&hist[keys[s] >> 20], 1u);
        }
        const float4 *v4 = (const float4 *)(src + head);
        const int n4 = (V - head) >> 2;
        int i = threadIdx.x;
        for (; i + 3 * kThreads < n4; i += 4 * kThreads) {
            float4 f[4];
#pragma unroll
            for (int j = 0; j < 4; j++)
                f[j] = __ldg(v4 + i + j * kThreads);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                uint32_t *d = keys + head + 4 * (i + j * kThreads);
                const uint32_t k0 = float_key(f[j].x), k1 = float_key(f[j].y);
                const uint32_t k2 = float_key(f[j].z), k3 = float_key(f[j].w);
                d[0] = k0;
                d[1] = k1;
                d[2] = k2;
                d[3] = k3;
                atomicAdd(&hist[k0 >> 20], 1u);
                atomicAdd(&hist[k1 >> 20], 1u);
                atomicAdd(&hist[k2 >> 20], 1u);
                atomicAdd(&hist[k3 >> 20], 1u);
            }
        }
        for (; i < n4; i += kThreads) {
            const float4 f = __ldg(v4 + i);
            uint32_t *d = keys + head + 4 * i;
            const uint32_t k0 = float_key(f.x), k1 = float_key(f.y);
            const uint32_t k2 = float_key(f.z), k3 = float_key(f.w);
            d[0] = k0;
            d[1] = k1;
            d[2] = k2;
            d[3] = k3;
            atomicAdd(&hist[k0 >> 20], 1u);
            atomicAdd(&hist[k1 >> 20], 1u);
            atomicAdd(&hist[k2 >> 20], 1u);
            atomicAdd(&hist[k3 >> 20], 1u);
        }
        for (int s = head + 4 * n4 + threadIdx.x; s < V; s += kThreads) {
            keys[s] = key(s);
            atomicAdd(&hist[keys[s] >> 20], 1u);
        }
    }
};

struct RowCandidates {
    const uint32_t *keys;
    const int32_t *idx;
    __device__ __forceinline__ uint32_t key(int64_t p) const { return keys[p]; }
    __device__ __forceinline__ int32_t index(int64_t p) const { return idx[p]; }
    __device__ __forceinline__ void stage(uint32_t *dst, int V, unsigned *hist) const
    {
        for (int s = threadIdx.x; s < V; s += kThreads) {
            const uint32_t u = keys[s];
            dst[s] = u;
            atomicAdd(&hist[u >> 20], 1u);
        }
    }
};

// Bin of the digit histogram hist[0..nb) (descending) where the count from
// the top reaches `need`; writes sh.bin and sh.need (what is still needed
// inside that bin). Thread t owns bins nb-1-t*per .. nb-per-t*per.
__device__ __forceinline__ void find_bin(Shared &sh, int nb, unsigned need)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int per = nb >= kThreads ? nb / kThreads : 1;
    const int hi = nb - 1 - tid * per;                 // first (highest) owned bin
    unsigned local = 0;
    if (hi >= 0)
        for (int j = 0; j < per; j++)
            local += sh.hist[hi - j];
    unsigned incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        sh.warp_tot[wid] = incl;
    __syncthreads();
    unsigned before = 0;
    for (int w = 0; w < wid; w++)
        before += sh.warp_tot[w];
    incl += before;
    const unsigned excl = incl - local;
    if (hi >= 0 && excl < need && need <= incl) {
        unsigned cum = excl;
        for (int j = 0; j < per; j++) {
            const unsigned hb = sh.hist[hi - j];
            if (cum + hb >= need) {
                sh.bin = (unsigned)(hi - j);
                sh.need = need - cum;
                break;
            }
            cum += hb;
        }
    }
    __syncthreads();
}

// Top-k of positions [0, V) of `src` (V > k) by (key descending, position
// ascending), written to out[0..k) in position order. Positions must be in
// ascending order of the index they report, so ties go to lower indices.
// The k-th largest key T is found with three radix digits (12, 12 and 8
// bits, most significant first). The first histogram is built while the row
// is staged; the keys of its threshold bin are then set aside (when there are
// at most kCand) so that the other two digits scan only them. The compaction
// gives every warp one
// contiguous segment of positions: the counts of keys above T and equal to T
// per segment decide, after one barrier, where each warp writes and how many
// of the keys equal to T it may still take.
template <bool RES, typename Src>
__device__ void block_select_t(const Src &src, int V, int k, int32_t *__restrict__ out,
                               uint32_t *keys, Shared &sh)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    auto key_at = [&](int s) -> uint32_t { return RES ? keys[s] : src.key(s); };
    // digit 1 (top 12 bits): histogram while the row is staged (or read)
    for (int b = tid; b < 4096; b += kThreads)
        sh.hist[b] = 0;
    if (tid == 0)
        sh.ncand = 0;
    __syncthreads();
    if (RES) {
        src.stage(keys, V, sh.hist);
    } else {
        for (int s = tid; s < V; s += kThreads)
            atomicAdd(&sh.hist[src.key(s) >> 20], 1u);
    }
    __syncthreads();
    find_bin(sh, 4096, (unsigned)k);
    uint32_t prefix = sh.bin << 20, pmask = 0xfff00000u;
    unsigned need = sh.need;
    const unsigned c1 = sh.hist[sh.bin];
    __syncthreads();                                    // sh.bin / sh.need reused
    // digits 2 and 3 (12 and 8 bits) over the keys of that bin only: kept
    // aside when there are few of them, else re-read from the row
    const bool few = c1 <= (unsigned)kCand;
    if (few) {
        for (int s = tid; s < V; s += kThreads) {
            const uint32_t u = key_at(s);
            if ((u & pmask) == prefix)
                sh.cand[atomicAdd(&sh.ncand, 1u)] = u;
        }
    }
#pragma unroll 1
    for (int p = 1; p < 3; p++) {
        const int shift = p == 1 ? 8 : 0;
        const int nb = p == 1 ? 4096 : 256;
        for (int b = tid; b < nb; b += kThreads)
            sh.hist[b] = 0;
        __syncthreads();
        if (few) {
            for (int j = tid; j < (int)c1; j += kThreads) {
                const uint32_t u = sh.cand[j];
                if ((u & pmask) == prefix)
                    atomicAdd(&sh.hist[(u >> shift) & (unsigned)(nb - 1)], 1u);
            }
        } else {
            for (int s = tid; s < V; s += kThreads) {
                const uint32_t u = key_at(s);
                if ((u & pmask) == prefix)
                    atomicAdd(&sh.hist[(u >> shift) & (unsigned)(nb - 1)], 1u);
            }
        }
        __syncthreads();
        find_bin(sh, nb, need);
        prefix |= sh.bin << shift;
        pmask |= (unsigned)(nb - 1) << shift;
        need = sh.need;
        __syncthreads();                                // sh.bin / sh.need reused
    }
    const uint32_t T = prefix;

    // compaction in position order, one contiguous segment per warp
    const int seg = ((V + kWarps - 1) / kWarps + 31) & ~31;
    const int w0 = wid * seg, w1 = w0 + seg < V ? w0 + seg : V;
    unsigned ngt = 0, neq = 0;                          // per lane, summed below
    for (int s = w0 + lane; s < w1; s += 32) {
        const uint32_t u = key_at(s);
        ngt += u > T;
        neq += u == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
        neq += __shfl_xor_sync(0xffffffffu, neq, o);
    }
    if (lane == 0) {
        sh.warp_cnt[0][wid] = ngt;
        sh.warp_cnt[1][wid] = neq;
    }
    __syncthreads();
    unsigned gt_before = 0, eq_before = 0;
    for (int w = 0; w < wid; w++) {
        gt_before += sh.warp_cnt[0][w];
        eq_before += sh.warp_cnt[1][w];
    }
    unsigned base = gt_before + (eq_before < need ? eq_before : need);
    unsigned eq_seen = eq_before;
    const unsigned lt = (1u << lane) - 1u;
    for (int s0 = w0; s0 < w1; s0 += 32) {
        const int s = s0 + lane;
        const uint32_t u = s < w1 ? key_at(s) : 0u;
        const bool gt = s < w1 && u > T;
        const bool eq = s < w1 && u == T;
        const unsigned eqb = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eqb & lt) < need);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        const unsigned pos = base + __popc(tb & lt);
        if (take && pos < (unsigned)k)
            out[pos] = src.index(s);
        base += __popc(tb);
        eq_seen += __popc(eqb);
    }
}

template <typename Src>
__device__ void block_select(const Src &src, int64_t V, int k, int32_t *__restrict__ out,
                             uint32_t *keys, bool res, Shared &sh)
{
    if (res)
        block_select_t<true>(src, (int)V, k, out, keys, sh);
    else
        block_select_t<false>(src, (int)V, k, out, keys, sh);
}

__global__ void __launch_bounds__(kThreads)
topk_kernel(const float *__restrict__ scores, int64_t rows, int64_t E, int64_t ld,
            const int64_t *__restrict__ q_pos, int m, int k, int32_t *__restrict__ idx,
            int resident, const int *__restrict__ row_flag)
{
    extern __shared__ uint32_t keys[];
    __shared__ Shared sh;
    __shared__ int fl[kThreads];
    auto one = [&](int64_t row) {
        const int64_t V = visible(q_pos[row], m, E);
        int32_t *out = idx + row * k;
        if (V <= k) {
            for (int j = threadIdx.x; j < k; j += kThreads)
                out[j] = j < V ? j : -1;
            return;
        }
        RowScores src{scores + row * ld};
        block_select(src, V, k, out, keys, resident && V <= kResident, sh);
        __syncthreads();                          // shared state reused by the next row
    };
    if (!row_flag) {
        one(blockIdx.x);                          // one row per block
        return;
    }
    // the flagged rows only: the flags of kThreads rows at a time, then the
    // flagged ones among them in turn
    for (int64_t r0 = (int64_t)blockIdx.x * kThreads; r0 < rows;
         r0 += (int64_t)gridDim.x * kThreads) {
        const int64_t my = r0 + threadIdx.x;
        const int f = my < rows ? row_flag[my] : 0;
        if (!__syncthreads_or(f))
            continue;
        fl[threadIdx.x] = f;
        __syncthreads();
        for (int j = 0; j < kThreads && r0 + j < rows; j++)
            if (fl[j])
                one(r0 + j);
        __syncthreads();                          // fl reused
    }
}

// ---------------------------------------------------------------------------
// Rows of 2049 .. 65535 entries (prefill), k <= 1024: one block of 16 warps
// per row, two blocks per SM.
//  1. A lower bound L from 1024 samples of the row (16 runs of 64 consecutive
//     entries spread over it): L is the 16-bit key prefix of the sample that
//     about 1.25 k + 4 sqrt(.) + 8 of the samples reach, when the row's k-th
//     largest entry is expected at k * 1024 / V of them.
//  2. Warp w reads its contiguous segment of the row and keeps the entries
//     with key >= L, in index order, in its own region of shared memory.
//  3. The exact top-k of the candidates (8-bit radix digits, histograms
//     updated once per group of equal digits of a warp), written in index
//     order: warp w's candidates follow those of warps < w.
// When the candidates are fewer than k or a warp's region overflows, steps 3
// run over the row itself (re-read from L2) instead: the result is the exact
// top-k of the row either way.

constexpr int kMidThreads = 512;
constexpr int kMidWarps = kMidThreads / 32;
constexpr int kMidCapW = 512;                 // candidates per warp region
constexpr int kMidMaxK = 1024;

template <typename IdxT>
struct SelShared {
    uint32_t ckey[kMidWarps][kMidCapW];
    IdxT cidx[kMidWarps][kMidCapW];
    uint32_t skey[1024];
    unsigned hist[256];
    unsigned wcnt[kMidWarps], wpre[kMidWarps], wpre2[kMidWarps];
    unsigned wgt[kMidWarps], weq[kMidWarps];
    unsigned bin, need, total;
    int fallback, last;
};
using MidShared = SelShared<uint16_t>;     // rows < 65536: 16-bit indices

// Adds 1 to hist[d] for every lane with `on`, one atomic per distinct d.
__device__ __forceinline__ void hist_add(unsigned *hist, unsigned d, bool on)
{
    const unsigned act = __ballot_sync(0xffffffffu, on);
    if (on) {
        const unsigned same = __match_any_sync(act, d);
        if ((threadIdx.x & 31) == __ffs(same) - 1)
            atomicAdd(&hist[d], (unsigned)__popc(same));
    }
}

// Digit of the 256-bin histogram (descending) where the count from the top
// reaches `need` (warp 0 scans; every thread reads the result after the
// barrier): sh.bin and sh.need (what is still needed inside that bin).
template <typename SH>
__device__ __forceinline__ void mid_find(SH &sh, unsigned need)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        unsigned local = 0;
#pragma unroll
        for (int j = 0; j < 8; j++)
            local += sh.hist[255 - 8 * lane - j];
        unsigned incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        const unsigned excl = incl - local;
        if (excl < need && need <= incl) {
            unsigned cum = excl;
            for (int j = 0; j < 8; j++) {
                const unsigned hb = sh.hist[255 - 8 * lane - j];
                if (cum + hb >= need) {
                    sh.bin = 255u - 8u * lane - j;
                    sh.need = need - cum;
                    break;
                }
                cum += hb;
            }
        }
    }
    __syncthreads();
}

// Exclusive prefix over warps of v (the same value on every lane of a warp):
// returns this warp's prefix.
__device__ __forceinline__ unsigned mid_warp_prefix(unsigned *slot, unsigned *pre, unsigned v)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0)
        slot[wid] = v;
    __syncthreads();
    if (threadIdx.x < 32) {
        const unsigned x = lane < kMidWarps ? slot[lane] : 0u;
        unsigned incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        if (lane < kMidWarps)
            pre[lane] = incl - x;
    }
    __syncthreads();
    return pre[wid];
}

// Element j of warp w: from its candidate region, or from its row segment.
template <typename SH>
struct MidSrc {
    const float *row;
    const SH *sh;
    int seg, V;
    bool cand;
    __device__ __forceinline__ int count(int w) const
    {
        if (cand)
            return (int)sh->wcnt[w];
        const int a = w * seg, b = a + seg < V ? a + seg : V;
        return b > a ? b - a : 0;
    }
    __device__ __forceinline__ uint32_t key(int w, int j) const
    {
        return cand ? sh->ckey[w][j] : float_key(__ldg(row + w * seg + j));
    }
    __device__ __forceinline__ int32_t index(int w, int j) const
    {
        return cand ? (int32_t)sh->cidx[w][j] : (int32_t)(w * seg + j);
    }
};

// Exact top-k of the source (more than k elements in total), written to out
// in index order; ties at the k-th key go to the lower indices.
template <typename SH>
__device__ void mid_select(const MidSrc<SH> &src, int k, int32_t *__restrict__ out, SH &sh)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int n = src.count(wid);
    uint32_t prefix = 0, pmask = 0;
    unsigned need = (unsigned)k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        if (threadIdx.x < 256)
            sh.hist[threadIdx.x] = 0;
        __syncthreads();
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t u = j < n ? src.key(wid, j) : 0u;
            hist_add(sh.hist, (u >> shift) & 255u, j < n && (u & pmask) == prefix);
        }
        __syncthreads();
        mid_find(sh, need);
        prefix |= sh.bin << shift;
        pmask |= 255u << shift;
        need = sh.need;
        __syncthreads();                                   // hist, bin, need reused
    }
    const uint32_t T = prefix;
    // every warp: its count of keys above T and equal to T, then the prefix
    // over warps decides where it writes and how many of the ties it takes
    unsigned ngt = 0, neq = 0;
    for (int j = lane; j < n; j += 32) {
        const uint32_t u = src.key(wid, j);
        ngt += u > T;
        neq += u == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
        neq += __shfl_xor_sync(0xffffffffu, neq, o);
    }
    const unsigned gt_before = mid_warp_prefix(sh.wgt, sh.wpre, ngt);
    const unsigned eq_before = mid_warp_prefix(sh.weq, sh.wpre2, neq);
    unsigned base = gt_before + (eq_before < need ? eq_before : need);
    unsigned eq_seen = eq_before;
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < n; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t u = j < n ? src.key(wid, j) : 0u;
        const bool gt = j < n && u > T;
        const bool eq = j < n && u == T;
        const unsigned eqb = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eqb & lt) < need);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        const unsigned pos = base + __popc(tb & lt);
        if (take && pos < (unsigned)k)
            out[pos] = src.index(wid, j);
        base += __popc(tb);
        eq_seen += __popc(eqb);
    }
}

__global__ void __launch_bounds__(kMidThreads, 2)
topk_mid_kernel(const float *__restrict__ scores, int64_t E, int64_t ld,
                const int64_t *__restrict__ q_pos, int m, int k, int32_t *__restrict__ idx)
{
    extern __shared__ uint8_t dyn[];
    MidShared &sh = *reinterpret_cast<MidShared *>(dyn);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const int V = (int)visible(q_pos[row], m, E);
    int32_t *out = idx + row * k;
    if (V <= k) {
        for (int j = tid; j < k; j += kMidThreads)
            out[j] = j < V ? j : -1;
        return;
    }
    const float *src = scores + row * ld;
    if (tid == 0)
        sh.fallback = 0;
    __syncthreads();
    // segments of the row: a multiple of 4 entries per warp
    const int seg = ((V + kMidWarps - 1) / kMidWarps + 3) & ~3;
    // 1. lower bound from the samples: warp w reads runs at two places
    uint32_t L = 0;
    if (V > 4 * k) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int r = wid * 2 + h;                          // run 0..31
            const int s0 = (int)(((int64_t)r * V) / 32);
            const int si = s0 + lane < V ? s0 + lane : V - 1;
            sh.skey[r * 32 + lane] = float_key(__ldg(src + si));
        }
        const float mu = (float)k * 1024.f / (float)V;
        unsigned ks = (unsigned)(1.25f * mu + 4.f * sqrtf(mu) + 8.f);
        ks = ks > 1024u ? 1024u : ks;
        uint32_t pre = 0, msk = 0;
        unsigned nd = ks;
#pragma unroll 1
        for (int shift = 24; shift >= 16; shift -= 8) {
            if (tid < 256)
                sh.hist[tid] = 0;
            __syncthreads();
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const uint32_t u = sh.skey[tid * 2 + h];
                hist_add(sh.hist, (u >> shift) & 255u, (u & msk) == pre);
            }
            __syncthreads();
            mid_find(sh, nd);
            pre |= sh.bin << shift;
            msk |= 255u << shift;
            nd = sh.need;
            __syncthreads();
        }
        L = pre;
    }
    // 2. candidates: warp w's segment, 128 entries per step (4 per lane),
    // kept in index order in the warp's region; the loads of four steps are
    // issued before any of them is used
    {
        const int a0 = wid * seg, a1 = a0 + seg < V ? a0 + seg : V;
        const bool vec = (((uintptr_t)(src + a0)) & 15u) == 0;
        unsigned cnt = 0;
        bool over = false;
        for (int b0 = a0; b0 < a1; b0 += 4 * 128) {
            uint32_t u[4][4];
#pragma unroll
            for (int st = 0; st < 4; st++) {
                const int p = b0 + st * 128 + 4 * lane;
                if (vec && p + 3 < a1) {
                    const float4 f = __ldg((const float4 *)(src + p));
                    u[st][0] = float_key(f.x);
                    u[st][1] = float_key(f.y);
                    u[st][2] = float_key(f.z);
                    u[st][3] = float_key(f.w);
                } else {
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        u[st][j] = p + j < a1 ? float_key(__ldg(src + p + j)) : 0u;
                }
            }
#pragma unroll
            for (int st = 0; st < 4; st++) {
                const int p = b0 + st * 128 + 4 * lane;
                unsigned c = 0;
#pragma unroll
                for (int j = 0; j < 4; j++)
                    c += (p + j < a1 && u[st][j] >= L) ? 1u : 0u;
                unsigned incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o)
                        incl += y;
                }
                unsigned pos = cnt + incl - c;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    if (p + j < a1 && u[st][j] >= L) {
                        if (pos < (unsigned)kMidCapW) {
                            sh.ckey[wid][pos] = u[st][j];
                            sh.cidx[wid][pos] = (uint16_t)(p + j);
                        }
                        ++pos;
                    }
                }
                cnt += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        over = cnt > (unsigned)kMidCapW;
        if (lane == 0) {
            sh.wcnt[wid] = over ? 0u : cnt;
            if (over)
                sh.fallback = 1;
        }
    }
    if (tid == 0)
        sh.total = 0;
    __syncthreads();
    if (tid < 32) {
        unsigned t = tid < kMidWarps ? sh.wcnt[tid] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            t += __shfl_xor_sync(0xffffffffu, t, o);
        if (tid == 0)
            sh.total = t;
    }
    __syncthreads();
    const bool fb = sh.fallback || sh.total < (unsigned)k;
    __syncthreads();
    MidSrc<MidShared> ms{src, &sh, seg, V, !fb};
    mid_select(ms, k, out, sh);
}

// ---------------------------------------------------------------------------
// Rows longer than the cluster path takes: the row is cut into chunks of
// kChunk entries handled by separate blocks, in four launches:
//   1. per-chunk histograms of the top 12 key bits;
//   2. the row's bin totals, a slice of bins per block;
//   3. per chunk: the bin b that holds the k-th largest key (from the totals,
//      worked out again by every block), then the chunk's candidates (keys
//      in bins >= b) compacted in index order into the chunk's own region;
//   4. per row: the candidate lists joined in chunk order, then the exact
//      block radix select over them.
// Scratch (caller workspace): histograms, totals, counts and candidate lists.

constexpr int64_t kChunk = 8192;
constexpr int kBins = 4096;
constexpr int64_t kMultiMinE = 65536;
constexpr int kCollectThreads = 512;

struct MultiWs {
    uint32_t *hist;      // [rows][nchunks][kBins]
    uint32_t *tot;       // [rows][kBins]
    uint32_t *cnt;       // [rows][nchunks] candidates per chunk
    uint32_t *ckey;      // [rows][E]  chunk c's candidates at c * kChunk
    int32_t *cidx;       // [rows][E]
    uint32_t *jkey;      // [rows][E]  joined candidate lists
    int32_t *jidx;       // [rows][E]
};

__host__ __device__ inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

__host__ __device__ inline MultiWs multi_ws(void *base, int64_t rows, int64_t E)
{
    const int64_t nchunks = (E + kChunk - 1) / kChunk;
    MultiWs w;
    char *p = (char *)base;
    w.hist = (uint32_t *)p;
    p += align256(rows * nchunks * kBins * sizeof(uint32_t));
    w.tot = (uint32_t *)p;
    p += align256(rows * kBins * sizeof(uint32_t));
    w.cnt = (uint32_t *)p;
    p += align256(rows * nchunks * sizeof(uint32_t));
    w.ckey = (uint32_t *)p;
    p += align256(rows * E * sizeof(uint32_t));
    w.cidx = (int32_t *)p;
    p += align256(rows * E * sizeof(int32_t));
    w.jkey = (uint32_t *)p;
    p += align256(rows * E * sizeof(uint32_t));
    w.jidx = (int32_t *)p;
    return w;
}

__host__ __device__ inline size_t multi_ws_bytes(int64_t rows, int64_t E)
{
    const int64_t nchunks = (E + kChunk - 1) / kChunk;
    return align256(rows * nchunks * kBins * sizeof(uint32_t)) +
           align256(rows * kBins * sizeof(uint32_t)) + align256(rows * nchunks * sizeof(uint32_t)) +
           4 * align256(rows * E * sizeof(uint32_t));
}

__global__ void __launch_bounds__(256)
topk_hist_kernel(const float *__restrict__ scores, int64_t E, int64_t ld,
                 const int64_t *__restrict__ q_pos, int m, int k, MultiWs w)
{
    __shared__ uint32_t hist[kBins];
    const int64_t row = blockIdx.y, c = blockIdx.x;
    const int64_t nchunks = gridDim.x;
    const int64_t V = visible(q_pos[row], m, E);
    for (int b = threadIdx.x; b < kBins; b += blockDim.x)
        hist[b] = 0;
    __syncthreads();
    if (V > k) {
        const float *src = scores + row * ld;
        const int64_t s1 = (c + 1) * kChunk < V ? (c + 1) * kChunk : V;
        for (int64_t s = c * kChunk + threadIdx.x; s < s1; s += blockDim.x)
            atomicAdd(&hist[float_key(src[s]) >> 20], 1u);
    }
    __syncthreads();
    uint32_t *dst = w.hist + (row * nchunks + c) * kBins;
    for (int b = threadIdx.x; b < kBins; b += blockDim.x)
        dst[b] = hist[b];
}

// Totals of a 256-bin slice of one row (grid: 16 slices x rows).
__global__ void __launch_bounds__(256)
topk_total_kernel(int nchunks, MultiWs w)
{
    const int64_t row = blockIdx.y;
    const int b = blockIdx.x * 256 + threadIdx.x;
    const uint32_t *h = w.hist + row * (int64_t)nchunks * kBins + b;
    uint32_t t = 0;
    int c = 0;
    for (; c + 4 <= nchunks; c += 4)
        t += h[(int64_t)c * kBins] + h[(int64_t)(c + 1) * kBins] + h[(int64_t)(c + 2) * kBins] +
             h[(int64_t)(c + 3) * kBins];
    for (; c < nchunks; c++)
        t += h[(int64_t)c * kBins];
    w.tot[row * kBins + b] = t;
}

__global__ void __launch_bounds__(kCollectThreads)
topk_collect_kernel(const float *__restrict__ scores, int64_t E, int64_t ld,
                    const int64_t *__restrict__ q_pos, int m, int k, MultiWs w)
{
    constexpr int NW = kCollectThreads / 32;
    constexpr int PER = kChunk / kCollectThreads;       // keys per thread (16)
    __shared__ uint32_t wsum[NW];
    __shared__ uint32_t s_b0;
    const int64_t row = blockIdx.y, c = blockIdx.x;
    const int nchunks = gridDim.x;
    const int64_t V = visible(q_pos[row], m, E);
    if (V <= k)
        return;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // the bin of the k-th largest key: thread i owns bins 4095-8i .. 4088-8i
    {
        const uint32_t *tot = w.tot + row * kBins;
        uint32_t tb[8], local = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            tb[j] = tot[kBins - 1 - 8 * tid - j];
            local += tb[j];
        }
        uint32_t v = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o)
                v += x;
        }
        if (lane == 31)
            wsum[wid] = v;
        __syncthreads();
        uint32_t before = 0;
        for (int j = 0; j < wid; j++)
            before += wsum[j];
        const uint32_t incl = v + before, excl = incl - local;
        if (excl < (uint32_t)k && (uint32_t)k <= incl) {
            uint32_t cum = excl;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                cum += tb[j];
                if (cum >= (uint32_t)k) {
                    s_b0 = (uint32_t)(kBins - 1 - 8 * tid - j);
                    break;
                }
            }
        }
        __syncthreads();
    }
    const uint32_t b0 = s_b0;
    // warp wid covers entries [c0 + 512 wid, +512) of the chunk, 32 at a time
    const float *src = scores + row * ld;
    const int64_t c0 = c * kChunk, s1 = c0 + kChunk < V ? c0 + kChunk : V;
    const int64_t wbase = c0 + (int64_t)wid * (32 * PER);
    uint32_t key[PER];
    uint32_t mine = 0;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int64_t sidx = wbase + i * 32 + lane;
        key[i] = sidx < s1 ? float_key(src[sidx]) : 0u;
        mine += (sidx < s1 && (key[i] >> 20) >= b0) ? 1u : 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mine += __shfl_xor_sync(0xffffffffu, mine, o);
    __syncthreads();                       // wsum reused
    if (lane == 0)
        wsum[wid] = mine;
    __syncthreads();
    uint32_t base = 0, total = 0;
    for (int j = 0; j < NW; j++) {
        base += j < wid ? wsum[j] : 0u;
        total += wsum[j];
    }
    uint32_t *ck = w.ckey + row * E + c0;
    int32_t *ci = w.cidx + row * E + c0;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int64_t sidx = wbase + i * 32 + lane;
        const bool cand = sidx < s1 && (key[i] >> 20) >= b0;
        const unsigned bal = __ballot_sync(0xffffffffu, cand);
        if (cand) {
            const uint32_t pos = base + __popc(bal & lt);
            ck[pos] = key[i];
            ci[pos] = (int32_t)sidx;
        }
        base += __popc(bal);
    }
    if (tid == 0)
        w.cnt[row * nchunks + c] = total;
}

__global__ void __launch_bounds__(kThreads)
topk_final_kernel(const int64_t *__restrict__ q_pos, int64_t E, int m, int k, int nchunks,
                  MultiWs w, int32_t *__restrict__ idx)
{
    extern __shared__ uint32_t keys[];
    __shared__ Shared sh;
    __shared__ uint32_t offs[1025];
    const int64_t row = blockIdx.x;
    const int64_t V = visible(q_pos[row], m, E);
    int32_t *out = idx + row * k;
    if (V <= k) {
        for (int j = threadIdx.x; j < k; j += kThreads)
            out[j] = j < V ? j : -1;
        return;
    }
    // join the chunks' lists in chunk order (so in index order): offsets by
    // a warp scan over the counts, then one warp per chunk copies
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (wid == 0) {
        uint32_t run = 0;
        for (int c0 = 0; c0 < nchunks; c0 += 32) {
            const int c = c0 + lane;
            const uint32_t n = c < nchunks ? w.cnt[row * nchunks + c] : 0u;
            uint32_t x = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (c < nchunks)
                offs[c] = run + x - n;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            offs[nchunks] = run;
    }
    __syncthreads();
    const int64_t C = offs[nchunks];
    uint32_t *jk = w.jkey + row * E;
    int32_t *ji = w.jidx + row * E;
    for (int c = wid; c < nchunks; c += kWarps) {
        const uint32_t o = offs[c], n = offs[c + 1] - o;
        const uint32_t *sk = w.ckey + row * E + (int64_t)c * kChunk;
        const int32_t *si = w.cidx + row * E + (int64_t)c * kChunk;
        for (uint32_t j = lane; j < n; j += 32) {
            jk[o + j] = sk[j];
            ji[o + j] = si[j];
        }
    }
    __syncthreads();
    RowCandidates src{jk, ji};
    block_select(src, C, k, out, keys, C <= kResident, sh);
}

// ---------------------------------------------------------------------------
// Long rows of up to kCluCtas * kCluChunk entries (decode over a 1 M-token
// context: 262144 entries): one launch, each row taken by a cluster of
// kCluCtas blocks, block c staging the keys of its contiguous share of the
// row in shared memory (bulk copies; plain loads when the share does not
// start on a 16-byte boundary). The blocks talk through distributed shared
// memory and hardware cluster barriers only.
//  1. Bound: every 32nd key of the row is a sample; with mu = k ns / V the
//     samples expected at or above the row's k-th largest key, a bound with
//     ks = 1.25 mu + 4 sqrt(mu) + 8 samples at or above it lies below that
//     key unless the sample is off by many standard deviations. Each block
//     takes the ceil(ks / kCluCtas)-th largest of its own samples (every
//     warp's largest ones by repeated warp maxima, merged by one warp); the
//     smallest of the blocks' values has at least ks samples at or above it.
//  2. Candidates: each warp keeps the (key, index) pairs of its 1024 entries
//     at or above the bound in its own region, in index order.
//  3. When the candidates number at least k and every region held its own,
//     block 0 gathers them in index order and selects exactly (digits from
//     the first bit in which the candidates differ, ties to the lower index);
//     the k-th largest key is at or above the bound, so every key that can
//     be selected is a candidate.
//  4. Otherwise (a bound that turned out too high, or candidates crowding one
//     part of the row) the cluster selects over all keys: three radix rounds
//     (11, 11, 10 bits) in which every block counts the digits of its keys
//     that match the prefix so far and reads the other blocks' counts, then
//     one more exchange of the counts above the threshold key and equal to it,
//     after which each block writes its own elements in index order.
constexpr int kCluCtas = 8;
constexpr int kCluThreads = 1024;
constexpr int kCluWarps = kCluThreads / 32;
constexpr int kCluChunk = 32768;                  // keys per block (128 KB of shared memory)
constexpr int kCluBins = 2048;
constexpr int kCluCopies = 4;
constexpr int kCluStep = 32;                      // sample spacing
constexpr int kCluRegion = 128;                   // candidate pairs per warp
constexpr int kCluGather = kCluChunk / 2;         // pairs block 0 gathers (in its key area)
constexpr int kCluSel = 256;                      // threads of block 0 that select among them
constexpr size_t kCluSmem =
    (size_t)(kCluChunk + kCluCopies * kCluBins + 2 * kCluBins + kCluBins) * sizeof(uint32_t);
static_assert(kCluWarps * kCluRegion * 2 <= kCluCopies * kCluBins, "regions alias the counters");
static_assert(kCluChunk / kCluStep <= kCluThreads, "one sample per thread");

__host__ __device__ inline bool cluster_takes(int64_t rows, int64_t E)
{
    return rows > 0 && rows <= 65535 && E >= kMultiMinE && E <= (int64_t)kCluCtas * kCluChunk;
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_map(const void *local, uint32_t rank)
{
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(local);
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    return ra;
}

// A 32-bit word of block `rank`'s shared memory, at the place `local` has in ours.
__device__ __forceinline__ uint32_t cluster_ld(const uint32_t *local, uint32_t rank)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_map(local, rank))
                 : "memory");
    return v;
}

__device__ __forceinline__ uint2 cluster_ld2(const uint2 *local, uint32_t rank)
{
    uint2 v;
    asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "r"(cluster_map(local, rank))
                 : "memory");
    return v;
}

struct CluShared {
    uint32_t wa[kCluWarps], wb[kCluWarps];
    uint32_t wcnt[kCluWarps];                     // candidates of each warp (read by block 0)
    uint32_t pre[kCluCtas][kCluWarps + 1];        // block 0: where each region's pairs go
    uint32_t samp[kCluThreads];
    uint32_t tl[kCluWarps][32];                   // each warp's largest samples
    uint32_t bin, above, off, take, x, L, nc, ovf, fast;
    uint32_t cnt[2];                              // published: keys > T, keys == T
    uint64_t staged;                              // the bulk copies of the share landed
    int never;                                    // an abort flag nothing sets
};

// Barrier of the first NT threads of the block (all of them: barrier 0;
// fewer: named barrier 1, which nothing else uses).
template <int NT>
__device__ __forceinline__ void team_sync()
{
    if (NT == kCluThreads)
        __syncthreads();
    else
        asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// Of the counts cnt[0 .. kCluBins) (digits), the digit holding the need-th
// largest element counted from the top, and how many lie above it, worked out
// by the first NT threads. Call with cnt complete and visible to them; the
// result is in sh.bin / sh.above after the closing barrier. Thread i owns the
// PER digits below 2047 - PER i.
template <int NT>
__device__ __forceinline__ void clu_find(const uint32_t *cnt, uint32_t need, CluShared &sh)
{
    constexpr int PER = kCluBins / NT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int top = kCluBins - 1 - PER * tid;
    uint32_t t[PER], loc = 0;
#pragma unroll
    for (int u = 0; u < PER; u++) {
        t[u] = cnt[top - u];
        loc += t[u];
    }
    uint32_t v = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o)
            v += x;
    }
    if (lane == 31)
        sh.wa[warp] = v;
    team_sync<NT>();
    uint32_t before = 0;
    if (lane < warp)
        before = sh.wa[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        before += __shfl_xor_sync(0xffffffffu, before, o);
    const uint32_t incl = v + before, excl = incl - loc;
    if (excl < need && need <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int u = 0; u < PER; u++) {
            if (cum + t[u] >= need) {
                sh.bin = (uint32_t)(top - u);
                sh.above = cum;
                break;
            }
            cum += t[u];
        }
    }
    team_sync<NT>();
}

// Exclusive prefix over the first NT threads of two per-thread counts, and
// their totals.
template <int NT>
__device__ __forceinline__ void clu_scan2(uint32_t a, uint32_t b, CluShared &sh, uint32_t *a_before,
                                          uint32_t *b_before, uint32_t *a_tot, uint32_t *b_tot)
{
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t va = a, vb = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t xa = __shfl_up_sync(0xffffffffu, va, o);
        const uint32_t xb = __shfl_up_sync(0xffffffffu, vb, o);
        if (lane >= o) {
            va += xa;
            vb += xb;
        }
    }
    if (lane == 31) {
        sh.wa[warp] = va;
        sh.wb[warp] = vb;
    }
    team_sync<NT>();
    const uint32_t wa = lane < NW ? sh.wa[lane] : 0u, wb = lane < NW ? sh.wb[lane] : 0u;
    uint32_t pa = lane < warp ? wa : 0u, pb = lane < warp ? wb : 0u, ta = wa, tb = wb;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, o);
        pb += __shfl_xor_sync(0xffffffffu, pb, o);
        ta += __shfl_xor_sync(0xffffffffu, ta, o);
        tb += __shfl_xor_sync(0xffffffffu, tb, o);
    }
    *a_before = pa + va - a;
    *b_before = pb + vb - b;
    *a_tot = ta;
    *b_tot = tb;
    team_sync<NT>();                                       // wa / wb are reused
}

// The exact top-k of C (key, index) pairs in index order (gk, gi), ties to
// the lower index, by the first kCluSel threads: the pairs' common top bits
// (from the smallest and largest key), then digits of up to 11 bits, the
// digit counts alternating between h0 and h1 (the next one cleared while the
// current one is filled); then an ordered write, each thread owning a run of
// consecutive pairs.
__device__ __forceinline__ void clu_select_team(const uint32_t *gk, const uint32_t *gi, uint32_t C,
                                                int k, uint32_t *h0, uint32_t *h1, int32_t *out,
                                                CluShared &sh)
{
    constexpr int NT = kCluSel, NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (uint32_t e = (uint32_t)tid; e < C; e += NT) {
        mn = min(mn, gk[e]);
        mx = max(mx, gk[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        sh.wa[warp] = mn;
        sh.wb[warp] = mx;
    }
    for (int b = tid; b < kCluBins; b += NT)
        h0[b] = 0;
    team_sync<NT>();
    mn = lane < NW ? sh.wa[lane] : 0xffffffffu;
    mx = lane < NW ? sh.wb[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    team_sync<NT>();                                     // wa / wb reused by clu_find
    int bits = mn == mx ? 0 : 32 - __clz(mn ^ mx);
    uint32_t pmask = bits == 32 ? 0u : ~((1u << bits) - 1u);
    uint32_t prefix = mn & pmask, need = (uint32_t)k;
    for (int r = 0; bits > 0; r++) {
        const int w = bits < 11 ? bits : 11;
        const int shift = bits - w;
        const uint32_t dm = (1u << w) - 1u;
        uint32_t *h = (r & 1) ? h1 : h0, *hn = (r & 1) ? h0 : h1;
        for (uint32_t e = (uint32_t)tid; e < C; e += NT) {
            const uint32_t kk = gk[e];
            if ((kk & pmask) == prefix)
                atomicAdd(&h[(kk >> shift) & dm], 1u);
        }
        for (int b = tid; b < kCluBins; b += NT)
            hn[b] = 0;
        team_sync<NT>();
        clu_find<NT>(h, need, sh);
        prefix |= sh.bin << shift;
        need -= sh.above;
        pmask |= dm << shift;
        bits = shift;
    }
    const uint32_t T = prefix;
    const uint32_t per = (C + NT - 1) / NT;
    const uint32_t e0 = (uint32_t)tid * per, e1 = min(C, e0 + per);
    uint32_t ng = 0, ne = 0;
    for (uint32_t e = e0; e < e1; e++) {
        ng += gk[e] > T ? 1u : 0u;
        ne += gk[e] == T ? 1u : 0u;
    }
    uint32_t g_b, e_b, g_t, e_t;
    clu_scan2<NT>(ng, ne, sh, &g_b, &e_b, &g_t, &e_t);
    uint32_t pos = g_b + min(e_b, need), er = e_b;
    for (uint32_t e = e0; e < e1; e++) {
        const uint32_t kk = gk[e];
        const bool sel = kk > T || (kk == T && er < need);
        er += kk == T ? 1u : 0u;
        if (sel && pos < (uint32_t)k)
            out[pos] = (int32_t)gi[e];
        pos += sel ? 1u : 0u;
    }
}

__global__ void __cluster_dims__(kCluCtas, 1, 1) __launch_bounds__(kCluThreads, 1)
topk_cluster_kernel(const float *__restrict__ scores, int64_t E, int64_t ld,
                    const int64_t *__restrict__ q_pos, int m, int k, int32_t *__restrict__ idx,
                    unsigned *err)
{
    extern __shared__ uint4 clu_smem[];
    uint32_t *keys = (uint32_t *)clu_smem;                  // [kCluChunk]
    uint32_t *hc = keys + kCluChunk;                        // [kCluCopies][kCluBins]
    uint2 *cand = (uint2 *)hc;                              //   or [kCluWarps][kCluRegion] pairs
    uint32_t *pub = hc + kCluCopies * kCluBins;             // [2][kCluBins] published counts
    uint32_t *tot = pub + 2 * kCluBins;                     // [kCluBins]
    __shared__ CluShared sh;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const uint32_t c = cluster_rank();
    const int64_t row = blockIdx.y;
    const int64_t V = visible(q_pos[row], m, E);
    int32_t *out = idx + row * k;
    if (V <= k) {
        // the same decision in every block of the cluster: no barrier follows
        for (int64_t j = (int64_t)c * kCluThreads + tid; j < k; j += kCluCtas * kCluThreads)
            out[j] = j < V ? (int32_t)j : -1;
        return;
    }
    // this block's share [b0, b0 + n) of the row, a multiple of 4 entries long
    const int64_t cs = (((V + kCluCtas - 1) / kCluCtas) + 3) & ~(int64_t)3;
    const int64_t b0 = (int64_t)c * cs;
    const int n = (int)(V - b0 < 0 ? 0 : (V - b0 < cs ? V - b0 : cs));
    const int ns_own = (n + kCluStep - 1) / kCluStep;
    const float *src = scores + row * ld + b0;
    if ((((uintptr_t)src) & 15u) == 0) {
        // the share's whole 16-byte words by bulk copies (pieces of 32 KB
        // from one thread), the last n % 4 entries by plain loads; then every
        // word turned into its key in place
        const int n4 = n >> 2;
        if (tid == 0) {
            sh.never = 0;
            tc::mbar_init(&sh.staged, 1);
            tc::fence_mbar_init();
        }
        __syncthreads();
        if (tid == 0) {
            tc::mbar_arrive_expect_tx(&sh.staged, (uint32_t)n4 * 16u);
            for (uint32_t off = 0; off < (uint32_t)n4 * 16u; off += 32768u) {
                const uint32_t len = min(32768u, (uint32_t)n4 * 16u - off);
                tc::bulk_load((uint8_t *)keys + off, (const uint8_t *)src + off, len, &sh.staged);
            }
        }
        for (int j = 4 * n4 + tid; j < n; j += kCluThreads) {
            keys[j] = float_key(__ldg(src + j));
            if ((j & (kCluStep - 1)) == 0)
                sh.samp[j / kCluStep] = keys[j];
        }
        if (!tc::mbar_wait(&sh.staged, 0, &sh.never, 100000000ull))
            report(err, CSA_ERR_TIMEOUT, K_TOPK, (unsigned)row, c);   // carries on: every
                                                                     // block keeps the
                                                                     // cluster's barriers
        uint4 *k4 = (uint4 *)keys;
#pragma unroll 4
        for (int i = tid; i < n4; i += kCluThreads) {
            const uint4 f = k4[i];
            const uint4 kk = make_uint4(float_key(__uint_as_float(f.x)), float_key(__uint_as_float(f.y)),
                                        float_key(__uint_as_float(f.z)), float_key(__uint_as_float(f.w)));
            k4[i] = kk;
            if ((i & 7) == 0)
                sh.samp[i >> 3] = kk.x;
        }
    } else {
#pragma unroll 8
        for (int j = tid; j < n; j += kCluThreads) {
            const uint32_t kk = float_key(__ldg(src + j));
            keys[j] = kk;
            if ((j & (kCluStep - 1)) == 0)
                sh.samp[j / kCluStep] = kk;
        }
    }
    __syncthreads();                           // keys and samples complete

    // ---- 1. the bound: the jl-th largest of this block's samples (each
    // warp's jl largest by repeated warp maxima, merged by warp 0), then the
    // smallest over the cluster
    {
        int64_t ns = 0;
        for (int q = 0; q < kCluCtas; q++) {
            const int64_t nq = V - q * cs < 0 ? 0 : (V - q * cs < cs ? V - q * cs : cs);
            ns += (nq + kCluStep - 1) / kCluStep;
        }
        const float mu = (float)k * (float)ns / (float)V;
        const int ks = (int)ceilf(1.25f * mu + 4.f * sqrtf(mu) + 8.f);
        const int jl = min((ks + kCluCtas - 1) / kCluCtas, 32);
        uint32_t v = tid < ns_own ? sh.samp[tid] : 0u;
        for (int it = 0; it < jl; it++) {
            uint32_t mx = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const unsigned who = __ballot_sync(0xffffffffu, v == mx);
            if (lane == __ffs(who) - 1)
                v = 0u;
            if (lane == 0)
                sh.tl[warp][it] = mx;
        }
        __syncthreads();
        uint32_t x = 0;
        if (warp == 0) {
            // lane l walks warp l's list (descending)
            int head = 0;
            uint32_t cur = sh.tl[lane][0];
            for (int it = 0; it < jl; it++) {
                uint32_t mx = cur;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                x = mx;
                const unsigned who = __ballot_sync(0xffffffffu, cur == mx);
                if (lane == __ffs(who) - 1) {
                    head++;
                    cur = head < jl ? sh.tl[lane][head] : 0u;
                }
            }
        }
        if (tid == 0)
            sh.x = x;
        // idle warps wait at the block barrier, not at the cluster barrier
        // (warps waiting there slow the ones still working)
        __syncthreads();
        cluster_arrive();
        cluster_wait();
        if (warp == 0) {
            uint32_t v = lane < kCluCtas ? cluster_ld(&sh.x, (uint32_t)lane) : 0xffffffffu;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0)
                sh.L = v;
        }
        __syncthreads();
    }
    const uint32_t L = sh.L;

    // ---- 2. candidates: warp w keeps its entries [1024 w, +1024) at or above L
    {
        const int wbase = warp * 1024;
        uint2 *reg = cand + warp * kCluRegion;
        uint32_t cnt = 0;
#pragma unroll 4
        for (int i = 0; i < 32; i++) {
            const int j = wbase + 32 * i + lane;
            const bool v = j < n;
            const uint32_t kk = v ? keys[j] : 0u;
            const bool on = v && kk >= L;
            const unsigned bal = __ballot_sync(0xffffffffu, on);
            const uint32_t at = cnt + __popc(bal & lt);
            if (on && at < (uint32_t)kCluRegion)
                reg[at] = make_uint2(kk, (uint32_t)(b0 + j));
            cnt += __popc(bal);
        }
        if (lane == 0)
            sh.wcnt[warp] = cnt;
        __syncthreads();
        if (warp == 0) {
            const uint32_t wc = sh.wcnt[lane];
            uint32_t tot_c = wc, ovf = wc > (uint32_t)kCluRegion ? 1u : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                tot_c += __shfl_xor_sync(0xffffffffu, tot_c, o);
                ovf |= __shfl_xor_sync(0xffffffffu, ovf, o);
            }
            if (lane == 0) {
                sh.nc = tot_c;
                sh.ovf = ovf;
            }
        }
        __syncthreads();
    }
    cluster_arrive();
    cluster_wait();
    if (warp == 0) {
        const bool on = lane < kCluCtas;
        const uint32_t nq = on ? cluster_ld(&sh.nc, (uint32_t)lane) : 0u;
        uint32_t ov = on ? cluster_ld(&sh.ovf, (uint32_t)lane) : 0u;
        uint32_t ni = nq;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, ni, o);
            if (lane >= o)
                ni += x;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            ov |= __shfl_xor_sync(0xffffffffu, ov, o);
        const uint32_t C = __shfl_sync(0xffffffffu, ni, 31);
        if (lane < kCluCtas)
            sh.pre[lane][kCluWarps] = ni - nq;           // first pair of block `lane`
        if (lane == 0)
            sh.fast = (ov == 0u && C >= (uint32_t)k && C <= (uint32_t)kCluGather) ? C : 0u;
    }
    __syncthreads();
    const uint32_t C = sh.fast;

    if (C > 0) {
        // ---- 3. block 0 gathers the pairs in index order and selects
        uint32_t *gk = keys, *gi = keys + kCluGather;
        if (c == 0) {
            // group g of 128 threads copies block g's regions
            const int g = tid >> 7, gt = tid & 127;
            if ((gt >> 5) == 0) {
                const uint32_t wc = cluster_ld(&sh.wcnt[gt], (uint32_t)g);
                uint32_t v = wc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
                    if (gt >= o)
                        v += x;
                }
                sh.pre[g][gt] = v - wc;                  // region offsets inside block g
                if (gt == 31)
                    sh.wa[g] = v;                        // block g's pair count
            }
            __syncthreads();
            const uint32_t base = sh.pre[g][kCluWarps], ng = sh.wa[g];
            for (uint32_t f = (uint32_t)gt; f < ng; f += 128) {
                // the region holding pair f of block g: the last w with pre[g][w] <= f
                int lo = 0, hi = kCluWarps - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (sh.pre[g][mid] <= f)
                        lo = mid;
                    else
                        hi = mid - 1;
                }
                const uint2 pr = cluster_ld2(cand + lo * kCluRegion + (f - sh.pre[g][lo]), (uint32_t)g);
                gk[base + f] = pr.x;
                gi[base + f] = pr.y;
            }
        }
        // the other blocks may leave once block 0 has read their pairs
        cluster_arrive();
        if (c == 0) {
            __syncthreads();                             // the gathered pairs
            if (tid < kCluSel)
                clu_select_team(gk, gi, C, k, tot, pub, out, sh);
            __syncthreads();
        }
        cluster_wait();
        return;
    }

    // ---- 4. every key: three radix rounds over the whole row
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)k;
#pragma unroll 1
    for (int r = 0; r < 3; r++) {
        const int shift = r == 0 ? 21 : (r == 1 ? 10 : 0);
        const uint32_t dmask = r == 2 ? 1023u : 2047u;
        for (int b = tid; b < kCluCopies * kCluBins; b += kCluThreads)
            hc[b] = 0;
        __syncthreads();
        uint32_t *h = hc + (lane & (kCluCopies - 1)) * kCluBins;
#pragma unroll 4
        for (int j = tid; j < n; j += kCluThreads) {
            const uint32_t kk = keys[j];
            if ((kk & pmask) == prefix)
                atomicAdd(&h[(kk >> shift) & dmask], 1u);
        }
        __syncthreads();
        uint32_t *pr = pub + (r & 1) * kCluBins;
        for (int b = tid; b < kCluBins; b += kCluThreads)
            pr[b] = hc[b] + hc[kCluBins + b] + hc[2 * kCluBins + b] + hc[3 * kCluBins + b];
        // every block's counts of this round are published; the buffer of the
        // round before the last is free again (its readers have passed the
        // previous barrier)
        cluster_arrive();
        cluster_wait();
        for (int b = tid; b < kCluBins; b += kCluThreads) {
            uint32_t t = 0;
#pragma unroll
            for (int q = 0; q < kCluCtas; q++)
                t += cluster_ld(pr + b, (uint32_t)q);
            tot[b] = t;
        }
        __syncthreads();
        clu_find<kCluThreads>(tot, need, sh);
        prefix |= sh.bin << shift;
        pmask |= dmask << shift;
        need -= sh.above;
        __syncthreads();                       // sh.bin and sh.above are rewritten next round
    }
    const uint32_t T = prefix;

    // counts above T and equal to T: warp w covers entries [1024 w, +1024)
    const int wbase = warp * 1024;
    uint32_t gt = 0, eq = 0;
#pragma unroll 4
    for (int i = 0; i < 32; i++) {
        const int j = wbase + 32 * i + lane;
        const bool v = j < n;
        const uint32_t kk = v ? keys[j] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, v && kk > T));
        eq += __popc(__ballot_sync(0xffffffffu, v && kk == T));
    }
    // per-warp prefix (one lane per warp contributes the warp's counts)
    uint32_t gt_b, eq_b, gt_c, eq_c;
    clu_scan2<kCluThreads>(lane == 0 ? gt : 0u, lane == 0 ? eq : 0u, sh, &gt_b, &eq_b, &gt_c, &eq_c);
    gt_b = __shfl_sync(0xffffffffu, gt_b, 0);
    eq_b = __shfl_sync(0xffffffffu, eq_b, 0);
    if (tid == 0) {
        sh.cnt[0] = gt_c;
        sh.cnt[1] = eq_c;
    }
    cluster_arrive();
    cluster_wait();
    if (warp == 0) {
        // lane q < kCluCtas: block q's counts; ties go to the lowest blocks first
        const bool on = lane < kCluCtas;
        const uint32_t g = on ? cluster_ld(&sh.cnt[0], (uint32_t)lane) : 0u;
        const uint32_t e = on ? cluster_ld(&sh.cnt[1], (uint32_t)lane) : 0u;
        uint32_t ei = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o)
                ei += x;
        }
        const uint32_t ebefore = ei - e;
        const uint32_t take = need > ebefore ? (need - ebefore < e ? need - ebefore : e) : 0u;
        const uint32_t sel = g + take;
        uint32_t si = sel;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o)
                si += x;
        }
        if (lane == (int)c) {
            sh.off = si - sel;
            sh.take = take;
        }
    }
    // the other blocks' shared memory is not read past this point
    cluster_arrive();
    __syncthreads();
    const uint32_t take = sh.take;
    uint32_t eqrun = eq_b;
    uint32_t pos = sh.off + gt_b + (eq_b < take ? eq_b : take);
#pragma unroll 4
    for (int i = 0; i < 32; i++) {
        const int j = wbase + 32 * i + lane;
        const bool v = j < n;
        const uint32_t kk = v ? keys[j] : 0u;
        const bool ise = v && kk == T;
        const unsigned be = __ballot_sync(0xffffffffu, ise);
        const bool sel = (v && kk > T) || (ise && eqrun + __popc(be & lt) < take);
        const unsigned bs = __ballot_sync(0xffffffffu, sel);
        const uint32_t at = pos + __popc(bs & lt);
        if (sel && at < (uint32_t)k)
            out[at] = (int32_t)(b0 + j);
        eqrun += __popc(be);
        pos += __popc(bs);
    }
    // a block leaves only when no other block of its cluster can still read
    // its shared memory
    cluster_wait();
}

// ---------------------------------------------------------------------------
// Short rows (E <= 32 * kPerLane): one warp per row, keys held in registers,
// per-warp 256-bin histograms in shared memory, warp ballots for the
// compaction; no block-wide barrier at all.

constexpr int kPerLane = 64;
constexpr int kWarpRowsPerBlock = 8;

template <int PER>
__global__ void __launch_bounds__(32 * kWarpRowsPerBlock)
topk_warp_kernel(const float *__restrict__ scores, int64_t rows, int64_t E, int64_t ld,
                 const int64_t *__restrict__ q_pos, int m, int k, int32_t *__restrict__ idx)
{
    __shared__ unsigned hist_all[kWarpRowsPerBlock][256];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kWarpRowsPerBlock + w;
    if (row >= rows)
        return;
    unsigned *hist = hist_all[w];
    const int64_t V = visible(q_pos[row], m, E);
    int32_t *out = idx + row * k;
    if (V <= k) {
        for (int j = lane; j < k; j += 32)
            out[j] = j < V ? j : -1;
        return;
    }
    const float *src = scores + row * ld;
    uint32_t key[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int64_t s = (int64_t)i * 32 + lane;
        key[i] = s < V ? float_key(src[s]) : 0u;
    }
    uint32_t prefix = 0, pmask = 0;
    unsigned need = (unsigned)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
        for (int b = 0; b < 8; b++)
            hist[lane * 8 + b] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < PER; i++) {
            const int64_t s = (int64_t)i * 32 + lane;
            if (s < V && (key[i] & pmask) == prefix)
                atomicAdd(&hist[(key[i] >> shift) & 255u], 1u);
        }
        __syncwarp();
        // lane l owns bins 255-8l .. 248-8l (descending)
        unsigned local = 0;
#pragma unroll
        for (int j = 0; j < 8; j++)
            local += hist[255 - 8 * lane - j];
        unsigned incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off)
                incl += v;
        }
        const unsigned excl = incl - local;
        unsigned bin = 0, nneed = need;
        const bool mine = excl < need && need <= incl;
        if (mine) {
            unsigned cum = excl;
            for (int j = 0; j < 8; j++) {
                const int b = 255 - 8 * lane - j;
                const unsigned hb = hist[b];
                if (cum + hb >= need) {
                    bin = (unsigned)b;
                    nneed = need - cum;
                    break;
                }
                cum += hb;
            }
        }
        const unsigned owner = __ballot_sync(0xffffffffu, mine);
        const int src_lane = owner ? __ffs(owner) - 1 : 0;
        bin = __shfl_sync(0xffffffffu, bin, src_lane);
        nneed = __shfl_sync(0xffffffffu, nneed, src_lane);
        prefix |= bin << shift;
        pmask |= 255u << shift;
        need = nneed;
        __syncwarp();
    }
    const uint32_t T = prefix;
    unsigned base = 0, eq_seen = 0;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int64_t s = (int64_t)i * 32 + lane;
        const bool in = s < V;
        const bool gt = in && key[i] > T;
        const bool eq = in && key[i] == T;
        const unsigned eqb = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eqb & lt) < need);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        const unsigned pos = base + __popc(tb & lt);
        if (take && pos < (unsigned)k)
            out[pos] = (int32_t)s;
        base += __popc(tb);
        eq_seen += __popc(eqb);
    }
    for (int j = (int)base + lane; j < k; j += 32)
        out[j] = -1;
}

}  // namespace

// ---------------------------------------------------------------------------
// Selection from candidate pairs (the indexer's candidate mode, one key
// chunk per row). Row r holds `lists` lists of pairs (score bits, index):
// list l has cnt[r][l] pairs at cand[r * cand_ld + l * room ..] (room = the
// row's E / 2 pairs over the lists), in no particular order: every visible
// entry whose score is at or above the row's lower bound. When every list fits
// in its room and there are at least k pairs, the row's top-k is the top-k of
// its pairs. One warp per row finds the k-th largest key T and how many keys
// equal to T to take (8-bit radix digits, most significant first, over the
// lists one after another), marks the chosen indices in a bitmap of the
// row's visible range (the lowest indices among the keys equal to T through
// a second bitmap), and writes the set bits in index order. A row whose pairs
// overflowed or number fewer than k is flagged (flag[r] = 1) for the full
// computation; the others get 0.

constexpr int kCandRows = 8;           // rows (warps) per block
constexpr int kCandMaxLists = 8;

constexpr int kCandBin = 512;          // keys of the threshold bin kept aside

struct __align__(16) CandWarp {
    unsigned hist[256];
    unsigned bin, need, bcnt, nb;
};

// Shared memory of one row: the digit histogram, the bitmap of chosen
// indices, and an area that holds the threshold bin's pairs (or, on the
// slow path, the bitmap of the keys equal to the threshold).
// Bitmaps keep word w at w + w / 32, so that the runs of 32 words that the
// lanes scan fall in different banks.
__host__ __device__ inline int cand_padded(int words) { return (words + words / 32 + 4) & ~3; }
__device__ __forceinline__ int bmw(uint32_t w) { return (int)(w + (w >> 5)); }
__host__ __device__ inline size_t cand_aside_bytes(int words)
{
    const size_t a = (size_t)kCandBin * 8, b = (size_t)cand_padded(words) * 4;
    return a > b ? a : b;
}
// (every part a multiple of 16 bytes: the histogram is read as 16-byte words)
__host__ __device__ inline size_t cand_warp_bytes(int words)
{
    static_assert(sizeof(CandWarp) % 16 == 0, "CandWarp must keep 16-byte alignment");
    return sizeof(CandWarp) + (size_t)cand_padded(words) * 4 + cand_aside_bytes(words);
}

// Bin of the warp's 256-bin histogram (descending) where the count from the
// top reaches `need`: g.bin, g.need (what is still needed inside it), g.bcnt.
__device__ __forceinline__ void warp_find(CandWarp &g, unsigned need)
{
    // lane l owns bins 255 - 8 l down to 248 - 8 l, read as two 16-byte words
    const int lane = threadIdx.x & 31;
    const uint4 lo4 = *reinterpret_cast<const uint4 *>(g.hist + 248 - 8 * lane);
    const uint4 hi4 = *reinterpret_cast<const uint4 *>(g.hist + 252 - 8 * lane);
    const unsigned h[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};  // descending
    unsigned local = 0;
#pragma unroll
    for (int j = 0; j < 8; j++)
        local += h[j];
    unsigned incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    const unsigned ex = incl - local;
    if (ex < need && need <= incl) {
        unsigned cum = ex;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (cum < need && cum + h[j] >= need) {
                g.bin = 255u - 8u * lane - j;
                g.need = need - cum;
                g.bcnt = h[j];
            }
            cum += h[j];
        }
    }
    __syncwarp();
}

__device__ __forceinline__ unsigned warp_excl(unsigned v)
{
    const int lane = threadIdx.x & 31;
    unsigned incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    return incl - v;
}

__global__ void __launch_bounds__(32 * kCandRows)
topk_cand_kernel(const TopkCandArgs a, int words)
{
    extern __shared__ __align__(16) uint8_t cdyn[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint8_t *gbase = cdyn + (size_t)wid * cand_warp_bytes(words);
    CandWarp &g = *reinterpret_cast<CandWarp *>(gbase);
    uint32_t *bm_gt = (uint32_t *)(gbase + sizeof(CandWarp));
    uint8_t *aside = (uint8_t *)(bm_gt + cand_padded(words));
    uint32_t *akey = (uint32_t *)aside;                 // threshold bin: keys
    uint32_t *aidx = akey + kCandBin;                   //                indices
    uint32_t *bm_eq = (uint32_t *)aside;                // slow path: keys equal to T
    const int64_t row = (int64_t)blockIdx.x * kCandRows + wid;
    if (row >= a.rows)
        return;
    const int k = a.k;
    int32_t *out = a.idx + row * k;
    const int64_t V = visible(a.q_pos[row], a.m, a.E);
    if (V <= k) {
        for (int j = lane; j < k; j += 32)
            out[j] = j < V ? j : -1;
        if (lane == 0)
            a.flag[row] = 0;
        return;
    }
    // 1. the lists: counts (the same on every lane)
    const int L = a.lists;
    const unsigned room = (unsigned)(a.E / 2 / L);
    const uint32_t *ccnt = a.cnt + row * L;
    const uint2 *crow = a.cand + row * a.cand_ld;
    unsigned total = 0;
    bool over = false;
#pragma unroll
    for (int x = 0; x < kCandMaxLists; x++) {
        const unsigned n = x < L ? ccnt[x] : 0u;
        over |= n > room;
        total += n;
    }
    if (over || total < (unsigned)k) {
        if (lane == 0)
            a.flag[row] = 1;
        return;
    }
    // f(key, index, valid) for every pair of every list, eight loads in
    // flight per lane
    auto each = [&](auto &&f) {
#pragma unroll 1
        for (int x = 0; x < L; x++) {
            const uint2 *lp = crow + (int64_t)x * room;
            const unsigned n = __ldg(ccnt + x);
            for (unsigned f0 = 0; f0 < n; f0 += 256) {
                uint2 p[8];
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const unsigned j = f0 + i * 32 + lane;
                    p[i] = j < n ? lp[j] : make_uint2(0u, 0xffffffffu);
                }
#pragma unroll
                for (int i = 0; i < 8; i++)
                    f(float_key(__uint_as_float(p[i].x)), p[i].y, f0 + i * 32 + lane < n);
            }
        }
    };
    const int W = (int)((V + 31) / 32);
    for (int w = lane; w < W; w += 32)
        bm_gt[bmw(w)] = 0u;
    // 2. smallest and largest key: the bits above their highest differing
    // bit are common to every pair, so the first digit starts below them
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    each([&](uint32_t u, uint32_t, bool v) {
        if (v) {
            kmin = u < kmin ? u : kmin;
            kmax = u > kmax ? u : kmax;
        }
    });
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const int d = kmin == kmax ? 0 : 32 - __clz(kmin ^ kmax);   // differing low bits
    const int shift = d > 8 ? d - 8 : 0;
    // bits common to every key above the first digit [shift, shift + 8)
    const uint32_t hi = shift + 8 >= 32 ? 0u : (kmin & ~((1u << (shift + 8)) - 1u));
    // 3. histogram of the first digit, the bin b that holds the k-th largest
    uint32_t T = kmin;
    unsigned need = (unsigned)k, bcnt = total;
    bool fast = true;
    if (d > 0) {
        for (int b = lane; b < 256; b += 32)
            g.hist[b] = 0;
        __syncwarp();
        // (keys spread over many bins here: one shared atomic per key)
        each([&](uint32_t u, uint32_t, bool v) {
            if (v)
                atomicAdd(&g.hist[(u >> shift) & 255u], 1u);
        });
        __syncwarp();
        warp_find(g, need);
        const uint32_t bin = g.bin;
        need = g.need;
        bcnt = g.bcnt;
        // 4. keys above bin b are chosen; the pairs of bin b are set aside
        // (when they fit)
        fast = bcnt <= (unsigned)kCandBin;
        unsigned nb = 0;
        each([&](uint32_t u, uint32_t s, bool v) {
            const uint32_t dg = (u >> shift) & 255u;
            if (v && dg > bin && (int64_t)s < V)
                atomicOr(&bm_gt[bmw(s >> 5)], 1u << (s & 31u));
            const bool in = v && dg == bin;
            const unsigned bal = __ballot_sync(0xffffffffu, in);
            const unsigned at = nb + (unsigned)__popc(bal & ((1u << lane) - 1u));
            if (fast && in && at < (unsigned)kCandBin) {
                akey[at] = u;
                aidx[at] = s;
            }
            nb += (unsigned)__popc(bal);
        });
        __syncwarp();
        if (fast) {
            // 5. the digits below the first one, over the pairs set aside
            // (they all agree on the bits from `shift` up)
            uint32_t sp = 0u, sm = 0u;
            for (int sh = shift - 8; sh > -8; sh -= 8) {
                const int s0 = sh > 0 ? sh : 0;
                const uint32_t dm = 255u >> (sh < 0 ? -sh : 0);
                for (int b = lane; b < 256; b += 32)
                    g.hist[b] = 0;
                __syncwarp();
                for (unsigned j = lane; j < bcnt; j += 32) {
                    const uint32_t u = akey[j];
                    if ((u & sm) == sp)
                        atomicAdd(&g.hist[(u >> s0) & dm], 1u);
                }
                __syncwarp();
                warp_find(g, need);
                sp |= g.bin << s0;
                sm |= dm << s0;
                need = g.need;
                __syncwarp();
            }
            T = hi | (bin << shift) | sp;
            // 6. within the bin: keys above T chosen, keys equal to T by index
            unsigned neq = 0;
            for (unsigned j0 = 0; j0 < bcnt; j0 += 32) {
                const unsigned j = j0 + lane;
                neq += (unsigned)__popc(__ballot_sync(0xffffffffu, j < bcnt && akey[j] == T));
            }
            for (unsigned j0 = 0; j0 < bcnt; j0 += 32) {
                const unsigned j = j0 + lane;
                if (j < bcnt) {
                    const uint32_t u = akey[j], s = aidx[j];
                    bool take = u > T;
                    if (u == T) {
                        if (need >= neq) {
                            take = true;
                        } else {
                            unsigned rank = 0;                  // equal keys at lower indices
                            for (unsigned i = 0; i < bcnt; i++)
                                rank += (akey[i] == T && aidx[i] < s) ? 1u : 0u;
                            take = rank < need;
                        }
                    }
                    if (take && (int64_t)s < V)
                        atomicOr(&bm_gt[bmw(s >> 5)], 1u << (s & 31u));
                }
            }
            __syncwarp();
        }
    }
    if (d == 0) {
        // every pair has the same key: the k lowest indices
        for (int w = lane; w < W; w += 32)
            bm_eq[bmw(w)] = 0u;
        __syncwarp();
        each([&](uint32_t, uint32_t s, bool v) {
            if (v && (int64_t)s < V)
                atomicOr(&bm_eq[bmw(s >> 5)], 1u << (s & 31u));
        });
        __syncwarp();
        fast = false;
        need = (unsigned)k;
        bcnt = total;
        T = kmin;
    } else if (!fast) {
        // slow path (a threshold bin of more than kCandBin pairs): the
        // digits below the first one over all the pairs of bin b, then the
        // keys equal to T in a second bitmap
        const uint32_t bin = g.bin;
        uint32_t sp = 0u, sm = 0u;
        for (int sh = shift - 8; sh > -8; sh -= 8) {
            const int s0 = sh > 0 ? sh : 0;
            const uint32_t dm = 255u >> (sh < 0 ? -sh : 0);
            for (int b = lane; b < 256; b += 32)
                g.hist[b] = 0;
            __syncwarp();
            each([&](uint32_t u, uint32_t, bool v) {
                hist_add(g.hist, (u >> s0) & dm,
                         v && ((u >> shift) & 255u) == bin && (u & sm) == sp);
            });
            __syncwarp();
            warp_find(g, need);
            sp |= g.bin << s0;
            sm |= dm << s0;
            need = g.need;
            __syncwarp();
        }
        T = hi | (bin << shift) | sp;
        for (int w = lane; w < W; w += 32)
            bm_eq[bmw(w)] = 0u;
        __syncwarp();
        each([&](uint32_t u, uint32_t s, bool v) {
            if (v && (int64_t)s < V) {
                if (u > T && (u >> shift) == (T >> shift))   // above T inside bin b
                    atomicOr(&bm_gt[bmw(s >> 5)], 1u << (s & 31u));
                else if (u == T)
                    atomicOr(&bm_eq[bmw(s >> 5)], 1u << (s & 31u));
            }
        });
        __syncwarp();
    }
    const int wper = (W + 31) / 32;
    const int w0 = lane * wper, w1 = w0 + wper < W ? w0 + wper : W;
    if (!fast) {
        // the `need` lowest indices among the keys equal to T
        unsigned c = 0;
        for (int w = w0; w < w1; w++)
            c += (unsigned)__popc(bm_eq[bmw(w)]);
        unsigned e = warp_excl(c);
        for (int w = w0; w < w1 && e < need; w++) {
            uint32_t x = bm_eq[bmw(w)];
            const unsigned pc = (unsigned)__popc(x);
            if (e + pc > need) {
                unsigned keep = need - e;
                uint32_t y = 0u;
                while (keep--) {
                    const uint32_t lb = x & (0u - x);
                    y |= lb;
                    x ^= lb;
                }
                x = y;
            }
            bm_gt[bmw(w)] |= x;
            e += (unsigned)__popc(x);
        }
        __syncwarp();
    }
    // 7. the chosen indices in ascending order
    unsigned c = 0;
    for (int w = w0; w < w1; w++)
        c += (unsigned)__popc(bm_gt[bmw(w)]);
    unsigned e = warp_excl(c);
    const unsigned tot = __reduce_add_sync(0xffffffffu, c);
    for (int w = w0; w < w1; w++) {
        uint32_t x = bm_gt[bmw(w)];
        while (x) {
            const int b = __ffs(x) - 1;
            x &= x - 1u;
            if (e < (unsigned)k)
                out[e] = w * 32 + b;
            ++e;
        }
    }
    for (int j = (int)tot + lane; j < k; j += 32)
        out[j] = -1;
    if (lane == 0)
        a.flag[row] = 0;
}

bool topk_cand_fits(int64_t E, int nchunks, int lists, int64_t rows)
{
    (void)rows;
    const int words = (int)((E + 31) / 32);
    return nchunks == 1 && lists >= 1 && lists <= kCandMaxLists &&
           kCandRows * cand_warp_bytes(words) <= 227 * 1024;
}

cudaError_t launch_topk_cand(const TopkCandArgs &a, cudaStream_t s)
{
    if (a.rows == 0)
        return cudaSuccess;
    const int words = (int)((a.E + 31) / 32);
    const size_t smem = kCandRows * cand_warp_bytes(words);
    cudaError_t e = cudaFuncSetAttribute(topk_cand_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    topk_cand_kernel<<<(unsigned)((a.rows + kCandRows - 1) / kCandRows), 32 * kCandRows, smem,
                       s>>>(a, words);
    return cudaGetLastError();
}

size_t topk_workspace_size(int64_t rows, int64_t E, int k)
{
    (void)k;
    if (cluster_takes(rows, E) || E < kMultiMinE || rows > 65535 || rows <= 0 || (E + kChunk - 1) / kChunk > 1024)
        return 0;
    return multi_ws_bytes(rows, E);
}

cudaError_t launch_topk(const TopkArgs &a, unsigned *err, cudaStream_t s)
{
    if (a.rows == 0)
        return cudaSuccess;
    if (a.E <= 32 * kPerLane) {
        const unsigned blocks = (unsigned)((a.rows + kWarpRowsPerBlock - 1) / kWarpRowsPerBlock);
        if (a.E <= 32 * 16)
            topk_warp_kernel<16><<<blocks, 32 * kWarpRowsPerBlock, 0, s>>>(
                a.scores, a.rows, a.E, a.ld, a.q_pos, a.m, a.k, a.idx);
        else if (a.E <= 32 * 32)
            topk_warp_kernel<32><<<blocks, 32 * kWarpRowsPerBlock, 0, s>>>(
                a.scores, a.rows, a.E, a.ld, a.q_pos, a.m, a.k, a.idx);
        else
            topk_warp_kernel<64><<<blocks, 32 * kWarpRowsPerBlock, 0, s>>>(
                a.scores, a.rows, a.E, a.ld, a.q_pos, a.m, a.k, a.idx);
        return cudaGetLastError();
    }
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kResident * (int)sizeof(uint32_t));
    if (cluster_takes(a.rows, a.E)) {
        cudaError_t e = cudaFuncSetAttribute(
            topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCluSmem);
        if (e != cudaSuccess)
            return e;
        topk_cluster_kernel<<<dim3(kCluCtas, (unsigned)a.rows), kCluThreads, kCluSmem, s>>>(
            a.scores, a.E, a.ld, a.q_pos, a.m, a.k, a.idx, err);
        return cudaGetLastError();
    }
    if (topk_workspace_size(a.rows, a.E, a.k) > 0) {
        const int nchunks = (int)((a.E + kChunk - 1) / kChunk);
        const MultiWs w = multi_ws(a.ws, a.rows, a.E);
        topk_hist_kernel<<<dim3(nchunks, (unsigned)a.rows), 256, 0, s>>>(a.scores, a.E, a.ld,
                                                                         a.q_pos, a.m, a.k, w);
        topk_total_kernel<<<dim3(kBins / 256, (unsigned)a.rows), 256, 0, s>>>(nchunks, w);
        topk_collect_kernel<<<dim3(nchunks, (unsigned)a.rows), kCollectThreads, 0, s>>>(
            a.scores, a.E, a.ld, a.q_pos, a.m, a.k, w);
        cudaFuncSetAttribute(topk_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kResident * (int)sizeof(uint32_t));
        topk_final_kernel<<<(unsigned)a.rows, kThreads, kResident * sizeof(uint32_t), s>>>(
            a.q_pos, a.E, a.m, a.k, nchunks, w, a.idx);
        return cudaGetLastError();
    }
    if (a.k <= kMidMaxK) {
        cudaFuncSetAttribute(topk_mid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(MidShared));
        topk_mid_kernel<<<(unsigned)a.rows, kMidThreads, sizeof(MidShared), s>>>(
            a.scores, a.E, a.ld, a.q_pos, a.m, a.k, a.idx);
        return cudaGetLastError();
    }
    const int resident = a.E > a.k;
    const int64_t cap = a.E < kResident ? a.E : kResident;
    const size_t smem = resident ? (size_t)cap * sizeof(uint32_t) : 0;
    topk_kernel<<<(unsigned)a.rows, kThreads, smem, s>>>(a.scores, a.rows, a.E, a.ld, a.q_pos,
                                                         a.m, a.k, a.idx, resident, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_topk_flagged(const TopkArgs &a, const int *flag, cudaStream_t s)
{
    if (a.rows == 0)
        return cudaSuccess;
    // the rows are re-read from memory at every digit past the staged size
    const int64_t cap = a.E < kResident ? a.E : kResident;
    const size_t smem = (size_t)cap * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kResident * (int)sizeof(uint32_t));
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148, nsm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
        sms = nsm;
    const int64_t chunks = (a.rows + kThreads - 1) / kThreads;
    const int64_t grid = chunks < sms ? chunks : sms;
    topk_kernel<<<(unsigned)grid, kThreads, smem, s>>>(a.scores, a.rows, a.E, a.ld, a.q_pos, a.m,
                                                       a.k, a.idx, 1, flag);
    return cudaGetLastError();
}

// Lower bound of each row for the candidate mode: from the row's visible
// samples (scores of keys 0, S, 2S, .. below V, ns = floor(V / S) of them),
// the ks-th largest, ks = 1.25 mu + 4 sqrt(mu) + 8 where mu = k ns / V is
// the number of samples expected at or above the row's k-th largest score:
// the row's k-th largest lies below it only when the sample is off by many
// standard deviations (then the row is recomputed in full). -inf (keep every
// visible key) when there are too few samples; NaN (keep none) when the row
// has at most k visible keys. One warp per row: the top 16 bits of that
// sample's key are found bit by bit, each step counting the samples at or
// above the candidate; the bound is the float of those bits with the rest
// zero (never above the sample itself).
constexpr int kBoundRows = 8;

__global__ void __launch_bounds__(32 * kBoundRows)
topk_bound_kernel(const TopkBoundArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kBoundRows + (threadIdx.x >> 5);
    if (row >= a.rows)
        return;
    const int64_t V = visible(a.q_pos[row], a.m, a.E);
    float out = __int_as_float(0x7fc00000);
    if (V > a.k) {
        out = -INFINITY;
        const int64_t ns = V / a.S;
        const float mu = (float)a.k * (float)ns / (float)V;
        const float ksf = 1.25f * mu + 4.f * sqrtf(mu) + 8.f;
        if (ns <= 1024 && ksf <= (float)ns) {
            const unsigned ks = (unsigned)ksf;
            const float *srow = a.samp + row * a.samp_ld;
            uint32_t u[32];
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const int64_t j = lane + 32 * i;
                u[i] = j < ns ? float_key(__ldg(srow + j)) : 0u;
            }
            uint32_t T = 0u;
#pragma unroll 1
            for (int bit = 31; bit >= 16; bit--) {
                const uint32_t c = T | (1u << bit);
                unsigned n = 0;
#pragma unroll
                for (int i = 0; i < 32; i++)
                    n += u[i] >= c ? 1u : 0u;
                if (__reduce_add_sync(0xffffffffu, n) >= ks)
                    T = c;
            }
            // back to a float (the key of +0 and -0 gives +0)
            out = __uint_as_float((T & 0x80000000u) ? (T & 0x7fffffffu) : ~T);
        }
    }
    if (lane == 0)
        a.bound[row] = out;
}

cudaError_t launch_topk_bound(const TopkBoundArgs &a, cudaStream_t s)
{
    if (a.rows == 0)
        return cudaSuccess;
    topk_bound_kernel<<<(unsigned)((a.rows + kBoundRows - 1) / kBoundRows), 32 * kBoundRows, 0,
                        s>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
