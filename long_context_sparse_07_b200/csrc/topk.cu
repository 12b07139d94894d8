// topk.cu -- top-k selector (Eq. 17): radix select over the visible scores.
//
// Scores are mapped to order-preserving 32-bit keys (larger float -> larger
// key, -0 folded onto +0). Radix digits, most significant first, find the key
// T of the k-th largest element and how many elements equal to T must be
// taken (ties prefer lower indices). A final pass in index order writes every
// element with key > T and the first `need` elements with key == T, so each
// row comes out in ascending index order. Three layouts of the work:
//  * short rows (<= 2048 visible): one warp per row, keys in registers;
//  * rows up to 64 K: one block per row, keys staged once in shared memory
//    when they fit (re-read from L2 otherwise), 12 + 12 + 8-bit digits;
//  * longer rows (decode): chunks of the row over many blocks, then one block
//    per row over the candidates of the threshold bin.
#include "common.cuh"
#include "kernels.h"

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
topk_kernel(const float *__restrict__ scores, int64_t E, int64_t ld,
            const int64_t *__restrict__ q_pos, int m, int k, int32_t *__restrict__ idx,
            int resident)
{
    extern __shared__ uint32_t keys[];
    __shared__ Shared sh;
    const int64_t row = blockIdx.x;
    const int64_t V = visible(q_pos[row], m, E);
    int32_t *out = idx + row * k;
    if (V <= k) {
        for (int j = threadIdx.x; j < k; j += kThreads)
            out[j] = j < V ? j : -1;
        return;
    }
    RowScores src{scores + row * ld};
    block_select(src, V, k, out, keys, resident && V <= kResident, sh);
}

// ---------------------------------------------------------------------------
// Long rows (many entries, few rows: decode): the row is cut into chunks of
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

size_t topk_workspace_size(int64_t rows, int64_t E, int k)
{
    (void)k;
    if (E < kMultiMinE || rows > 65535 || rows <= 0 || (E + kChunk - 1) / kChunk > 1024)
        return 0;
    return multi_ws_bytes(rows, E);
}

cudaError_t launch_topk(const TopkArgs &a, unsigned *err, cudaStream_t s)
{
    (void)err;
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
    const int resident = a.E > a.k;
    const int64_t cap = a.E < kResident ? a.E : kResident;
    const size_t smem = resident ? (size_t)cap * sizeof(uint32_t) : 0;
    topk_kernel<<<(unsigned)a.rows, kThreads, smem, s>>>(a.scores, a.E, a.ld, a.q_pos, a.m,
                                                         a.k, a.idx, resident);
    return cudaGetLastError();
}

}  // namespace csa
