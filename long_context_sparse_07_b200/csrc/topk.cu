// topk.cu -- top-k selector (Eq. 17): radix select over the visible scores.
//
// One block per score row. Scores are mapped to order-preserving 32-bit keys
// (larger float -> larger key, -0 folded onto +0). Four 8-bit digit passes,
// most significant first, find the key T of the k-th largest element and how
// many elements equal to T must be taken (ties prefer lower indices). A final
// pass in index order writes every element with key > T and the first
// `need` elements with key == T, so each row comes out in ascending index
// order. When the visible row fits, its keys are staged once in shared
// memory and every pass reads them from there; longer rows are re-read from
// global memory (L2) on each pass.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kResident = 40960;   // keys staged in shared memory (160 KB)

struct Shared {
    unsigned hist[256];
    unsigned warp_tot[kWarps];
    unsigned bin, need;
};

// Exclusive block-wide prefix count of a per-thread flag; returns the
// thread's rank and writes the block total to *total.
__device__ __forceinline__ unsigned block_rank(bool flag, Shared &sh, unsigned *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned ballot = __ballot_sync(0xffffffffu, flag);
    const unsigned in_warp = __popc(ballot & ((1u << lane) - 1u));
    __syncthreads();                       // warp_tot free for reuse
    if (lane == 0)
        sh.warp_tot[warp] = __popc(ballot);
    __syncthreads();
    unsigned before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
        const unsigned v = sh.warp_tot[w];
        before += (w < warp) ? v : 0u;
        tot += v;
    }
    *total = tot;
    return before + in_warp;
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
    const float *src = scores + row * ld;

    if (V <= k) {
        for (int j = threadIdx.x; j < k; j += kThreads)
            out[j] = j < V ? j : -1;
        return;
    }
    const bool res = resident && V <= kResident;
    if (res) {
        for (int64_t s = threadIdx.x; s < V; s += kThreads)
            keys[s] = float_key(src[s]);
        __syncthreads();
    }

    uint32_t prefix = 0, pmask = 0;
    unsigned need = (unsigned)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += kThreads)
            sh.hist[b] = 0;
        if (threadIdx.x == 0) {
            sh.bin = 0;
            sh.need = need;
        }
        __syncthreads();
        for (int64_t s = threadIdx.x; s < V; s += kThreads) {
            const uint32_t u = res ? keys[s] : float_key(src[s]);
            if ((u & pmask) == prefix)
                atomicAdd(&sh.hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins 255-8l .. 248-8l (descending); find the bin
            // where the count from the top reaches `need`.
            const int lane = threadIdx.x;
            unsigned local = 0;
#pragma unroll
            for (int j = 0; j < 8; j++)
                local += sh.hist[255 - 8 * lane - j];
            unsigned incl = local;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off)
                    incl += v;
            }
            const unsigned excl = incl - local;
            if (excl < need && need <= incl) {
                unsigned cum = excl;
                for (int j = 0; j < 8; j++) {
                    const int b = 255 - 8 * lane - j;
                    const unsigned hb = sh.hist[b];
                    if (cum + hb >= need) {
                        sh.bin = (unsigned)b;
                        sh.need = need - cum;
                        break;
                    }
                    cum += hb;
                }
            }
        }
        __syncthreads();
        prefix |= sh.bin << shift;
        pmask |= 255u << shift;
        need = sh.need;
        __syncthreads();
    }

    // compaction in index order
    const uint32_t T = prefix;
    unsigned base = 0, eq_seen = 0;
    for (int64_t c0 = 0; c0 < V; c0 += kThreads) {
        const int64_t s = c0 + threadIdx.x;
        uint32_t u = 0;
        if (s < V)
            u = res ? keys[s] : float_key(src[s]);
        const bool gt = s < V && u > T;
        const bool eq = s < V && u == T;
        unsigned eq_tot, take_tot;
        const unsigned eq_rank = block_rank(eq, sh, &eq_tot);
        const bool take = gt || (eq && eq_seen + eq_rank < need);
        const unsigned pos = block_rank(take, sh, &take_tot);
        if (take && base + pos < (unsigned)k)
            out[base + pos] = (int32_t)s;
        base += take_tot;
        eq_seen += eq_tot;
    }
    for (int j = (int)base + threadIdx.x; j < k; j += kThreads)
        out[j] = -1;
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
    const int resident = a.E > a.k;
    const int64_t cap = a.E < kResident ? a.E : kResident;
    const size_t smem = resident ? (size_t)cap * sizeof(uint32_t) : 0;
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kResident * (int)sizeof(uint32_t));
    topk_kernel<<<(unsigned)a.rows, kThreads, smem, s>>>(a.scores, a.E, a.ld, a.q_pos, a.m,
                                                         a.k, a.idx, resident);
    return cudaGetLastError();
}

}  // namespace csa
