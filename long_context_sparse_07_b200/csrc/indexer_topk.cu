// indexer_topk.cu -- the lightning-indexer scores (Eq. 16) and the top-k
// selection (Eq. 17) in one call, without writing the score rows.
//
// For rows much longer than k the selection keeps a small fraction of every
// row, so the full score rows (4 bytes per visible pair, written by the
// indexer and read back by the top-k) are most of the traffic between the
// two steps. Here:
//  1. the indexer scores a sample of the keys (every S-th key, S a power of
//     two with at most 1024 samples per row) for every query;
//  2. a lower bound L per row from its sample scores: a rank of the sample
//     that the row's k-th largest score exceeds with a wide margin;
//  3. the indexer runs over all keys in candidate mode: its epilogue writes
//     only the (score, index) pairs of scores at or above L, each warp into
//     its own list per token;
//  4. an exact radix select over each row's pairs writes the k indices in
//     ascending order;
//  5. rows whose pairs cannot decide the top-k (fewer than k of them, or
//     more than their room) are flagged by step 4 and recomputed in full:
//     the indexer scores only the flagged rows (blocks without one exit at
//     once) and the block top-k selects over them.
// The result is the top-k of the full score rows in every case. Shapes the
// tensor-core indexer does not take, rows not much longer than k, and calls
// with too few token blocks to give each block whole rows (decode: a few
// queries, whose score rows cost little to write and read back) run the two
// plain calls through the same workspace.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

size_t a256(size_t b) { return (b + 255) / 256 * 256; }

// Sample spacing: a power of two >= 32 with at most 1024 samples per row.
int sample_step(int64_t E)
{
    int64_t S = 32;
    while ((E + S - 1) / S > 1024)
        S *= 2;
    return (int)S;
}

// Candidate lists per row: one per epilogue warp that reduces the row's
// token (4, or 8 with two warp sets).
constexpr int kMaxLists = 8;

struct Layout {
    size_t region, samp, bound, cnt, flag, topk, total;
};

Layout layout(int B, int64_t n_q, int64_t E, int k)
{
    const int64_t rows = (int64_t)B * n_q;
    const int S = sample_step(E);
    Layout l;
    l.region = 0;
    l.samp = l.region + a256((size_t)rows * E * 4);
    l.bound = l.samp + a256((size_t)rows * (E / S > 0 ? E / S : 1) * 4);
    l.cnt = l.bound + a256((size_t)rows * 4);
    l.flag = l.cnt + a256((size_t)rows * kMaxLists * 4);
    l.topk = l.flag + a256((size_t)rows * 4);
    l.total = l.topk + a256(topk_workspace_size(rows, E, k));
    return l;
}

}  // namespace

size_t indexer_topk_workspace_size(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                                   csa_dtype dt)
{
    (void)hI;
    (void)cI;
    (void)dt;
    if ((int64_t)B * n_q <= 0 || E <= 0)
        return 0;
    return layout(B, n_q, E, k).total;
}

namespace {

// Whether the call takes the candidate path, with its key chunking.
bool fused_plan(const IndexerArgs &full, int k, int *nchunks, int *lists, int64_t *key_chunk,
                unsigned *err, cudaStream_t s)
{
    const int64_t E = full.E;
    const int S = sample_step(E);
    *nchunks = 1;
    *lists = 1;
    *key_chunk = E;
    if (!(E > 0 && E >= 16 * (int64_t)k && E % S == 0 && indexer_tc_takes(full)))
        return false;
    IndexerTcExtra plan;
    plan.fuse = true;
    plan.plan_only = true;
    plan.nchunks_out = nchunks;
    plan.key_chunk_out = key_chunk;
    plan.lists_out = lists;
    if (launch_indexer_tc_ex(full, plan, err, s) != cudaSuccess)
        return false;
    // candidate mode needs whole rows in one block (many token blocks, as
    // in prefill); with few queries the score rows are small and the two
    // plain calls are faster
    const int64_t rows = (int64_t)full.B * full.n_q;
    return *nchunks == 1 && *lists <= kMaxLists && topk_cand_fits(E, *nchunks, *lists, rows);
}

}  // namespace

int indexer_topk_launches(const IndexerArgs &ix, int k)
{
    const int64_t rows = (int64_t)ix.B * ix.n_q;
    if (rows == 0)
        return 0;
    int nchunks, lists;
    int64_t key_chunk;
    if (fused_plan(ix, k, &nchunks, &lists, &key_chunk, nullptr, 0))
        return 6;
    return (ix.E > 0 ? 1 : 0) + (topk_workspace_size(rows, ix.E, k) > 0 ? 4 : 1);
}

cudaError_t launch_indexer_topk(const IndexerTopkArgs &a, unsigned *err, cudaStream_t s)
{
    const IndexerArgs &ix = a.ix;
    const int64_t rows = (int64_t)ix.B * ix.n_q;
    if (rows == 0)
        return cudaSuccess;
    const int64_t E = ix.E;
    const Layout l = layout(ix.B, ix.n_q, E, a.k);
    char *ws = (char *)a.ws;
    float *region = (float *)(ws + l.region);
    float *samp = (float *)(ws + l.samp);
    float *bound = (float *)(ws + l.bound);
    uint32_t *cnt = (uint32_t *)(ws + l.cnt);
    int *flag = (int *)(ws + l.flag);
    void *tws = l.total > l.topk ? (void *)(ws + l.topk) : nullptr;

    IndexerArgs full = ix;
    full.scores = region;
    full.ld = E;
    const TopkArgs tk{region, rows, E, E, ix.q_pos, ix.m, a.k, a.idx, tws};

    const int S = sample_step(E);
    int nchunks = 1, lists = 1;
    int64_t key_chunk = E;
    const bool fused = fused_plan(full, a.k, &nchunks, &lists, &key_chunk, err, s);
    if (!fused) {
        if (E > 0) {
            cudaError_t e = launch_indexer(full, err, s);
            if (e != cudaSuccess)
                return e;
        }
        return launch_topk(tk, err, s);
    }
    // 1. sample scores: keys 0, S, 2S, .. as a table of E / S keys whose
    // visibility bound is m * S
    IndexerArgs smp = ix;
    smp.E = E / S;
    smp.m = ix.m * S;
    smp.scores = samp;
    smp.ld = E / S;
    IndexerTcExtra xs;
    xs.key_step = S;
    cudaError_t e = launch_indexer_tc_ex(smp, xs, err, s);
    if (e != cudaSuccess)
        return e;
    // 2. lower bounds
    const TopkBoundArgs tb{samp, E / S, ix.q_pos, ix.m, S, a.k, E, rows, bound};
    e = launch_topk_bound(tb, s);
    if (e != cudaSuccess)
        return e;
    // 3. candidate pairs
    IndexerTcExtra xc;
    xc.fuse = true;
    xc.bound = bound;
    xc.k = a.k;
    xc.cnt = cnt;
    e = launch_indexer_tc_ex(full, xc, err, s);
    if (e != cudaSuccess)
        return e;
    // 4. exact selection from the pairs
    const TopkCandArgs tc{(const uint2 *)region, E / 2, cnt, nchunks, lists, key_chunk,
                          ix.q_pos, ix.m, E, rows, a.k, a.idx, flag};
    e = launch_topk_cand(tc, s);
    if (e != cudaSuccess)
        return e;
    // 5. the flagged rows in full
    IndexerTcExtra xf;
    xf.row_flag = flag;
    e = launch_indexer_tc_ex(full, xf, err, s);
    if (e != cudaSuccess)
        return e;
    return launch_topk_flagged(tk, flag, s);
}

}  // namespace csa
