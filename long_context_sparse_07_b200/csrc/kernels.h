// kernels.h -- host-side launchers of the device kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

struct CompressArgs {
    const void *Ca, *Cb, *Za, *Zb;
    const float *Ba, *Bb;
    int64_t n;
    int c, m, overlap;
    csa_dtype in_dt;
    csa_entries out;
};
cudaError_t launch_compress(const CompressArgs &a, unsigned *err, cudaStream_t s);

struct IndexerArgs {
    const void *qI;
    const float *qI_scale, *wI;
    csa_entries kI;
    const int64_t *q_pos;
    int B;
    int64_t n_q, E;
    int hI, cI, m;
    csa_dtype dt;
    float *scores;
    int64_t ld;
};
cudaError_t launch_indexer(const IndexerArgs &a, unsigned *err, cudaStream_t s);

struct TopkArgs {
    const float *scores;
    int64_t rows, E, ld;
    const int64_t *q_pos;
    int m, k;
    int32_t *idx;
    void *ws;
};
cudaError_t launch_topk(const TopkArgs &a, unsigned *err, cudaStream_t s);
size_t topk_workspace_size(int64_t rows, int64_t E, int k);

// Options of the tensor-core indexer beyond the plain call.
struct IndexerTcExtra {
    int key_step = 1;                // key s of the table is row s * key_step of kI
    const int *row_flag = nullptr;   // score only rows whose flag is nonzero
    bool fuse = false;               // candidate mode (see indexer_tc.cu)
    const float *bound = nullptr;    // candidate mode: per-row lower bounds
    int k = 0;
    uint32_t *cnt = nullptr;         // [rows][nchunks][lists] pair counts
    bool plan_only = false;          // only report the key chunking
    int *nchunks_out = nullptr;
    int64_t *key_chunk_out = nullptr;
    int *lists_out = nullptr;
};
bool indexer_tc_takes(const IndexerArgs &a);
cudaError_t launch_indexer_tc_ex(const IndexerArgs &a, const IndexerTcExtra &x, unsigned *err,
                                 cudaStream_t s);

// Selection from the candidate pairs of the indexer's candidate mode: writes
// idx rows (or flags the row when its pairs do not decide the top-k).
struct TopkCandArgs {
    const uint2 *cand;               // (float bits of the score, index)
    int64_t cand_ld;
    const uint32_t *cnt;
    int nchunks, lists;
    int64_t key_chunk;
    const int64_t *q_pos;
    int m;
    int64_t E, rows;
    int k;
    int32_t *idx;
    int *flag;
};
cudaError_t launch_topk_cand(const TopkCandArgs &a, cudaStream_t s);
bool topk_cand_fits(int64_t E, int nchunks, int lists, int64_t rows);
// Per-row lower bound for the candidate mode from sample scores.
struct TopkBoundArgs {
    const float *samp;               // [rows, samp_ld]: scores of keys 0, S, 2S, ..
    int64_t samp_ld;
    const int64_t *q_pos;
    int m, S, k;
    int64_t E, rows;
    float *bound;
};
cudaError_t launch_topk_bound(const TopkBoundArgs &a, cudaStream_t s);
// Top-k of the flagged rows only (rows whose flag is zero are left alone).
cudaError_t launch_topk_flagged(const TopkArgs &a, const int *flag, cudaStream_t s);

// The indexer and the top-k in one call (csa_indexer_topk).
struct IndexerTopkArgs {
    IndexerArgs ix;
    int k;
    int32_t *idx;
    void *ws;
    size_t ws_bytes;
};
cudaError_t launch_indexer_topk(const IndexerTopkArgs &a, unsigned *err, cudaStream_t s);
int indexer_topk_launches(const IndexerArgs &ix, int k);
size_t indexer_topk_workspace_size(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                                   csa_dtype dt);


struct AttendArgs {
    const void *q;
    csa_dtype q_dt;
    csa_entries kv;
    int64_t E;
    const int32_t *idx;   // selection lists [B * n_q, k] (sparse only)
    int dense;            // 1: every visible entry is a key (HCA); 0: idx lists them
    int k, m;
    const void *kwin;
    int64_t win_rows;
    const int64_t *win_pos0;
    int n_win;
    const int64_t *q_pos;
    const float *sink;
    int B;
    int64_t n_q;
    int h;
    float scale;
    void *out;
    float *lse;
    void *ws;
    size_t ws_bytes;
};
cudaError_t launch_attend(const AttendArgs &a, unsigned *err, cudaStream_t s);

// Host-side checks of an attention call (everything but the workspace);
// CSA_OK or the status the call returns, with csa_last_message() set.
csa_status check_attend(const char *what, const void *q, csa_dtype q_dt, const csa_entries &kv,
                        int64_t E, const int32_t *idx, int k, int m, const void *kwin,
                        int64_t win_rows, int n_win, const int64_t *q_pos, const float *sink,
                        int B, int64_t n_q, int h, void *out);

struct NormRopeArgs {
    void *x;
    csa_dtype dt;
    const float *gamma;
    int64_t rows;
    int heads, c, rope_dims;
    const int64_t *pos;
    int64_t pos_mul, pos_add;
    int normalise;
    float eps, base;
};
cudaError_t launch_norm_rope(const NormRopeArgs &a, cudaStream_t s);

// C[M, N] (+ group offsets) = A[M, K] . B[N, K]^T, bf16, for `groups`
// independent groups: group j reads A columns j * a_col_off .., B rows
// j * b_row_off .., writes C columns j * c_col_off ..
struct GemmArgs {
    const void *A, *B;
    void *C;
    int64_t M;
    int N, K, groups;
    int64_t lda, b_rows, ldc;
    int64_t a_col_off, b_row_off, c_col_off;
};
cudaError_t launch_gemm_nt(const GemmArgs &g, unsigned *err, cudaStream_t s);

// One bounded wait that nothing completes (csa_debug_wait_probe).
cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned *err, cudaStream_t s);

// Sets the text that csa_last_message() returns on this thread.
void set_last_message(const char *msg);
size_t attend_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys);

}  // namespace csa
