/*
 * csa.h -- C ABI of the CSA / HCA hot path (B200, sm_100a).
 *
 * The method is DeepSeek-V4's Compressed Sparse Attention (CSA) and Heavily
 * Compressed Attention (HCA), as restated on the pages "DeepSeek-V4: Towards
 * Highly Efficient Million-Token Context Intelligence" (ai-papers-daily notes,
 * Modules B, C, D, F) and "DeepSeek V4 大模型算法解析" (section 二 核心算法).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers to dense, row-major, contiguous
 *    buffers that the caller owns and allocates. The library allocates no
 *    memory and keeps no state between calls except one device error word
 *    per GPU (see csa_get_error).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call only enqueues work on it and returns; results are
 *    ready when the stream reaches that point.
 *  - Positions: q_pos[b][t] is the absolute position of a query in its
 *    sequence (prefill: 0 .. n-1; decode: the context length minus one).
 *    The compressed entries visible to a query at position t are
 *    V_t = min(E, floor((t + 1) / m)): entry i covers tokens m*i .. m*i+m-1
 *    and is visible once its last token is at or before t.
 *  - Validation: each call checks its arguments on the host (null pointers,
 *    sizes, 16-byte alignment of every vector-loaded buffer, supported
 *    dtype/shape combinations) before launching anything. On failure it
 *    returns CSA_ERR_INVALID_ARG or CSA_ERR_UNSUPPORTED, launches nothing and
 *    writes nothing; csa_last_message() then describes the failure.
 *  - Device-side checks (a selection index outside [0, V_t), a window
 *    position outside the window buffer) never trap: the offending key is
 *    skipped and the device error word records CSA_ERR_BOUNDS, which
 *    csa_get_error reports.
 *  - A launch failure returns CSA_ERR_CUDA.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_F32 = 0,   /* IEEE binary32 */
    CSA_BF16 = 1,  /* bfloat16 */
    CSA_E4M3 = 2,  /* 8-bit float e4m3 (finite, max 448), always with scales */
    CSA_E2M1 = 3   /* 4-bit float e2m1 (max 6), two per byte, with block scales
                      (indexer keys only) */
} csa_dtype;

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = -1,
    CSA_ERR_UNSUPPORTED = -2,
    CSA_ERR_CUDA = -3,
    CSA_ERR_TIMEOUT = -4,
    CSA_ERR_BOUNDS = -5
} csa_status;

/*
 * A table of KV entries of width c, `rows` rows (compressed entries, or
 * indexer keys of width c_I).
 *   plain layout: dt = CSA_F32 or CSA_BF16, rope_dims = 0, scale = rope =
 *     NULL; body is [rows, c].
 *   fp8 layout (low-precision KV storage, Module F): dt = CSA_E4M3;
 *     body is [rows, c - rope_dims] e4m3 codes; scale is
 *     [rows, (c - rope_dims) / scale_group] float32 (> 0); the value of
 *     body[r][j] is code * scale[r][j / scale_group]; when rope_dims > 0 the
 *     trailing rope_dims channels are stored unscaled as bfloat16 in rope
 *     [rows, rope_dims].
 *   fp4 layout (indexer keys: Module F, "the indexer's QK path runs in FP4"):
 *     dt = CSA_E2M1, scale_group = 32, rope_dims = 0, rope = NULL, c a
 *     multiple of 32; body is [rows, c / 2] bytes, channel j in the low
 *     nibble of byte j / 2 when j is even, in the high nibble when odd; the
 *     `scale` pointer holds [rows, c / 32] uint8 block exponents (not
 *     floats): the value of channel j is e2m1(code) * 2^(e[r][j / 32] - 127).
 *     Within a row the exponents span at most 8 (max - min <= 8), which the
 *     compressor guarantees; larger spans read wrong values.
 * The same struct describes inputs (read) and outputs (written); `body`,
 * `scale` and `rope` are cast to const by readers.
 */
typedef struct {
    void *body;
    float *scale;
    void *rope;
    int c;
    int rope_dims;
    int scale_group;
    csa_dtype dt;
} csa_entries;

/* ABI version: bumped on any incompatible change of this header. */
int csa_abi_version(void);

/* Human-readable text of a status code (static storage). */
const char *csa_status_string(csa_status s);

/* Text of the last host-side validation failure of this thread (static,
 * thread-local storage; empty when none). */
const char *csa_last_message(void);

/*
 * csa_compress_kv -- token-level compressor.
 *   CSA (overlap = 1), Eq. 9-12 (Module B step 1; the overlapping windows of
 *   "第一阶段"): entry i, channel j pools rows m*i .. m*i+m-1 of Ca and rows
 *   m*(i-1) .. m*i-1 of Cb with the softmax (over those 2m token positions,
 *   per channel) of the logits Za + Ba and Zb + Bb. Entry 0 has no previous
 *   block: its Cb half is left out of the softmax.
 *   HCA (overlap = 0), Eq. 20-23 (Module C): m = m' rows of Ca with logits
 *   Za + Ba; Cb, Zb and Bb must be NULL.
 * Arguments:
 *   Ca, Cb, Za, Zb  [n, c] of in_dt (F32 or BF16), rows = tokens.
 *   Ba, Bb          [m, c] float32 position biases.
 *   n               tokens; n % m == 0 (an incomplete tail block is not an
 *                   entry); E = n / m entries are written.
 *   out             [E, c] entries: plain F32/BF16, or the fp8 layout with
 *                   scale_group dividing c - rope_dims (per-group scale =
 *                   max(amax / 448, 2^-126), codes rounded to nearest even
 *                   and saturated; rope channels stored as bf16), or the fp4
 *                   layout (indexer keys; c / 32 blocks per row, 32 / vector
 *                   width lanes each: each block takes the smallest scale
 *                   2^E with 6 * 2^E >= its largest magnitude, raised to the
 *                   row's largest E - 8 when below it; an all-zero row takes
 *                   E = 0; codes rounded to nearest even).
 * Requirements: c / 8 (bf16) or c / 4 (f32) a power of two of at most 256,
 *   1 <= m <= 1024,
 *   all buffers 16-byte aligned.
 */
csa_status csa_compress_kv(const void *Ca, const void *Cb, const void *Za, const void *Zb,
                           const float *Ba, const float *Bb, int64_t n, int c, int m,
                           int overlap, csa_dtype in_dt, csa_entries out, void *stream);

/*
 * csa_indexer_scores -- lightning-indexer scores, Eq. 16 (Module B step 2):
 *   I[b][t][s] = sum_h wI[b][t][h] * ReLU(qI[b][t][h] . kI[b][s])
 * for every visible entry s < V_t. There is no softmax and no scale factor.
 * Entries s >= V_t of a score row are NOT written (the selection never
 * reads them).
 * Arguments:
 *   qI        [B, n_q, hI, cI] of dt; dt = CSA_E4M3 requires qI_scale
 *             [B, n_q, hI] float32 > 0 (one scale per query head), else NULL.
 *   wI        [B, n_q, hI] float32 head weights.
 *   kI        keys, rows = B * E (batch b owns rows b*E .. b*E+E-1), c = cI;
 *             kI.dt must equal dt, or be CSA_E2M1 (FP4 keys) with dt =
 *             CSA_E4M3 (FP4 keys against e4m3 queries: the products are
 *             exact in the 8-bit tensor-core path, FP4 saving half of the
 *             key bytes); for CSA_E4M3, scale_group == cI (one
 *             positive scale per key) and rope_dims == 0.
 *   q_pos     [B, n_q] int64 query positions.
 *   m         compression ratio used for visibility.
 *   scores    [B, n_q, ld] float32, ld >= E.
 * Requirements: cI % 16 == 0, cI <= 256, 1 <= hI <= 128.
 */
csa_status csa_indexer_scores(const void *qI, const float *qI_scale, const float *wI,
                              csa_entries kI, const int64_t *q_pos, int B, int64_t n_q,
                              int64_t E, int hI, int cI, int m, csa_dtype dt, float *scores,
                              int64_t ld, void *stream);

/*
 * csa_topk -- top-k selector, Eq. 17 (Module B step 2):
 * for each row r, the min(k, V_r) visible entries (s < V_r, V_r from
 * q_pos[r] and m) with the largest scores. Equal scores prefer the lower
 * index (+0 and -0 are equal). The row of idx lists the chosen indices in
 * ascending order, then -1 up to k. Scores must not be NaN.
 * Arguments:
 *   scores    [rows, ld] float32 (only s < V_r is read).
 *   q_pos     [rows] int64.
 *   idx       [rows, k] int32 output.
 *   workspace, ws_bytes   device scratch of at least
 *             csa_topk_workspace_size(rows, E, k) bytes, 256-byte aligned
 *             (may be NULL when that size is 0; it is nonzero for rows of
 *             more than 262144 entries, which are split over many blocks
 *             in four launches; rows of 65536 .. 262144 entries take one
 *             launch, a cluster of 8 blocks per row, and no workspace).
 *             The caller owns it; nothing in it must be initialised.
 * Requirements: 1 <= k <= 4096.
 */
csa_status csa_topk(const float *scores, int64_t rows, int64_t E, int64_t ld,
                    const int64_t *q_pos, int m, int k, int32_t *idx, void *workspace,
                    size_t ws_bytes, void *stream);
size_t csa_topk_workspace_size(int64_t rows, int64_t E, int k);

/*
 * csa_indexer_topk -- the indexer scores (Eq. 16) and the top-k selection
 * (Eq. 17) of Module B step 2 in one call: idx gets exactly what
 * csa_indexer_scores followed by csa_topk would write (the same entries, in
 * ascending order, ties to the lower index, -1 padding), but the full score
 * rows are not written when the rows are much longer than k. For e4m3 or
 * bf16 indexers that the tensor-core kernel takes (hI in {16, 32, 64}, cI
 * bytes 128 or 256), E >= 16 k, E a multiple of the sample spacing (32,
 * doubled until a row has at most 1024 samples) and enough queries that
 * every indexer block owns whole rows (prefill), the call
 *   1. scores every query against that sample of the keys,
 *   2. runs the indexer keeping, per query, only the scores at or above a
 *      lower bound taken from its sample scores (a rank of the sample that
 *      the k-th largest score of the row exceeds with a wide margin),
 *   3. selects the top-k exactly from those candidates,
 *   4. recomputes in full the rows whose candidates cannot decide it (fewer
 *      than k, or more than the workspace holds): rare for scores that are
 *      not massively tied; correct in every case.
 * Other calls (decode among them: a few rows, cheap to write and read back)
 * run the two plain calls through the workspace.
 * Arguments: as csa_indexer_scores (without scores / ld), plus
 *   k         1 <= k <= 4096.
 *   idx       [B * n_q, k] int32 output.
 *   workspace csa_indexer_topk_workspace_size(B, n_q, E, hI, cI, k, dt)
 *             bytes of device scratch, 256-byte aligned, owned by the caller;
 *             nothing in it must be initialised. It holds a [B * n_q, E]
 *             float32 area (score rows or candidate pairs) and small tables.
 */
csa_status csa_indexer_topk(const void *qI, const float *qI_scale, const float *wI,
                            csa_entries kI, const int64_t *q_pos, int B, int64_t n_q, int64_t E,
                            int hI, int cI, int m, csa_dtype dt, int k, int32_t *idx,
                            void *workspace, size_t ws_bytes, void *stream);
size_t csa_indexer_topk_workspace_size(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                                       csa_dtype dt);
/* Kernel launches csa_indexer_topk makes for these shapes (6 on the
 * candidate path, 2 to 5 for the two plain calls) on the current device,
 * for 16-byte aligned qI and kI; -1 for arguments out of range. */
int csa_indexer_topk_launches(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                              csa_dtype dt);

/*
 * csa_sparse_mqa -- shared-KV multi-query attention over the selected
 * compressed entries, Eq. 18-19 (Module B step 3), joined by the sliding-window
 * branch and the attention sink (Module D). Every key is also its own value.
 * For query (b, t) and head i the key set is
 *   { kv[b][idx[b*n_q+t][j]] : idx >= 0 }  (entries, each must be < V_t)
 *   U { kwin[b][p - win_pos0[b]] : max(0, t - n_win + 1) <= p <= t }
 * and, with z_j = scale * q . key_j, M = max(max_j z_j, sink[i]),
 *   out = sum_j e^{z_j - M} key_j / (sum_j e^{z_j - M} + e^{sink[i] - M})
 *   lse = M + log(sum_j e^{z_j - M} + e^{sink[i] - M}).
 * Arguments:
 *   q         [B, n_q, h, c] of q_dt (F32 or BF16); out has the same shape
 *             and dtype.
 *   kv        entries, rows = B * E (batch b owns rows b*E ..), width c;
 *             plain (dt == q_dt) or the fp8 layout (bf16 queries only).
 *   E, m      entries per batch and the compression ratio that fixes
 *             V_t = min(E, floor((t + 1) / m)); a listed index outside
 *             [0, V_t) is skipped and recorded as CSA_ERR_BOUNDS.
 *   idx       [B * n_q, k] int32 (ascending or not; -1 = empty slot).
 *   kwin      [B, win_rows, c] of q_dt: raw KV rows; row r of batch b holds
 *             position win_pos0[b] + r (win_pos0 NULL means 0).
 *   sink      [h] float32 per-head sink logits (-inf disables the sink).
 *   lse       [B, n_q, h] float32 or NULL.
 *   workspace csa_mqa_workspace_size(...) bytes of device scratch, or NULL
 *             when that size is 0.
 * Requirements: c a power of two from 64 to 1024, 1 <= h <= 128,
 *   0 <= k <= 4096, n_win >= 0; q, out, kwin and entry buffers 16-byte
 *   aligned.
 */
csa_status csa_sparse_mqa(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                          const int32_t *idx, int k, const void *kwin, int64_t win_rows,
                          const int64_t *win_pos0, int n_win, const int64_t *q_pos,
                          const float *sink, int B, int64_t n_q, int h, float scale,
                          void *out, float *lse, void *workspace, size_t ws_bytes,
                          void *stream);

/*
 * hca_dense_mqa -- HCA core attention, Eq. 24-26 (Module C): as
 * csa_sparse_mqa, but every visible entry s < V_t (V_t from m = m') is a key
 * instead of a selection.
 */
csa_status hca_dense_mqa(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                         const void *kwin, int64_t win_rows, const int64_t *win_pos0,
                         int n_win, const int64_t *q_pos, const float *sink, int B,
                         int64_t n_q, int h, float scale, void *out, float *lse,
                         void *workspace, size_t ws_bytes, void *stream);

/* Device scratch bytes that csa_sparse_mqa / hca_dense_mqa need for this
 * shape (split-KV partial results for small query counts); 0 when none. */
size_t csa_mqa_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys);

/*
 * csa_sparse_mqa_noalloc -- csa_sparse_mqa without a workspace argument, for
 * callers that cannot allocate device memory on their hot path (code hosted
 * by a framework that owns all device memory through pre-reserved pools, or
 * a decode loop that cannot afford the device-wide synchronisation an
 * allocation may cause). The method on the reference pages has no
 * counterpart of this call: it only changes where the scratch lives.
 *   Scratch (the split-key partial results) comes from one file-scope device
 *   array of csa_noalloc_scratch_bytes() bytes (32 MiB) that every GPU loading
 *   the library holds until the process exits. The call allocates nothing.
 *   Every other argument, the results and the error behaviour are those of
 *   csa_sparse_mqa. A shape whose scratch (csa_mqa_workspace_size) exceeds the
 *   array returns CSA_ERR_UNSUPPORTED, launches nothing and says so in
 *   csa_last_message().
 *   The first call on a device looks up the array's device address (with
 *   that device current); make it before capturing the stream into a graph.
 *   The address is kept for the life of the process and does not survive a
 *   device reset (cudaDeviceReset): do not call this entry point on a device
 *   after resetting it in the same process.
 *   The 32 MiB cover a decode step of 8 queries, 64 heads of width 512, 1024
 *   selected entries and a 128-row window.
 *   All calls share the one array and each call overwrites the part it uses
 *   before reading it, so nothing needs clearing; but calls that may overlap
 *   on the GPU (different streams, or different host threads on one device)
 *   race on it and must be serialised by the caller.
 */
csa_status csa_sparse_mqa_noalloc(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                                  const int32_t *idx, int k, const void *kwin, int64_t win_rows,
                                  const int64_t *win_pos0, int n_win, const int64_t *q_pos,
                                  const float *sink, int B, int64_t n_q, int h, float scale,
                                  void *out, float *lse, void *stream);
size_t csa_noalloc_scratch_bytes(void);

/*
 * csa_norm_rope -- Q/KV RMSNorm and partial RoPE before the core attention,
 * and the rotation of its output back by the query position (Module D: "Q/KV
 * normalisation", "partial RoPE": RoPE only on the last 64 dims of queries
 * and KV entries; since an entry is key and value, the output o_t then
 * carries the entries' absolute positions, and turning its last 64 dims by
 * the position -t leaves relative positions). In place on x, [rows, heads, c]
 * of dt (F32 or BF16), per head vector:
 *   when normalise: x <- x / sqrt(mean_j x_j^2 + eps) * gamma[j]
 *                   (gamma [c] float32, or NULL for a gain of 1);
 *   then the last rope_dims dims turn in adjacent pairs (c - R + 2p,
 *   c - R + 2p + 1), p < R / 2, by phi_p = P * base^(-2p / R):
 *   (a, b) <- (a cos phi - b sin phi, a sin phi + b cos phi), with the
 *   position P = pos_mul * (pos ? pos[row] : row) + pos_add (pos [rows]
 *   int64 or NULL). Queries: pos = q_pos, pos_mul = 1; compressed entry i:
 *   pos = NULL, pos_mul = m, pos_add = m - 1 (the position of its last
 *   token); window rows: pos = NULL, pos_mul = 1, pos_add = the position of
 *   row 0; the attention output: pos = q_pos, pos_mul = -1, normalise = 0.
 *   The method's pages fix neither the pairing, the base, the entry
 *   positions nor eps; these are this library's readings.
 * Requirements: c in {64, 128, 256, 512, 1024}; rope_dims even, <= c;
 *   eps > 0 when normalising; base > 1 when rope_dims > 0; x 16-byte aligned.
 */
csa_status csa_norm_rope(void *x, csa_dtype dt, const float *gamma, int64_t rows, int heads, int c,
                         int rope_dims, const int64_t *pos, int64_t pos_mul, int64_t pos_add,
                         int normalise, float eps, float base, void *stream);

/*
 * csa_grouped_out_proj -- grouped output projection (Module B step 4: the
 * n_h head outputs are cut into g groups, each group is projected to an
 * intermediate d_g, and the concatenation is projected to d), bf16 operands
 * with float32 accumulation:
 *   u[t, j d_g + e] = sum_x o[t, j K_g + x] * Wg[j d_g + e, x]   (j < g,
 *                     K_g = h c / g; group j holds heads j h/g .. (j+1) h/g - 1)
 *   out[t, f]       = sum_y u[t, y] * Wo[f, y]
 * Arguments (all bf16, row-major, 16-byte aligned, owned by the caller):
 *   o   [n, h, c]      attention outputs;
 *   Wg  [g * dg, K_g]  the g group weights, output features by input features;
 *   Wo  [d, g * dg]    the final weight;
 *   u   [n, g * dg]    written: the grouped projections, stored as bf16;
 *   out [n, d]         written.
 * Requirements: g divides h; K_g a multiple of 64; dg and d multiples of
 *   256. The pages fix g = 8, d_g = 1024 (Flash) but no weight layout or
 *   intermediate precision; the layout above and bf16 u are this library's.
 */
csa_status csa_grouped_out_proj(const void *o, const void *Wg, const void *Wo, int64_t n, int h,
                                int c, int g, int dg, int d, void *u, void *out, void *stream);

/*
 * csa_debug_wait_probe -- checks the device-side failure path. Launches one
 * thread that waits, through the same bounded mbarrier wait every pipeline
 * kernel uses, on a barrier that nothing completes; after limit_ns
 * nanoseconds (1e3 .. 1e9) the wait gives up and the device error word
 * records CSA_ERR_TIMEOUT, which the next csa_get_error returns (and clears).
 * Nothing is left in flight and the device stays usable. The method has no
 * counterpart of this call: it exists so that tests can make a device wait
 * expire without faulting or hanging the GPU.
 */
csa_status csa_debug_wait_probe(uint64_t limit_ns, void *stream);

/*
 * csa_get_error -- synchronises the current device, reads and clears its
 * device error word, and returns the status it held (CSA_OK if none). When
 * buf is not NULL, a description (at most len bytes, NUL-terminated) is
 * written to it. Call it after a batch of work to confirm that no device-side
 * check fired.
 */
csa_status csa_get_error(char *buf, size_t len);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H */
