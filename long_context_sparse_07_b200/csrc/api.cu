// api.cu -- the C ABI of csa.h: argument validation, device error word and
// dispatch to the kernel launchers. No call allocates device memory.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace {

__device__ unsigned g_err[4];

thread_local char g_msg[512];

csa_status fail(csa_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

constexpr int kMaxDevices = 64;
unsigned *g_err_ptr[kMaxDevices];

// Device address of this GPU's error word (looked up once per device).
unsigned *err_word()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_err) != cudaSuccess)
            return nullptr;
        g_err_ptr[dev] = (unsigned *)p;
    }
    return g_err_ptr[dev];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

csa_status launched(cudaError_t e, const char *what)
{
    if (e != cudaSuccess)
        return fail(CSA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    g_msg[0] = 0;
    return CSA_OK;
}

#define REQUIRE(cond, st, ...)                                                           \
    do {                                                                                 \
        if (!(cond))                                                                     \
            return fail(st, __VA_ARGS__);                                                \
    } while (0)

csa_status check_entries(const csa_entries &t, int c, bool allow_fp8, const char *what,
                         bool allow_fp4 = false)
{
    REQUIRE(t.body, CSA_ERR_INVALID_ARG, "%s: body is NULL", what);
    REQUIRE(t.c == c, CSA_ERR_INVALID_ARG, "%s: c = %d, expected %d", what, t.c, c);
    REQUIRE(aligned16(t.body), CSA_ERR_INVALID_ARG, "%s: body not 16-byte aligned", what);
    if (t.dt == CSA_E2M1) {
        REQUIRE(allow_fp4, CSA_ERR_UNSUPPORTED, "%s: e2m1 entries are for indexer keys only",
                what);
        REQUIRE(c % 32 == 0, CSA_ERR_UNSUPPORTED, "%s: e2m1 entries need c %% 32 == 0", what);
        REQUIRE(t.scale && ((uintptr_t)t.scale & 3u) == 0, CSA_ERR_INVALID_ARG,
                "%s: e2m1 entries need 4-byte aligned block exponents in `scale`", what);
        REQUIRE(t.scale_group == 32 && t.rope_dims == 0 && !t.rope, CSA_ERR_INVALID_ARG,
                "%s: e2m1 entries need scale_group 32 and no rope part", what);
        return CSA_OK;
    }
    if (t.dt == CSA_E4M3) {
        REQUIRE(allow_fp8, CSA_ERR_UNSUPPORTED, "%s: e4m3 entries not supported here", what);
        REQUIRE(t.scale && aligned16(t.scale), CSA_ERR_INVALID_ARG,
                "%s: e4m3 entries need 16-byte aligned scales", what);
        REQUIRE(t.rope_dims >= 0 && t.rope_dims < c, CSA_ERR_INVALID_ARG,
                "%s: rope_dims = %d out of range", what, t.rope_dims);
        REQUIRE((t.rope_dims > 0) == (t.rope != nullptr), CSA_ERR_INVALID_ARG,
                "%s: rope pointer must be given exactly when rope_dims > 0", what);
        REQUIRE(!t.rope || aligned16(t.rope), CSA_ERR_INVALID_ARG,
                "%s: rope not 16-byte aligned", what);
        REQUIRE(t.scale_group > 0 && (c - t.rope_dims) % t.scale_group == 0,
                CSA_ERR_INVALID_ARG, "%s: scale_group %d must divide c - rope_dims = %d", what,
                t.scale_group, c - t.rope_dims);
        REQUIRE((c - t.rope_dims) % 16 == 0 && t.rope_dims % 8 == 0, CSA_ERR_UNSUPPORTED,
                "%s: c - rope_dims must be a multiple of 16 and rope_dims of 8", what);
    } else {
        REQUIRE(t.dt == CSA_F32 || t.dt == CSA_BF16, CSA_ERR_INVALID_ARG,
                "%s: unknown dtype %d", what, (int)t.dt);
        REQUIRE(t.rope_dims == 0, CSA_ERR_INVALID_ARG,
                "%s: rope_dims must be 0 for plain entries", what);
    }
    return CSA_OK;
}

}  // namespace

namespace csa {
void set_last_message(const char *msg) { snprintf(g_msg, sizeof g_msg, "%s", msg); }
}  // namespace csa

extern "C" {

int csa_abi_version(void) { return 1; }

const char *csa_status_string(csa_status s)
{
    switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case CSA_ERR_CUDA: return "CUDA error";
    case CSA_ERR_TIMEOUT: return "device wait timed out";
    case CSA_ERR_BOUNDS: return "index out of bounds on the device";
    }
    return "unknown status";
}

const char *csa_last_message(void) { return g_msg; }

csa_status csa_compress_kv(const void *Ca, const void *Cb, const void *Za, const void *Zb,
                           const float *Ba, const float *Bb, int64_t n, int c, int m,
                           int overlap, csa_dtype in_dt, csa_entries out, void *stream)
{
    const char *w = "csa_compress_kv";
    REQUIRE(Ca && Za && Ba, CSA_ERR_INVALID_ARG, "%s: Ca, Za and Ba are required", w);
    if (overlap)
        REQUIRE(Cb && Zb && Bb, CSA_ERR_INVALID_ARG, "%s: overlap needs Cb, Zb and Bb", w);
    else
        REQUIRE(!Cb && !Zb && !Bb, CSA_ERR_INVALID_ARG,
                "%s: without overlap Cb, Zb and Bb must be NULL", w);
    REQUIRE(m >= 1 && m <= 1024, CSA_ERR_INVALID_ARG, "%s: m = %d out of [1, 1024]", w, m);
    REQUIRE(n >= 0 && n % m == 0, CSA_ERR_INVALID_ARG, "%s: n = %lld must be a multiple of m",
            w, (long long)n);
    REQUIRE(in_dt == CSA_F32 || in_dt == CSA_BF16, CSA_ERR_UNSUPPORTED,
            "%s: input dtype must be F32 or BF16", w);
    const int vec = in_dt == CSA_BF16 ? 8 : 4;
    REQUIRE(c > 0 && c % vec == 0 && pow2(c / vec) && c / vec <= 256, CSA_ERR_UNSUPPORTED,
            "%s: c = %d unsupported (c / %d must be a power of two <= 256)", w, c, vec);
    REQUIRE(aligned16(Ca) && aligned16(Za) && aligned16(Ba) && (!overlap ||
            (aligned16(Cb) && aligned16(Zb) && aligned16(Bb))), CSA_ERR_INVALID_ARG,
            "%s: inputs must be 16-byte aligned", w);
    csa_status st = check_entries(out, c, true, "csa_compress_kv(out)", true);
    if (st != CSA_OK)
        return st;
    if (out.dt == CSA_E4M3) {
        REQUIRE(out.scale_group % vec == 0 && pow2(out.scale_group / vec) &&
                out.scale_group / vec <= 32, CSA_ERR_UNSUPPORTED,
                "%s: scale_group %d unsupported for this input dtype", w, out.scale_group);
    }
    if (out.dt == CSA_E2M1)
        REQUIRE(c / vec <= 32, CSA_ERR_UNSUPPORTED,
                "%s: e2m1 output needs a row within one warp (c / %d <= 32)", w, vec);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    csa::CompressArgs a{Ca, Cb, Za, Zb, Ba, Bb, n, c, m, overlap ? 1 : 0, in_dt, out};
    return launched(csa::launch_compress(a, err, (cudaStream_t)stream), w);
}

}  // extern "C"

namespace {

// Host-side checks shared by the indexer calls (scores and outputs aside).
csa_status check_indexer(const char *w, const void *qI, const float *qI_scale, const float *wI,
                         const csa_entries &kI, const int64_t *q_pos, int B, int64_t n_q,
                         int64_t E, int hI, int cI, int m, csa_dtype dt)
{
    REQUIRE(qI && wI && q_pos, CSA_ERR_INVALID_ARG, "%s: qI, wI and q_pos are required", w);
    REQUIRE(B >= 0 && n_q >= 0 && E >= 0 && E <= INT32_MAX, CSA_ERR_INVALID_ARG,
            "%s: bad B / n_q / E", w);
    REQUIRE(hI >= 1 && hI <= 128, CSA_ERR_UNSUPPORTED, "%s: hI = %d out of [1, 128]", w, hI);
    REQUIRE(cI >= 16 && cI <= 256 && cI % 16 == 0, CSA_ERR_UNSUPPORTED,
            "%s: cI = %d unsupported", w, cI);
    REQUIRE(m >= 1, CSA_ERR_INVALID_ARG, "%s: m must be >= 1", w);
    REQUIRE(dt == CSA_F32 || dt == CSA_BF16 || dt == CSA_E4M3, CSA_ERR_INVALID_ARG,
            "%s: unknown dtype", w);
    REQUIRE(kI.dt == dt || (kI.dt == CSA_E2M1 && dt == CSA_E4M3), CSA_ERR_INVALID_ARG,
            "%s: kI dtype must equal the qI dtype (or be e2m1 with e4m3 queries)", w);
    char what[64];
    snprintf(what, sizeof what, "%s(kI)", w);
    csa_status st = check_entries(kI, cI, true, what, true);
    if (st != CSA_OK)
        return st;
    if (dt == CSA_E4M3)
        REQUIRE(qI_scale, CSA_ERR_INVALID_ARG, "%s: e4m3 queries need qI_scale", w);
    if (kI.dt == CSA_E4M3)
        REQUIRE(kI.scale_group == cI && kI.rope_dims == 0, CSA_ERR_UNSUPPORTED,
                "%s: e4m3 keys need one scale per key and no rope part", w);
    REQUIRE(aligned16(qI), CSA_ERR_INVALID_ARG, "%s: qI not 16-byte aligned", w);
    return CSA_OK;
}

}  // namespace

extern "C" {

csa_status csa_indexer_scores(const void *qI, const float *qI_scale, const float *wI,
                              csa_entries kI, const int64_t *q_pos, int B, int64_t n_q,
                              int64_t E, int hI, int cI, int m, csa_dtype dt, float *scores,
                              int64_t ld, void *stream)
{
    const char *w = "csa_indexer_scores";
    REQUIRE(scores, CSA_ERR_INVALID_ARG, "%s: scores is required", w);
    csa_status st = check_indexer(w, qI, qI_scale, wI, kI, q_pos, B, n_q, E, hI, cI, m, dt);
    if (st != CSA_OK)
        return st;
    REQUIRE(ld >= E, CSA_ERR_INVALID_ARG, "%s: ld < E", w);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    csa::IndexerArgs a{qI, qI_scale, wI, kI, q_pos, B, n_q, E, hI, cI, m, dt, scores, ld};
    if ((int64_t)B * n_q == 0 || E == 0)
        return CSA_OK;
    return launched(csa::launch_indexer(a, err, (cudaStream_t)stream), w);
}

size_t csa_topk_workspace_size(int64_t rows, int64_t E, int k)
{
    return csa::topk_workspace_size(rows, E, k);
}

size_t csa_indexer_topk_workspace_size(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                                       csa_dtype dt)
{
    if (B < 0 || n_q < 0 || E < 0 || E > INT32_MAX || k < 1 || k > 4096)
        return 0;
    return csa::indexer_topk_workspace_size(B, n_q, E, hI, cI, k, dt);
}

int csa_indexer_topk_launches(int B, int64_t n_q, int64_t E, int hI, int cI, int k,
                              csa_dtype dt)
{
    if (B < 0 || n_q < 0 || E < 0 || E > INT32_MAX || k < 1 || k > 4096 ||
        (dt != CSA_F32 && dt != CSA_BF16 && dt != CSA_E4M3))
        return -1;
    // 16-byte aligned stand-ins: only the shapes decide
    static const uint8_t dummy[16] __attribute__((aligned(256))) = {0};
    csa_entries kI{};
    kI.body = const_cast<uint8_t *>(dummy);
    kI.c = cI;
    kI.dt = dt;
    csa::IndexerArgs ix{dummy, nullptr, nullptr, kI, nullptr, B, n_q, E, hI, cI, 1, dt,
                        nullptr, E};
    return csa::indexer_topk_launches(ix, k);
}

csa_status csa_indexer_topk(const void *qI, const float *qI_scale, const float *wI,
                            csa_entries kI, const int64_t *q_pos, int B, int64_t n_q, int64_t E,
                            int hI, int cI, int m, csa_dtype dt, int k, int32_t *idx,
                            void *workspace, size_t ws_bytes, void *stream)
{
    const char *w = "csa_indexer_topk";
    REQUIRE(idx, CSA_ERR_INVALID_ARG, "%s: idx is required", w);
    csa_status st = check_indexer(w, qI, qI_scale, wI, kI, q_pos, B, n_q, E, hI, cI, m, dt);
    if (st != CSA_OK)
        return st;
    REQUIRE(k >= 1 && k <= 4096, CSA_ERR_UNSUPPORTED, "%s: k = %d out of [1, 4096]", w, k);
    REQUIRE((int64_t)B * n_q <= INT32_MAX, CSA_ERR_INVALID_ARG, "%s: too many rows", w);
    const size_t need = csa::indexer_topk_workspace_size(B, n_q, E, hI, cI, k, dt);
    REQUIRE(ws_bytes >= need && (need == 0 || workspace), CSA_ERR_INVALID_ARG,
            "%s: workspace of %zu bytes required", w, need);
    REQUIRE(((uintptr_t)workspace & 255u) == 0, CSA_ERR_INVALID_ARG,
            "%s: workspace must be 256-byte aligned", w);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    csa::IndexerArgs ix{qI, qI_scale, wI, kI, q_pos, B, n_q, E, hI, cI, m, dt, nullptr, E};
    csa::IndexerTopkArgs a{ix, k, idx, workspace, ws_bytes};
    return launched(csa::launch_indexer_topk(a, err, (cudaStream_t)stream), w);
}

csa_status csa_topk(const float *scores, int64_t rows, int64_t E, int64_t ld,
                    const int64_t *q_pos, int m, int k, int32_t *idx, void *workspace,
                    size_t ws_bytes, void *stream)
{
    const char *w = "csa_topk";
    REQUIRE(scores && q_pos && idx, CSA_ERR_INVALID_ARG, "%s: scores, q_pos and idx required", w);
    REQUIRE(rows >= 0 && rows <= INT32_MAX && E >= 0 && E <= INT32_MAX && ld >= E,
            CSA_ERR_INVALID_ARG, "%s: bad rows / E / ld", w);
    REQUIRE(k >= 1 && k <= 4096, CSA_ERR_UNSUPPORTED, "%s: k = %d out of [1, 4096]", w, k);
    REQUIRE(m >= 1, CSA_ERR_INVALID_ARG, "%s: m must be >= 1", w);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    const size_t need = csa::topk_workspace_size(rows, E, k);
    REQUIRE(ws_bytes >= need && (need == 0 || workspace), CSA_ERR_INVALID_ARG,
            "%s: workspace of %zu bytes required", w, need);
    REQUIRE(((uintptr_t)workspace & 255u) == 0, CSA_ERR_INVALID_ARG,
            "%s: workspace must be 256-byte aligned", w);
    csa::TopkArgs a{scores, rows, E, ld, q_pos, m, k, idx, workspace};
    return launched(csa::launch_topk(a, err, (cudaStream_t)stream), w);
}

size_t csa_mqa_workspace_size(int B, int64_t n_q, int h, int c, int64_t max_keys)
{
    return csa::attend_workspace_size(B, n_q, h, c, max_keys);
}

}  // extern "C"

namespace csa {

// Host-side checks of an attention call, workspace excluded (see csa.h).
csa_status check_attend(const char *w, const void *q, csa_dtype q_dt, const csa_entries &kv,
                        int64_t E, const int32_t *idx, int k, int m, const void *kwin,
                        int64_t win_rows, int n_win, const int64_t *q_pos, const float *sink,
                        int B, int64_t n_q, int h, void *out)
{
    REQUIRE(q && out && q_pos && sink, CSA_ERR_INVALID_ARG,
            "%s: q, out, q_pos and sink are required", w);
    REQUIRE(q_dt == CSA_F32 || q_dt == CSA_BF16, CSA_ERR_UNSUPPORTED,
            "%s: q dtype must be F32 or BF16", w);
    const int c = kv.c;
    REQUIRE(c >= 64 && c <= 1024 && pow2(c), CSA_ERR_UNSUPPORTED,
            "%s: c = %d unsupported (a power of two from 64 to 1024)", w, c);
    csa_status st = check_entries(kv, c, q_dt == CSA_BF16, w);
    if (st != CSA_OK)
        return st;
    REQUIRE(kv.dt == q_dt || kv.dt == CSA_E4M3, CSA_ERR_UNSUPPORTED,
            "%s: entries dtype must match q (or be e4m3 with bf16 q)", w);
    REQUIRE(h >= 1 && h <= 128, CSA_ERR_UNSUPPORTED, "%s: h = %d out of [1, 128]", w, h);
    REQUIRE(B >= 0 && n_q >= 0 && (int64_t)B * n_q <= INT32_MAX && E >= 0 && E <= INT32_MAX,
            CSA_ERR_INVALID_ARG, "%s: bad B / n_q / E", w);
    REQUIRE(m >= 1, CSA_ERR_INVALID_ARG, "%s: m must be >= 1", w);
    REQUIRE(k >= 0 && k <= 4096, CSA_ERR_UNSUPPORTED, "%s: k = %d out of [0, 4096]", w, k);
    REQUIRE(k == 0 || idx, CSA_ERR_INVALID_ARG, "%s: idx required when k > 0", w);
    REQUIRE(n_win >= 0, CSA_ERR_INVALID_ARG, "%s: n_win < 0", w);
    REQUIRE(n_win == 0 || (kwin && win_rows >= 1 && aligned16(kwin)), CSA_ERR_INVALID_ARG,
            "%s: a window needs a 16-byte aligned kwin with win_rows >= 1", w);
    REQUIRE(aligned16(q) && aligned16(out), CSA_ERR_INVALID_ARG,
            "%s: q and out must be 16-byte aligned", w);
    return CSA_OK;
}

}  // namespace csa

extern "C" {

static csa_status attend_common(const char *w, const void *q, csa_dtype q_dt, csa_entries kv,
                                int64_t E, int dense, const int32_t *idx, int k, int m,
                                const void *kwin,
                                int64_t win_rows, const int64_t *win_pos0, int n_win,
                                const int64_t *q_pos, const float *sink, int B, int64_t n_q,
                                int h, float scale, void *out, float *lse, void *workspace,
                                size_t ws_bytes, void *stream)
{
    csa_status st = csa::check_attend(w, q, q_dt, kv, E, idx, k, m, kwin, win_rows, n_win,
                                      q_pos, sink, B, n_q, h, out);
    if (st != CSA_OK)
        return st;
    const int c = kv.c;
    const size_t need = csa::attend_workspace_size(B, n_q, h, c, (dense ? E : k) + n_win);
    REQUIRE(ws_bytes >= need && (need == 0 || workspace), CSA_ERR_INVALID_ARG,
            "%s: workspace of %zu bytes required", w, need);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    if ((int64_t)B * n_q == 0)
        return CSA_OK;
    csa::AttendArgs a{q, q_dt, kv, E, idx, dense, k, m, kwin, n_win > 0 ? win_rows : 0, win_pos0,
                      n_win, q_pos, sink, B, n_q, h, scale, out, lse, workspace, ws_bytes};
    return launched(csa::launch_attend(a, err, (cudaStream_t)stream), w);
}

csa_status csa_sparse_mqa(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                          const int32_t *idx, int k, const void *kwin, int64_t win_rows,
                          const int64_t *win_pos0, int n_win, const int64_t *q_pos,
                          const float *sink, int B, int64_t n_q, int h, float scale,
                          void *out, float *lse, void *workspace, size_t ws_bytes,
                          void *stream)
{
    return attend_common("csa_sparse_mqa", q, q_dt, kv, E, 0, idx, k, m, kwin, win_rows,
                         win_pos0, n_win, q_pos, sink, B, n_q, h, scale, out, lse, workspace,
                         ws_bytes, stream);
}

csa_status hca_dense_mqa(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                         const void *kwin, int64_t win_rows, const int64_t *win_pos0,
                         int n_win, const int64_t *q_pos, const float *sink, int B,
                         int64_t n_q, int h, float scale, void *out, float *lse,
                         void *workspace, size_t ws_bytes, void *stream)
{
    return attend_common("hca_dense_mqa", q, q_dt, kv, E, 1, nullptr, 0, m, kwin, win_rows,
                         win_pos0, n_win, q_pos, sink, B, n_q, h, scale, out, lse, workspace,
                         ws_bytes, stream);
}

csa_status csa_norm_rope(void *x, csa_dtype dt, const float *gamma, int64_t rows, int heads, int c,
                         int rope_dims, const int64_t *pos, int64_t pos_mul, int64_t pos_add,
                         int normalise, float eps, float base, void *stream)
{
    const char *w = "csa_norm_rope";
    REQUIRE(x, CSA_ERR_INVALID_ARG, "%s: x is NULL", w);
    REQUIRE(dt == CSA_F32 || dt == CSA_BF16, CSA_ERR_UNSUPPORTED, "%s: dtype must be F32 or BF16",
            w);
    REQUIRE(rows >= 0 && heads >= 1, CSA_ERR_INVALID_ARG, "%s: bad rows / heads", w);
    REQUIRE(c == 64 || c == 128 || c == 256 || c == 512 || c == 1024, CSA_ERR_UNSUPPORTED,
            "%s: c = %d unsupported (64 .. 1024, a power of two)", w, c);
    REQUIRE(rope_dims >= 0 && rope_dims <= c && rope_dims % 2 == 0, CSA_ERR_INVALID_ARG,
            "%s: rope_dims = %d must be even and at most c", w, rope_dims);
    REQUIRE(!normalise || eps > 0.f, CSA_ERR_INVALID_ARG, "%s: eps must be positive", w);
    REQUIRE(rope_dims == 0 || base > 1.f, CSA_ERR_INVALID_ARG, "%s: base must exceed 1", w);
    REQUIRE(aligned16(x), CSA_ERR_INVALID_ARG, "%s: x must be 16-byte aligned", w);
    csa::NormRopeArgs a{x, dt, gamma, rows, heads, c, rope_dims, pos, pos_mul, pos_add,
                        normalise ? 1 : 0, eps, base};
    return launched(csa::launch_norm_rope(a, (cudaStream_t)stream), w);
}

csa_status csa_grouped_out_proj(const void *o, const void *Wg, const void *Wo, int64_t n, int h,
                                int c, int g, int dg, int d, void *u, void *out, void *stream)
{
    const char *w = "csa_grouped_out_proj";
    REQUIRE(o && Wg && Wo && u && out, CSA_ERR_INVALID_ARG, "%s: every buffer is required", w);
    REQUIRE(n >= 0 && n <= INT32_MAX && h >= 1 && c >= 1 && g >= 1 && h % g == 0,
            CSA_ERR_INVALID_ARG, "%s: bad n / h / c / g (g must divide h)", w);
    const int64_t Kg = (int64_t)h * c / g;
    REQUIRE(Kg % 64 == 0 && Kg <= INT32_MAX, CSA_ERR_UNSUPPORTED,
            "%s: h c / g = %lld must be a multiple of 64", w, (long long)Kg);
    REQUIRE(dg >= 256 && dg % 256 == 0 && d >= 256 && d % 256 == 0, CSA_ERR_UNSUPPORTED,
            "%s: d_g and d must be multiples of 256", w);
    REQUIRE((int64_t)g * dg % 64 == 0, CSA_ERR_UNSUPPORTED, "%s: g d_g must be a multiple of 64",
            w);
    REQUIRE(aligned16(o) && aligned16(Wg) && aligned16(Wo) && aligned16(u) && aligned16(out),
            CSA_ERR_INVALID_ARG, "%s: buffers must be 16-byte aligned", w);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    if (n == 0)
        return CSA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    csa::GemmArgs a1{o, Wg, u, n, dg, (int)Kg, g, (int64_t)h * c, (int64_t)g * dg,
                     (int64_t)g * dg, Kg, dg, dg};
    cudaError_t e = csa::launch_gemm_nt(a1, err, s);
    if (e != cudaSuccess)
        return launched(e, w);
    csa::GemmArgs a2{u, Wo, out, n, d, g * dg, 1, (int64_t)g * dg, d, d, 0, 0, 0};
    return launched(csa::launch_gemm_nt(a2, err, s), w);
}

csa_status csa_debug_wait_probe(uint64_t limit_ns, void *stream)
{
    const char *w = "csa_debug_wait_probe";
    REQUIRE(limit_ns >= 1000u && limit_ns <= 1000000000u, CSA_ERR_INVALID_ARG,
            "%s: limit_ns = %llu out of [1e3, 1e9]", w, (unsigned long long)limit_ns);
    unsigned *err = err_word();
    REQUIRE(err, CSA_ERR_CUDA, "%s: no CUDA device", w);
    return launched(csa::launch_wait_probe(limit_ns, err, (cudaStream_t)stream), w);
}

csa_status csa_get_error(char *buf, size_t len)
{
    if (cudaDeviceSynchronize() != cudaSuccess) {
        if (buf && len)
            snprintf(buf, len, "CUDA error: %s", cudaGetErrorString(cudaGetLastError()));
        return CSA_ERR_CUDA;
    }
    unsigned h[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(h, g_err, sizeof h) != cudaSuccess)
        return CSA_ERR_CUDA;
    const unsigned zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_err, zero, sizeof zero) != cudaSuccess)
        return CSA_ERR_CUDA;
    const csa_status st = (csa_status)(-(int)h[0]);
    if (buf && len) {
        if (h[0])
            snprintf(buf, len, "%s (kernel %u, detail %u %u)", csa_status_string(st), h[1], h[2],
                     h[3]);
        else
            snprintf(buf, len, "%s", "ok");
    }
    return st;
}

}  // extern "C"
