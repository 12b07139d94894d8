// noalloc.cu -- csa_sparse_mqa for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc on their hot path: code hosted inside a
// framework that owns every byte of device memory through pre-reserved pools
// and forbids new allocations, or a decode loop that must not pay the
// implicit device-wide synchronisation an allocation can cause. For them,
// csa_sparse_mqa_noalloc takes its scratch (the split-key partial results of
// the attention) from a file-scope device array of fixed size instead of a
// caller-provided workspace. The array lives in every GPU that loads the
// library, for the life of the process.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// 32 MiB per GPU: enough for an 8-query decode step with 64 heads of width
// 512 over 1024 selected entries and a 128-row window (18 key chunks per
// query, 18.9 MB of partial results).
constexpr size_t kScratchBytes = 32u << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of this GPU's scratch array. In host code the array's name
// only stands in for the symbol, so the address is looked up once per device,
// with that device current, and kept for the life of the process: it does
// not survive a reset of the device (cudaDeviceReset), after which this entry
// point must not be called again in the same process.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t csa_noalloc_scratch_bytes(void) { return kScratchBytes; }

csa_status csa_sparse_mqa_noalloc(const void *q, csa_dtype q_dt, csa_entries kv, int64_t E, int m,
                                  const int32_t *idx, int k, const void *kwin, int64_t win_rows,
                                  const int64_t *win_pos0, int n_win, const int64_t *q_pos,
                                  const float *sink, int B, int64_t n_q, int h, float scale,
                                  void *out, float *lse, void *stream)
{
    // the arguments are checked before the scratch is sized from them
    const csa_status st = csa::check_attend("csa_sparse_mqa_noalloc", q, q_dt, kv, E, idx, k, m,
                                            kwin, win_rows, n_win, q_pos, sink, B, n_q, h, out);
    if (st != CSA_OK)
        return st;
    const size_t need = csa_mqa_workspace_size(B, n_q, h, kv.c, (int64_t)k + n_win);
    if (need > kScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "csa_sparse_mqa_noalloc: this shape needs %zu bytes of scratch; the fixed "
                 "array holds %zu (use csa_sparse_mqa with a workspace)",
                 need, kScratchBytes);
        csa::set_last_message(msg);
        return CSA_ERR_UNSUPPORTED;
    }
    // set-up on the first call on each device (before any stream capture)
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess)
        return CSA_ERR_CUDA;
    return csa_sparse_mqa(q, q_dt, kv, E, m, idx, k, kwin, win_rows, win_pos0, n_win, q_pos, sink,
                          B, n_q, h, scale, out, lse, scratch, need > 0 ? kScratchBytes : 0,
                          stream);
}

}  // extern "C"
