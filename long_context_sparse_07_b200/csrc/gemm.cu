// gemm.cu -- the grouped output projection (Module B step 4) on the
// 5th-generation tensor cores.
//
// The n_h head outputs of a token are cut into g groups; group j (n_h / g
// heads, K_g = n_h c / g values) is projected to d_g values, and the g
// results are concatenated and projected to d:
//   U[:, j d_g : (j+1) d_g] = O[:, j K_g : (j+1) K_g] . W_g[j]^T   (j < g)
//   OUT = U . W_o^T
// Both are "NT" products C[M, N] = A[M, K] . B[N, K]^T with bf16 operands,
// float32 accumulation and bf16 results: A rows are tokens, B rows are output
// features (weights stored [out, in]), both K-major.
//
// One persistent kernel takes either product (the first as g independent
// groups): tiles of M = 128 rows x N = 256 columns, K in steps of 64 through
// a 4-stage TMA ring (128-byte swizzle), accumulators double-buffered in
// tensor memory so that the epilogue of one tile overlaps the MMAs of the
// next. Warp 0 issues the TMA loads, warp 1 the MMAs, warps 2-5 (one per TMEM
// lane quarter) drain the accumulators to bf16 rows of C. Tiles run n-tile
// fastest, so the CTAs working at one time share their A rows through L2.
// Every wait is bounded; on expiry the kernel records CSA_ERR_TIMEOUT, lets
// its copies and products land and returns.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma_host.h"

namespace csa {

namespace {

constexpr int GM = 128, GN = 256, GK = 64;
constexpr int GSTAGES = 4;
constexpr int GTHREADS = 192;
constexpr uint32_t GA_BYTES = GM * GK * 2, GB_BYTES = GN * GK * 2;
constexpr uint32_t GIDESC = tc::idesc_bf16(GM, GN);

struct GemmDev {
    int64_t M;
    int N, K, groups;
    int64_t a_col_off, b_row_off, c_col_off;   // per group
    __nv_bfloat16 *C;
    int64_t ldc;
    unsigned *err;
};

__global__ void __launch_bounds__(GTHREADS, 1)
gemm_nt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const GemmDev a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = sm;
    uint8_t *sB = sm + GSTAGES * GA_BYTES;
    uint64_t *bars = (uint64_t *)(sB + GSTAGES * GB_BYTES);
    uint64_t *full = bars, *empty = bars + GSTAGES;
    uint64_t *accf = bars + 2 * GSTAGES, *acce = accf + 2, *done = acce + 2;
    uint32_t *tmem_slot = (uint32_t *)(done + 1);
    int *abort_flag = (int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t mt = (a.M + GM - 1) / GM;
    const int nt = a.N / GN;
    const int64_t ntiles = (int64_t)a.groups * mt * nt;
    const int ksteps = a.K / GK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < GSTAGES; i++) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&accf[i], 1);
            tc::mbar_init(&acce[i], 4);
        }
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
        tc::tma_prefetch_desc(&tmA);
        tc::tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int *abortv = abort_flag;

    // tile t -> (group, m tile, n tile), n fastest
    auto coords = [&](int64_t t, int &grp, int64_t &mi, int &ni) {
        ni = (int)(t % nt);
        const int64_t r = t / nt;
        mi = r % mt;
        grp = (int)(r / mt);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                int grp, ni;
                int64_t mi;
                coords(t, grp, mi, ni);
                const int ax = (int)(grp * a.a_col_off);
                const int ay = (int)(mi * GM);
                const int by = (int)(grp * a.b_row_off + (int64_t)ni * GN);
                for (int ks = 0; ks < ksteps; ks++, it++) {
                    const int st = it % GSTAGES;
                    if (it >= GSTAGES &&
                        !tc::mbar_wait(&empty[st], ((it / GSTAGES) - 1) & 1, abortv)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[st], GA_BYTES + GB_BYTES);
                    tc::tma_load_2d(sA + st * GA_BYTES, &tmA, &full[st], ax + ks * GK, ay);
                    tc::tma_load_2d(sB + st * GB_BYTES, &tmB, &full[st], ks * GK, by);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_GEMM, blockIdx.x, 0);
            }
            // let the copies in flight land before the block exits
            volatile int never = 0;
            for (uint32_t j = it > GSTAGES ? it - GSTAGES : 0; j < it; j++)
                static_cast<void>(
                    tc::mbar_wait(&full[j % GSTAGES], (j / GSTAGES) & 1, &never, 200000000ull));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            uint32_t it = 0, tc_ = 0;
            bool ok = true;
            const uint32_t sAa = tc::smem_u32(sA), sBa = tc::smem_u32(sB);
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x, tc_++) {
                const int buf = tc_ & 1;
                if (tc_ >= 2 && !tc::mbar_wait(&acce[buf], ((tc_ / 2) - 1) & 1, abortv)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * GN);
                for (int ks = 0; ks < ksteps; ks++, it++) {
                    const int st = it % GSTAGES;
                    if (!tc::mbar_wait(&full[st], (it / GSTAGES) & 1, abortv)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
#pragma unroll
                    for (int kk = 0; kk < GK / 16; kk++) {
                        const uint64_t ad = tc::sdesc_sw128(sAa + st * GA_BYTES + kk * 32);
                        const uint64_t bd = tc::sdesc_sw128(sBa + st * GB_BYTES + kk * 32);
                        tc::mma_f16(d, ad, bd, GIDESC, (ks | kk) != 0);
                    }
                    tc::mma_commit(&empty[st]);
                }
                if (!ok)
                    break;
                tc::mma_commit(&accf[buf]);
            }
            if (!ok) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_GEMM, blockIdx.x, 1);
            }
            tc::mma_commit(done);
            volatile int never = 0;
            static_cast<void>(tc::mbar_wait(done, 0, &never, 200000000ull));
        }
    } else {
        // ---------------- epilogue: warps 2-5, lane quarter warp % 4 = rows
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t tc_ = 0;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, tc_++) {
            int grp, ni;
            int64_t mi;
            coords(t, grp, mi, ni);
            const int buf = tc_ & 1;
            if (!tc::mbar_wait(&accf[buf], (tc_ / 2) & 1, abortv)) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_GEMM, blockIdx.x, 2);
                break;
            }
            tc::fence_after();
            const int64_t r = mi * GM + row;
            __nv_bfloat16 *crow = a.C + r * a.ldc + grp * a.c_col_off + (int64_t)ni * GN;
#pragma unroll 1
            for (int ch = 0; ch < GN / 32; ch++) {
                uint32_t v[32];
                tc::tmem_ld32(lane_addr + (uint32_t)(buf * GN + ch * 32), v);
                tc::tmem_ld_wait();
                if (r < a.M) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                        pk[j] = *(const uint32_t *)&b2;
                    }
                    uint4 *dst = (uint4 *)(crow + ch * 32);
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                tc::mbar_arrive(&acce[buf]);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

size_t gemm_smem_bytes() { return 1024 + GSTAGES * (GA_BYTES + GB_BYTES) + 256; }

cudaError_t launch_gemm_nt(const GemmArgs &g, unsigned *err, cudaStream_t s)
{
    CUtensorMap tmA, tmB;
    if (!make_tmap_2d(&tmA, g.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.M,
                      (uint64_t)g.lda, GM) ||
        !make_tmap_2d(&tmB, g.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.b_rows,
                      (uint64_t)g.K, GN))
        return cudaErrorInvalidValue;
    GemmDev d;
    d.M = g.M;
    d.N = g.N;
    d.K = g.K;
    d.groups = g.groups;
    d.a_col_off = g.a_col_off;
    d.b_row_off = g.b_row_off;
    d.c_col_off = g.c_col_off;
    d.C = (__nv_bfloat16 *)g.C;
    d.ldc = g.ldc;
    d.err = err;
    const size_t smem = gemm_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(gemm_nt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = (int64_t)g.groups * ((g.M + GM - 1) / GM) * (g.N / GN);
    const int64_t grid = tiles < sms ? tiles : sms;
    if (grid <= 0)
        return cudaSuccess;
    gemm_nt_kernel<<<(unsigned)grid, GTHREADS, smem, s>>>(tmA, tmB, d);
    return cudaGetLastError();
}

}  // namespace csa
