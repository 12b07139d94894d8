// indexer_tc.cu -- lightning-indexer scores (Eq. 16) on the 5th-generation
// tensor cores (tcgen05 + TMEM), fed by TMA.
//
// The contraction q^I . k^I is the one dense GEMM of the path. Operands are
// swapped so that each TMEM lane holds one compressed key: the MMA computes
//   D[key][(token, head)] = sum_x kI[key][x] * qI[token][head][x]
// with M = 128 keys (A, streamed), N = NT tokens x HI heads (B, resident),
// K = c_I (bf16: kind::f16, 16 per MMA; e4m3: kind::f8f6f4, 32 per MMA).
// The epilogue thread that owns a key lane then reduces over heads inside
// its registers: I[t][s] = kscale[s] * sum_h w'[t][h] * ReLU(D[s][(t, h)]),
// with w' = wI * qI_scale (scales are positive, so they commute with ReLU);
// pairs of heads go through one packed fp32 FMA (fma.rn.f32x2).
//
// A block owns NSUB x NT tokens: every key tile in shared memory feeds NSUB
// MMAs of N = NT x HI (one per group of NT tokens), so a key tile is read
// from L2 once per NSUB x NT tokens. The accumulators of consecutive
// (key tile, token group) pairs alternate between two TMEM buffers, so the
// epilogue of one overlaps the MMA of the next.
//
// Warp roles: warp 0 issues TMA loads (query tile once, then a ring of
// key-tile stages), warp 1 owns TMEM and issues the MMAs, warps 2.. drain the
// accumulators and write score rows: four warps per TMEM lane quarter when a
// token group holds 4 or more tokens (each takes a quarter of the tokens),
// since the head reduction costs more than the MMAs that feed it. Key tiles
// past the causal bound of every token of the block are never loaded; score
// entries s >= V_t are not written. Token blocks are launched longest first
// (the causal triangle makes the last tokens' rows the longest). Every wait
// is bounded; on expiry the block records CSA_ERR_TIMEOUT, drains its own
// copies and returns.
//
// FP4 keys (K4; e2m1 codes with a power-of-two scale 2^(e - 127) per 32
// channels, against e4m3 queries): the key tiles arrive packed (64 bytes per
// key) in a ring of their own, and added warps turn each key into e4m3 codes
// in the swizzled layout the MMA reads: channel value e2m1 * 2^-(emax - e)
// (e4m3 holds every such value exactly for emax - e <= 8), the key's largest
// block scale 2^(emax - 127) being applied in the epilogue like an e4m3
// key's scale. The products are then exact in the e4m3 MMA.
#include <cuda_fp4.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma_host.h"

namespace csa {

namespace {

struct TcArgs {
    const float *wI, *qI_scale, *kI_scale;
    const int64_t *q_pos;
    int64_t n_q, E;
    int m, kb;            // kb: 128-byte blocks per row of c_I
    int nchunks;
    int64_t key_chunk;
    float *scores;
    int64_t ld;
    int64_t ks_stride;    // key s has its scale at kI_scale[s * ks_stride]
                          // (FP4: its 4 block exponents at kI_exp[4 * s * ks_stride])
    const uint8_t *kI_exp;
    const int *row_flag;  // when set: blocks none of whose tokens is flagged exit
    // candidate mode (FUSE): every visible key of row r scoring at or above
    // bound[r] is kept as a (score bits, index) pair in cand; rows of at most
    // k visible keys keep nothing
    const float *bound;
    int k;
    uint2 *cand;          // row r, chunk c, list l: cand[r * cand_ld + c * key_chunk / 2
                          //                             + l * room of a list ..]
    int64_t cand_ld;
    uint32_t *cnt;        // [rows][nchunks][lists] pairs found (may exceed the room)
    unsigned *err;
};

template <bool FP8, int HI, int NT, int NSUB, bool K4 = false>
struct Cfg {
    static constexpr int N = NT * HI;          // columns of one accumulator
    static constexpr int TT = NT * NSUB;       // tokens of a block
    static constexpr int QROWS = TT * HI;      // query rows (token, head) of a block
    // epilogue: SPLIT warps per TMEM lane quarter drain NT / SPLIT tokens
    // each; with one token per group (decode) two such warp sets drain
    // alternate accumulators (set s takes those in TMEM buffer s). A token's
    // HI columns are read in chunks of CW columns, the next chunk loading
    // while one is reduced.
    static constexpr int NSET = NT == 1 ? 2 : 1;
    static constexpr int SPLIT = NT >= 4 ? 4 : NT;
    static constexpr int TPW = NT / SPLIT;
    static constexpr int CW = HI < 32 ? HI : 32;
    static constexpr int CPT = HI / CW;
    static constexpr int NE = 4 * NSET * SPLIT;         // epilogue warps
    static constexpr int UW = K4 ? (NT == 1 ? 8 : 2) : 0;  // FP4 unpack warps
    static constexpr int THREADS = 32 * (2 + NE + UW);
    // FP4 keys (c_I = 128): a 16 KB e4m3 stage and an 8 KB packed stage each;
    // one-token blocks (decode) are sized for two blocks per SM
    static constexpr int K4_BUDGET = NT == 1 ? 113 * 1024 : 227 * 1024;
    static constexpr int K4_STAGES_FIT =
        (K4_BUDGET - 2048 - QROWS * 128 - QROWS * 4 - TT * 16 - 256 - 128) / (16384 + 8192);
    static constexpr int STAGES =
        K4 ? (K4_STAGES_FIT > 6 ? 6 : K4_STAGES_FIT) : (FP8 ? (NSUB > 1 ? 4 : 6) : 4);
    static constexpr int TMEM_COLS = (2 * N) < 32 ? 32 : 2 * N;
    static constexpr uint32_t IDESC = FP8 ? tc::idesc_e4m3(128, N) : tc::idesc_bf16(128, N);
    static size_t smem_bytes(int kb)
    {
        return 1024 + (size_t)kb * QROWS * 128 + (size_t)STAGES * kb * 16384 +
               (K4 ? (size_t)STAGES * 8192 + 128 : 0) + 256 + QROWS * 4 + TT * 16;
    }
};

// Byte permute (default mode): byte n of the result is byte (c >> 4n) & 7 of
// {b, a} (a = bytes 0-3); with bit 3 of that selector set, the selected
// byte's top bit is replicated over the result byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// sum_h w[h] * max(x[h], 0) over HI heads (x: raw TMEM words), two heads per
// packed fp32 FMA, two independent accumulator pairs.
template <int HI>
__device__ __forceinline__ float relu_dot(const uint32_t *x, const float *w)
{
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < HI; j += 4) {
        const float4 wv = *(const float4 *)(w + j);
        const float2 xa = make_float2(fmaxf(__uint_as_float(x[j]), 0.f),
                                      fmaxf(__uint_as_float(x[j + 1]), 0.f));
        const float2 xb = make_float2(fmaxf(__uint_as_float(x[j + 2]), 0.f),
                                      fmaxf(__uint_as_float(x[j + 3]), 0.f));
        acc0 = __ffma2_rn(xa, make_float2(wv.x, wv.y), acc0);
        acc1 = __ffma2_rn(xb, make_float2(wv.z, wv.w), acc1);
    }
    acc0 = __fadd2_rn(acc0, acc1);
    return acc0.x + acc0.y;
}

template <bool FP8, int HI, int NT, int NSUB, bool FUSE, bool K4>
__global__ void __launch_bounds__(Cfg<FP8, HI, NT, NSUB, K4>::THREADS, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmq,
                  const TcArgs a)
{
    using C = Cfg<FP8, HI, NT, NSUB, K4>;
    constexpr int N = C::N;
    constexpr int TT = C::TT;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int KB = a.kb;
    uint8_t *sB = smem;
    uint8_t *sA = sB + (size_t)KB * C::QROWS * 128;
    uint8_t *sR = sA + (size_t)S * KB * 16384;               // K4: packed key tiles
    uint64_t *bars = (uint64_t *)(sR + (K4 ? (size_t)S * 8192 : 0));
    uint64_t *full = bars, *empty = bars + S, *bfull = bars + 2 * S;
    uint64_t *accf = bfull + 1, *acce = accf + 2, *done = acce + 2;
    uint64_t *rfull = bars + 18, *rempty = bars + 24;          // K4 (S <= 6)
    uint32_t *tmem_slot = (uint32_t *)(bars + 30);
    int *abort_flag = (int *)(tmem_slot + 1);
    float *wsm = (float *)(bars + 32);
    int64_t *vt = (int64_t *)(wsm + C::QROWS);
    float *lbound = (float *)(vt + TT);            // FUSE: per token
    // K4: e4m3 byte of each e2m1 magnitude times 2^-j, j = 0..8 (2 words each)
    uint32_t *lut = (uint32_t *)((uint8_t *)vt + TT * 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int64_t ttiles = (a.n_q + TT - 1) / TT;
    // longest rows first: token block (ttiles - 1) is launched first
    const int64_t tile = ttiles - 1 - blockIdx.x / a.nchunks;
    const int chunk = blockIdx.x % a.nchunks;
    const int64_t t0 = tile * TT;

    if (threadIdx.x < TT) {
        const int64_t t = t0 + threadIdx.x;
        int64_t v = t < a.n_q ? visible(a.q_pos[(int64_t)b * a.n_q + t], a.m, a.E) : 0;
        if (a.row_flag && v > 0 && a.row_flag[(int64_t)b * a.n_q + t] == 0)
            v = 0;                                 // a row that needs no scores
        vt[threadIdx.x] = v;
    }
    if (threadIdx.x == 0)
        *abort_flag = 0;
    __syncthreads();
    int64_t vmax = 0;
#pragma unroll
    for (int tt = 0; tt < TT; tt++)
        vmax = vt[tt] > vmax ? vt[tt] : vmax;
    const int64_t s_begin = (int64_t)chunk * a.key_chunk;
    int64_t s_end = s_begin + a.key_chunk;
    if (s_end > vmax)
        s_end = vmax;
    if (s_end <= s_begin)
        return;                                   // uniform: nothing visible here
    const int ntiles = (int)((s_end - s_begin + 127) / 128);

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < S; i++) {
            tc::mbar_init(&full[i], K4 ? C::UW : 1);
            tc::mbar_init(&empty[i], 1);
            if (K4) {
                tc::mbar_init(&rfull[i], 1);
                tc::mbar_init(&rempty[i], C::UW);
            }
        }
        tc::mbar_init(bfull, 1);
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&accf[i], 1);
            tc::mbar_init(&acce[i], 4 * C::SPLIT);     // the warps that drain buffer i
        }
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmk);
        tc::tma_prefetch_desc(&tmq);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (warp >= 2 && warp < 2 + C::NE) {
        for (int col = threadIdx.x - 64; col < C::QROWS; col += 32 * C::NE) {
            const int tt = col / HI, hh = col % HI;
            const int64_t t = t0 + tt;
            float wv = 0.f;
            if (t < a.n_q) {
                const int64_t r = ((int64_t)b * a.n_q + t) * HI + hh;
                wv = a.wI[r];
                if (FP8)
                    wv *= a.qI_scale[r];
            }
            wsm[col] = wv;
        }
        if constexpr (FUSE) {
            // each token's bound (NaN: the row keeps nothing here, all of its
            // visible keys being the selection)
            for (int tt = threadIdx.x - 64; tt < TT; tt += 32 * C::NE) {
                const int64_t t = t0 + tt;
                lbound[tt] = t < a.n_q && vt[tt] > a.k ? a.bound[(int64_t)b * a.n_q + t]
                                                        : __int_as_float(0x7fc00000);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer
            const int xstep = FP8 ? 128 : 64;    // elements per 128-byte block
            constexpr int QBOX = C::QROWS < 256 ? C::QROWS : 256;
            int issued = 0;
            bool ok = true;
            tc::mbar_arrive_expect_tx(bfull, (uint32_t)(KB * C::QROWS * 128));
            for (int kb = 0; kb < KB; kb++)
                for (int r0 = 0; r0 < C::QROWS; r0 += QBOX)
                    tc::tma_load_2d(sB + ((size_t)kb * C::QROWS + r0) * 128, &tmq, bfull,
                                    kb * xstep, (int)(((int64_t)b * a.n_q + t0) * HI + r0));
            // K4: the packed tiles go to their own ring, freed by the unpack
            // warps; otherwise the e4m3 / bf16 tiles straight to the MMA ring
            uint64_t *lfull = K4 ? rfull : full, *lempty = K4 ? rempty : empty;
            for (int i = 0; i < ntiles && ok; i++) {
                const int st = i % S;
                if (i >= S && !tc::mbar_wait(&lempty[st], ((i / S) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int row0 = (int)((int64_t)b * a.E + s_begin + (int64_t)i * 128);
                if constexpr (K4) {
                    tc::mbar_arrive_expect_tx(&rfull[st], 8192u);
                    tc::tma_load_2d(sR + (size_t)st * 8192, &tmk, &rfull[st], 0, row0);
                } else {
                    tc::mbar_arrive_expect_tx(&full[st], (uint32_t)(KB * 16384));
                    for (int kb = 0; kb < KB; kb++)
                        tc::tma_load_2d(sA + (size_t)(st * KB + kb) * 16384, &tmk, &full[st],
                                        kb * xstep, row0);
                }
                issued = i + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_INDEXER_TC, blockIdx.x, 0);
                // let the copies already in flight land before the block exits
                volatile int never = 0;
                static_cast<void>(tc::mbar_wait(bfull, 0, &never, 200000000ull));
                for (int i = issued - S < 0 ? 0 : issued - S; i < issued; i++)
                    static_cast<void>(tc::mbar_wait(&lfull[i % S], (i / S) & 1, &never, 200000000ull));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: for each key tile, one MMA group per
            // token group into the next accumulator buffer
            bool ok = tc::mbar_wait(bfull, 0, abort_flag);
            const uint32_t sBa = tc::smem_u32(sB);
            for (int i = 0; i < ntiles && ok; i++) {
                const int st = i % S;
                if (!tc::mbar_wait(&full[st], (i / S) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t sAa = tc::smem_u32(sA + (size_t)st * KB * 16384);
#pragma unroll 1
                for (int j = 0; j < NSUB && ok; j++) {
                    const int g = i * NSUB + j, buf = g & 1;
                    if (g >= 2 && !tc::mbar_wait(&acce[buf], ((g / 2) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t d = tmem + (uint32_t)(buf * N);
#pragma unroll 1
                    for (int kb = 0; kb < KB; kb++) {
#pragma unroll
                        for (int kk = 0; kk < 4; kk++) {
                            const uint64_t ad = tc::sdesc_sw128(sAa + kb * 16384 + kk * 32);
                            const uint64_t bd = tc::sdesc_sw128(
                                sBa + ((uint32_t)kb * C::QROWS + (uint32_t)j * N) * 128 + kk * 32);
                            if (FP8)
                                tc::mma_f8(d, ad, bd, C::IDESC, (kb | kk) != 0);
                            else
                                tc::mma_f16(d, ad, bd, C::IDESC, (kb | kk) != 0);
                        }
                    }
                    tc::mma_commit(&accf[buf]);
                }
                tc::mma_commit(&empty[st]);
            }
            if (!ok) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_INDEXER_TC, blockIdx.x, 1);
            }
            // every MMA issued above has completed once `done` flips
            tc::mma_commit(done);
            volatile int never = 0;
            static_cast<void>(tc::mbar_wait(done, 0, &never, 200000000ull));
        }
    } else if (warp < 2 + C::NE) {
        // ---------------- epilogue: warps 2..; set = which TMEM buffer (with
        // two sets), lane quarter = warp % 4; in each token group, tokens
        // part * TPW .. part * TPW + TPW - 1
        constexpr int CW = C::CW, CPT = C::CPT, NC = C::TPW * C::CPT;
        const int q4 = warp & 3;
        const int set = (warp - 2) / (4 * C::SPLIT);
        const int part = ((warp - 2) >> 2) % C::SPLIT;
        const int row = q4 * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        // FUSE: a token's pairs from this key chunk go to one list per
        // epilogue warp that reduces it ((set, lane quarter): 4 NSET lists),
        // each with an equal share of the chunk's room; the warp counts its
        // lists in registers (the same count on every lane)
        constexpr int LISTS = 4 * C::NSET;
        const unsigned room_l =
            (unsigned)(((s_begin + a.key_chunk < a.E ? s_begin + a.key_chunk : a.E) - s_begin) / 2 /
                       LISTS);
        const int list = set * 4 + q4;
        const unsigned lt = (1u << lane) - 1u;
        // per token of this warp (slot j * TPW + x): its list, bound and
        // visible length, kept in registers across the key tiles
        // (the candidate area of a row is at most a few MB: offsets within a
        // block's rows fit in 32 bits)
        constexpr int SLOTS = FUSE ? NSUB * C::TPW : 1;
        uint2 *const dbase =
            a.cand + ((int64_t)b * a.n_q + t0) * a.cand_ld + s_begin / 2 + (int64_t)list * room_l;
        const unsigned cld = (unsigned)a.cand_ld;
        unsigned wc[SLOTS];
        float lbv[SLOTS];
#pragma unroll
        for (int j = 0; j < SLOTS; j++) {
            const int tt = (j / C::TPW) * NT + part * C::TPW + j % C::TPW;
            wc[j] = 0u;
            lbv[j] = FUSE ? lbound[tt] : 0.f;
        }
        bool ok = true;
        for (int i = 0; i < ntiles && ok; i++) {
            if (C::NSET == 2 && NSUB == 1 && (i & 1) != set)
                continue;
            const int64_t s = s_begin + (int64_t)i * 128 + row;
            // the key's scale is requested before the wait for its accumulator
            float ks = 1.f;
            if constexpr (K4) {
                // the key's largest block scale, 2^(emax - 127)
                ks = 0.f;
                if (s < a.E) {
                    const uint32_t ex =
                        __ldg((const uint32_t *)a.kI_exp + ((int64_t)b * a.E + s) * a.ks_stride);
                    const uint32_t em = max(max(ex & 255u, (ex >> 8) & 255u),
                                            max((ex >> 16) & 255u, ex >> 24));
                    ks = em ? __uint_as_float(em << 23) : __uint_as_float(1u << 22);
                }
            } else if (FP8) {
                ks = s < a.E ? __ldg(a.kI_scale + ((int64_t)b * a.E + s) * a.ks_stride) : 0.f;
            }
            auto group = [&](const int j) {
                const int g = i * NSUB + j, buf = g & 1;
                if (C::NSET == 2 && buf != set)
                    return;
                if (!tc::mbar_wait(&accf[buf], (g / 2) & 1, abort_flag)) {
                    *abort_flag = 1;
                    report(a.err, CSA_ERR_TIMEOUT, K_INDEXER_TC, blockIdx.x, 2);
                    ok = false;
                    return;
                }
                tc::fence_after();
                const uint32_t base = lane_addr + (uint32_t)(buf * N);
                // chunk c: columns (part * TPW + c / CPT) * HI + (c % CPT) * CW
                uint32_t rb[2][CW];
                auto load = [&](int c, uint32_t(&r)[CW]) {
                    const uint32_t col = (uint32_t)((part * C::TPW + c / CPT) * HI + (c % CPT) * CW);
                    if constexpr (CW == 32)
                        tc::tmem_ld32(base + col, r);
                    else
                        tc::tmem_ld16(base + col, r);
                };
                load(0, rb[0]);
                tc::tmem_ld_wait();
                float sacc = 0.f;
#pragma unroll
                for (int c = 0; c < NC; c++) {
                    if (c + 1 < NC)
                        load(c + 1, rb[(c + 1) & 1]);
                    const int tl = part * C::TPW + c / CPT;   // token inside the group
                    const int tt = j * NT + tl;               // token inside the block
                    sacc += relu_dot<CW>(rb[c & 1], wsm + tt * HI + (c % CPT) * CW);
                    if (c % CPT == CPT - 1) {
                        const int64_t t = t0 + tt;
                        if constexpr (FUSE) {
                            // candidates of token tt: the lanes at or above
                            // its bound, in lane order after this list's count
                            const int sl = j * C::TPW + c / CPT;
                            const float v = sacc * ks;
                            const bool on = s < vt[tt] && v >= lbv[sl];
                            const unsigned bal = __ballot_sync(0xffffffffu, on);
                            const unsigned at = wc[sl] + (unsigned)__popc(bal & lt);
                            if (on && at < room_l)
                                dbase[(unsigned)tt * cld + at] =
                                    make_uint2(__float_as_uint(v), (uint32_t)s);
                            wc[sl] += (unsigned)__popc(bal);
                        } else {
                            if (t < a.n_q && s < vt[tt])
                                a.scores[((int64_t)b * a.n_q + t) * a.ld + s] = sacc * ks;
                        }
                        sacc = 0.f;
                    }
                    if (c + 1 < NC)
                        tc::tmem_ld_wait();
                }
                tc::fence_before();
                __syncwarp();
                if (lane == 0)
                    tc::mbar_arrive(&acce[buf]);
            };
            if constexpr (FUSE) {
                // unrolled, so that every list count stays in a register
#pragma unroll
                for (int j = 0; j < NSUB; j++)
                    if (ok)
                        group(j);
            } else {
#pragma unroll 1
                for (int j = 0; j < NSUB && ok; j++)
                    group(j);
            }
        }
        if constexpr (FUSE) {
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < NSUB; j++)
#pragma unroll
                    for (int x = 0; x < C::TPW; x++) {
                        const int64_t t = t0 + j * NT + part * C::TPW + x;
                        if (t < a.n_q)
                            a.cnt[(((int64_t)b * a.n_q + t) * a.nchunks + chunk) * LISTS +
                                  list] = wc[j * C::TPW + x];
                    }
            }
        }
    } else if constexpr (K4) {
        // ---------------- FP4 unpack warps: packed key rows -> e4m3 rows in
        // the 128-byte swizzled layout of the MMA's A tile. A block's 32
        // channels share one j = emax - e; the e4m3 bytes of the 8 e2m1
        // magnitudes times 2^-j come from a table of two words selected with
        // byte permutes, the sign bits are moved in with a second permute.
        const int uw = warp - 2 - C::NE;
        if (uw == 0 && lane < 9) {
            uint32_t t[2] = {0u, 0u};
#pragma unroll
            for (int mag = 0; mag < 8; mag++) {
                const __half_raw h = __nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)mag, __NV_E2M1);
                const float v = __half2float(__half(h)) * __uint_as_float((uint32_t)(127 - lane) << 23);
                const uint32_t e8 = (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
                t[mag >> 2] |= e8 << (8 * (mag & 3));
            }
            lut[2 * lane] = t[0];
            lut[2 * lane + 1] = t[1];
        }
        tc::named_bar_sync(1, 32 * C::UW);
        // thread ut takes RPT rows (or, with more threads than rows, BPT of
        // a row's 4 channel blocks); the block exponents of its rows are
        // loaded one tile ahead (rows past the table, zero-filled, take j = 0)
        constexpr int UT = 32 * C::UW;
        constexpr int TPR = UT > 128 ? UT / 128 : 1;         // threads per row
        constexpr int RPT = UT >= 128 ? 1 : 128 / UT;        // rows per thread
        constexpr int BPT = 4 / TPR;                         // blocks per thread
        const int ut = uw * 32 + lane;
        auto row_of = [&](int x) { return ut / TPR + x * (UT / TPR); };
        auto exps_of = [&](int i, uint32_t(&e)[RPT]) {
#pragma unroll
            for (int x = 0; x < RPT; x++) {
                const int64_t s = s_begin + (int64_t)i * 128 + row_of(x);
                e[x] = (i < ntiles && s < a.E)
                           ? __ldg((const uint32_t *)a.kI_exp + ((int64_t)b * a.E + s) * a.ks_stride)
                           : 0x7f7f7f7fu;
            }
        };
        uint32_t exn[RPT];
        exps_of(0, exn);
        bool ok = true;
        for (int i = 0; i < ntiles && ok; i++) {
            const int st = i % S;
            uint32_t exc[RPT];
#pragma unroll
            for (int x = 0; x < RPT; x++)
                exc[x] = exn[x];
            exps_of(i + 1, exn);
            if (!tc::mbar_wait(&rfull[st], (i / S) & 1, abort_flag) ||
                (i >= S && !tc::mbar_wait(&empty[st], ((i / S) - 1) & 1, abort_flag))) {
                *abort_flag = 1;
                report(a.err, CSA_ERR_TIMEOUT, K_INDEXER_TC, blockIdx.x, 3);
                ok = false;
                break;
            }
#pragma unroll
            for (int x = 0; x < RPT; x++) {
                const int r = row_of(x);
                const uint32_t ex = exc[x];
                const uint32_t em = max(max(ex & 255u, (ex >> 8) & 255u),
                                        max((ex >> 16) & 255u, ex >> 24));
                const uint8_t *src = sR + (size_t)st * 8192 + r * 64;
                uint8_t *dst = sA + (size_t)st * 16384 + r * 128;
#pragma unroll
                for (int q = 0; q < BPT; q++) {
                    // rotated by row: spreads the banks
                    const int blk = (ut % TPR) * BPT + ((q + (r >> 1)) & (BPT - 1));
                    const uint4 w = *(const uint4 *)(src + blk * 16);
                    int j = (int)(em - ((ex >> (8 * blk)) & 255u));
                    j = j > 8 ? 8 : j;
                    const uint32_t t0 = lut[2 * j], t1 = lut[2 * j + 1];
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                    uint32_t o[8];
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        // word u: channels 8u .. 8u + 7 of the block, channel
                        // 2c in the low nibble of byte c
                        const uint32_t x = wv[u], xs = x << 4;
                        const uint32_t m0 = prmt(t0, t1, x & 0x7777u);
                        const uint32_t m1 = prmt(t0, t1, (x >> 16) & 0x7777u);
                        // sign of channel 2c: top bit of byte c of x << 4;
                        // of channel 2c + 1: top bit of byte c of x (the
                        // selector's bit 3 replicates that bit over the byte)
                        const uint32_t s0 = prmt(xs, x, 0xD9C8u) & 0x80808080u;
                        const uint32_t s1 = prmt(xs, x, 0xFBEAu) & 0x80808080u;
                        o[2 * u] = m0 | s0;
                        o[2 * u + 1] = m1 | s1;
                    }
                    // channels 32 blk .. 32 blk + 31: 16-byte chunks 2 blk and
                    // 2 blk + 1 of the row, at chunk ^ (row % 8)
                    *(uint4 *)(dst + (((2 * blk) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *(uint4 *)(dst + (((2 * blk + 1) ^ (r & 7)) << 4)) =
                        make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
            // the tile's generic writes become visible to the tensor core
            tc::fence_async_shared();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&full[st]);
                tc::mbar_arrive(&rempty[st]);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <bool FP8, int HI, int NT, int NSUB, bool FUSE, bool K4>
cudaError_t launch_one(const IndexerArgs &a, const IndexerTcExtra &x, unsigned *err, cudaStream_t s)
{
    using C = Cfg<FP8, HI, NT, NSUB, K4>;
    const int esize = FP8 ? 1 : 2;
    TcArgs t;
    t.wI = a.wI;
    t.qI_scale = a.qI_scale;
    t.kI_scale = K4 ? nullptr : a.kI.scale;
    t.kI_exp = K4 ? (const uint8_t *)a.kI.scale : nullptr;
    t.q_pos = a.q_pos;
    t.n_q = a.n_q;
    t.E = a.E;
    t.m = a.m;
    t.kb = a.cI * esize / 128;
    const int64_t ttiles = (a.n_q + C::TT - 1) / C::TT;
    // few token tiles: split the keys of each tile over several blocks, sized
    // so that all blocks run in one wave (two resident blocks per SM)
    int dev = 0, sms = 148, nsm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
        sms = nsm;
    const int64_t target = 2 * (int64_t)sms;
    t.key_chunk = a.E;
    t.nchunks = 1;
    if (ttiles * a.B < target) {
        const int64_t want = (target + ttiles * a.B - 1) / (ttiles * a.B);
        const int64_t per = (a.E + want - 1) / want;
        t.key_chunk = (per + 127) / 128 * 128;
        t.nchunks = (int)((a.E + t.key_chunk - 1) / t.key_chunk);
    }
    t.scores = a.scores;
    t.ld = a.ld;
    t.ks_stride = x.key_step;
    t.row_flag = x.row_flag;
    t.bound = x.bound;
    t.k = x.k;
    t.cand = (uint2 *)a.scores;
    t.cand_ld = a.ld / 2;
    t.cnt = x.cnt;
    t.err = err;
    if (x.nchunks_out)
        *x.nchunks_out = t.nchunks;
    if (x.lists_out)
        *x.lists_out = 4 * C::NSET;
    if (x.key_chunk_out)
        *x.key_chunk_out = t.key_chunk;
    if (x.plan_only)
        return cudaSuccess;
    CUtensorMap tmk, tmq;
    const CUtensorMapDataType dt =
        FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // key s of the table is row s * key_step of kI.body (FP4: packed rows
    // of c_I / 2 bytes, unswizzled)
    const bool km = K4 ? make_tmap_bytes(&tmk, a.kI.body, (uint64_t)a.B * a.E, (uint64_t)a.cI / 2,
                                         (uint64_t)x.key_step * a.cI / 2, 128, a.cI / 2)
                       : make_tmap_2d(&tmk, a.kI.body, dt, esize, (uint64_t)a.B * a.E, a.cI, 128,
                                      (uint64_t)x.key_step * a.cI * esize);
    if (!km || !make_tmap_2d(&tmq, a.qI, dt, esize, (uint64_t)a.B * a.n_q * HI, a.cI,
                             C::QROWS < 256 ? C::QROWS : 256))
        return cudaErrorInvalidValue;
    const size_t smem = C::smem_bytes(t.kb);
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<FP8, HI, NT, NSUB, FUSE, K4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid((unsigned)(ttiles * t.nchunks), (unsigned)a.B);
    indexer_tc_kernel<FP8, HI, NT, NSUB, FUSE, K4><<<grid, C::THREADS, smem, s>>>(tmk, tmq, t);
    return cudaGetLastError();
}

template <bool FP8, int HI, int NT, int NSUB>
cudaError_t launch_mode(const IndexerArgs &a, const IndexerTcExtra &x, unsigned *err,
                        cudaStream_t s)
{
    if constexpr (FP8) {
        if (a.kI.dt == CSA_E2M1)
            return x.fuse ? launch_one<FP8, HI, NT, NSUB, true, true>(a, x, err, s)
                          : launch_one<FP8, HI, NT, NSUB, false, true>(a, x, err, s);
    }
    return x.fuse ? launch_one<FP8, HI, NT, NSUB, true, false>(a, x, err, s)
                  : launch_one<FP8, HI, NT, NSUB, false, false>(a, x, err, s);
}

template <bool FP8>
cudaError_t dispatch_heads(const IndexerArgs &a, const IndexerTcExtra &x, unsigned *err,
                           cudaStream_t s, bool few)
{
    // prefill: a block takes 16 tokens (e4m3) or one group of N = 256 (bf16,
    // whose key tiles are twice the size); decode: one token per block
    switch (a.hI) {
    case 16:
        return few ? launch_mode<FP8, 16, 1, 1>(a, x, err, s)
                   : launch_mode<FP8, 16, 16, 1>(a, x, err, s);
    case 32:
        if (few)
            return launch_mode<FP8, 32, 1, 1>(a, x, err, s);
        if constexpr (FP8)
            return launch_mode<FP8, 32, 8, 2>(a, x, err, s);
        else
            return launch_mode<FP8, 32, 8, 1>(a, x, err, s);
    case 64:
        if (few)
            return launch_mode<FP8, 64, 1, 1>(a, x, err, s);
        if constexpr (FP8)
            return launch_mode<FP8, 64, 4, 4>(a, x, err, s);
        else
            return launch_mode<FP8, 64, 4, 1>(a, x, err, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool indexer_tc_takes(const IndexerArgs &a)
{
    if (a.dt == CSA_F32)
        return false;
    // FP4 keys: e4m3 queries, c_I = 128 (64-byte packed rows)
    if (a.kI.dt == CSA_E2M1 && (a.dt != CSA_E4M3 || a.cI != 128))
        return false;
    if (a.hI != 16 && a.hI != 32 && a.hI != 64)
        return false;
    const int esize = a.dt == CSA_E4M3 ? 1 : 2;
    if ((a.cI * esize) % 128 != 0 || a.cI * esize > 256)
        return false;
    return ((uintptr_t)a.qI & 15) == 0 && ((uintptr_t)a.kI.body & 15) == 0;
}

cudaError_t launch_indexer_tc_ex(const IndexerArgs &a, const IndexerTcExtra &x, unsigned *err,
                                 cudaStream_t s)
{
    const bool few = a.n_q <= 8;
    return a.dt == CSA_E4M3 ? dispatch_heads<true>(a, x, err, s, few)
                            : dispatch_heads<false>(a, x, err, s, few);
}

cudaError_t launch_indexer_tc(const IndexerArgs &a, unsigned *err, cudaStream_t s, bool *taken)
{
    *taken = indexer_tc_takes(a);
    if (!*taken)
        return cudaSuccess;
    return launch_indexer_tc_ex(a, IndexerTcExtra{}, err, s);
}

}  // namespace csa
