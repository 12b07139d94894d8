/*
 * csa_oracle.c -- plain, slow, float64 CPU restatement of the CSA / HCA path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or load
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header or constant table with the CUDA
 * library.
 *
 * Source of each step (DeepSeek-V4 technical report as restated on the web
 * pages "DeepSeek-V4: Towards Highly Efficient Million-Token Context
 * Intelligence" (ai-papers-daily notes) and "DeepSeek V4 大模型算法解析"):
 *   compression ............ Module B step 1, Eq. 9-12 (overlapping windows:
 *                            C^a rows mi..m(i+1)-1, C^b rows m(i-1)..mi-1,
 *                            softmax over the 2m logits Z + B, per channel)
 *   HCA compression ........ Module C, Eq. 20-23 (m' rows, no overlap)
 *   indexer score .......... Module B step 2, Eq. 16
 *   top-k selection ........ Module B step 2, Eq. 17
 *   shared-KV attention .... Module B step 3, Eq. 18-19, with the sliding
 *                            window branch and the attention sink of Module D
 *   low-precision storage .. Module F (fp8 body, bf16 RoPE dims; FP4
 *                            indexer keys)
 * Readings where the pages are silent are listed beside each function.
 *
 * Every function takes inputs already decoded exactly to double and computes
 * in double with plain loops, in the order the equations state.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Compressed entries visible to the query at absolute position t: entry i
 * covers tokens m*i .. m*i+m-1 and is visible once its last token is at or
 * before t (only earlier compressed blocks, Module D "sliding window"; a
 * block that the query itself completes counts as earlier). */
int64_t oracle_visible(int64_t t, int m, int64_t E)
{
    int64_t v = (t + 1) / m;
    return v < E ? v : E;
}

/* ---------------------------------------------------------------- e4m3 --- */

/* Value of an e4m3 code: sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent 0 is subnormal (mantissa/8 * 2^-6); 0x7F / 0xFF are NaN. */
double oracle_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, f = code & 7;
    double v;
    if (e == 15 && f == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)f / 8.0, -6);
    else
        v = ldexp(1.0 + (double)f / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest e4m3 code to x (finite), ties to the even code, values beyond the
 * largest finite magnitude (448) saturate to it. */
uint8_t oracle_e4m3_code(double x)
{
    uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? 0x80 : 0;
    double a = fabs(x);
    int lo = 0, hi = 0x7E;                 /* magnitudes increase with code */
    if (a >= oracle_e4m3_value(0x7E))
        return sign | 0x7E;
    while (hi - lo > 1) {                  /* value(lo) <= a < value(hi) */
        int mid = (lo + hi) / 2;
        if (oracle_e4m3_value((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dl = a - oracle_e4m3_value((uint8_t)lo);
    double dh = oracle_e4m3_value((uint8_t)hi) - a;
    int code = (dl < dh) ? lo : (dh < dl) ? hi : ((lo & 1) ? hi : lo);
    return (uint8_t)(sign | code);
}

/* fp8 storage of rows of compressed entries (Module F). Reading adopted for
 * the unstated quantiser: per group of `group` channels the float32 values
 * x are scaled by s = max(amax / 448, 2^-126) (float32 arithmetic, the
 * precision the stored scale has) and rounded to the nearest code. */
void oracle_quantize_e4m3(const double *x, int64_t rows, int cols, int group,
                          uint8_t *codes, float *scales)
{
    int groups = cols / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int g = 0; g < groups; g++) {
            float amax = 0.0f;
            for (int j = 0; j < group; j++) {
                float v = (float)x[r * cols + g * group + j];
                if (fabsf(v) > amax)
                    amax = fabsf(v);
            }
            float s = amax / 448.0f;
            if (s < FLT_MIN)
                s = FLT_MIN;
            scales[r * groups + g] = s;
            for (int j = 0; j < group; j++) {
                float v = (float)x[r * cols + g * group + j];
                float y = v / s;
                codes[r * cols + g * group + j] = oracle_e4m3_code((double)y);
            }
        }
    }
}

/* Stored value of an fp8 entry: code value times its group's scale. */
void oracle_dequantize(const uint8_t *codes, const float *scales, int64_t rows,
                       int cols, int group, double *out)
{
    int groups = cols / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int j = 0; j < cols; j++)
            out[r * cols + j] = oracle_e4m3_value(codes[r * cols + j]) *
                                (double)scales[r * groups + j / group];
}

/* ------------------------------------------------- fp4 indexer keys --- */

/* Value of a 4-bit e2m1 code (1 sign bit, 2 exponent bits with bias 1, 1
 * mantissa bit; no infinities or NaN): the FP4 of the indexer path (Module F:
 * "the indexer's QK path runs in FP4"). Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, f = code & 1;
    double v = e == 0 ? 0.5 * f : ldexp(1.0 + 0.5 * f, e - 1);
    return s ? -v : v;
}

/* Nearest e2m1 code to x, ties to the code with the even (zero) mantissa
 * bit, magnitudes beyond 6 saturate to 6; the sign bit is the sign of x. */
uint8_t oracle_e2m1_code(double x)
{
    uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? 8 : 0;
    double a = fabs(x);
    if (a >= 6.0)
        return sign | 7;
    int lo = 0, hi = 7;                   /* magnitudes increase with code */
    while (hi - lo > 1) {                 /* value(lo) <= a < value(hi) */
        int mid = (lo + hi) / 2;
        if (oracle_e2m1_value((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dl = a - oracle_e2m1_value((uint8_t)lo);
    double dh = oracle_e2m1_value((uint8_t)hi) - a;
    int code = (dl < dh) ? lo : (dh < dl) ? hi : ((lo & 1) ? hi : lo);
    return (uint8_t)(sign | code);
}

/* FP4 storage of indexer-key rows. Readings adopted for what the pages leave
 * open (they name FP4 only):
 *  - blocks of 32 consecutive channels share a power-of-two scale 2^E, the
 *    smallest one with 6 * 2^E >= the block's largest magnitude (so no value
 *    saturates), taken on the float32 values;
 *  - within a row the block exponents span at most 8 binades (a block whose
 *    exponent would be lower takes max_E - 8), so that a row can be brought
 *    to one scale exactly in 8-bit floats;
 *  - an all-zero block takes the row's lowest allowed exponent; an all-zero
 *    row takes exponent 0;
 *  - codes are the nearest e2m1 values of x / 2^E (float32 quotient).
 * Layout: packed[r][j / 2] holds channel j in its low nibble when j is even,
 * in its high nibble when odd; exps[r][b] = E_b + 127 (the block scale is
 * 2^(exps - 127)). cols must be a multiple of 32. */
void oracle_quantize_e2m1(const double *x, int64_t rows, int cols, uint8_t *packed,
                          uint8_t *exps)
{
    int blocks = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        int E[64];
        int any = 0, emax = -100000;
        for (int b = 0; b < blocks; b++) {
            float amax = 0.0f;
            for (int j = 0; j < 32; j++) {
                float v = (float)x[r * cols + b * 32 + j];
                if (fabsf(v) > amax)
                    amax = fabsf(v);
            }
            if (amax > 0.0f) {
                int e = -160;                       /* smallest e: 6 * 2^e >= amax */
                while (ldexp(6.0, e) < (double)amax)
                    e++;
                while (ldexp(6.0, e - 1) >= (double)amax)
                    e--;
                E[b] = e;
                any = 1;
                if (e > emax)
                    emax = e;
            } else {
                E[b] = -100000;
            }
        }
        for (int b = 0; b < blocks; b++) {
            int e = any ? (E[b] < emax - 8 ? emax - 8 : E[b]) : 0;
            exps[r * blocks + b] = (uint8_t)(e + 127);
            for (int j = 0; j < 32; j++) {
                int ch = b * 32 + j;
                float v = (float)x[r * cols + ch];
                float y = ldexpf(v, -e);
                uint8_t q = oracle_e2m1_code((double)y);
                uint8_t *dst = &packed[r * (cols / 2) + ch / 2];
                if (ch & 1)
                    *dst = (uint8_t)((*dst & 0x0F) | (q << 4));
                else
                    *dst = (uint8_t)((*dst & 0xF0) | q);
            }
        }
    }
}

/* Stored value of an FP4 key channel: its code's value times its block's
 * scale 2^(exps - 127). */
void oracle_dequantize_e2m1(const uint8_t *packed, const uint8_t *exps, int64_t rows, int cols,
                            double *out)
{
    int blocks = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int j = 0; j < cols; j++) {
            uint8_t byte = packed[r * (cols / 2) + j / 2];
            uint8_t q = (j & 1) ? (byte >> 4) : (byte & 15);
            out[r * cols + j] =
                ldexp(oracle_e2m1_value(q), (int)exps[r * blocks + j / 32] - 127);
        }
}

/* --------------------------------------------------------- compression --- */

/* Eq. 9-12 (overlap = 1) and Eq. 20-23 (overlap = 0, C = Ca, Z = Za, B = Ba).
 * For entry i and channel j the logits are Za[m*i + r][j] + Ba[r][j] and,
 * with overlap, Zb[m*(i-1) + r][j] + Bb[r][j] for r < m; a softmax over those
 * (per channel, over token positions) weights the matching rows of Ca / Cb.
 * Entry 0 has no previous block: its b-half is left out of the softmax. */
void oracle_compress(const double *Ca, const double *Cb, const double *Za,
                     const double *Zb, const double *Ba, const double *Bb,
                     int64_t n, int c, int m, int overlap, double *out)
{
    int64_t E = n / m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < E; i++) {
        int with_b = overlap && i > 0;
        for (int j = 0; j < c; j++) {
            double mx = -INFINITY;
            for (int r = 0; r < m; r++) {
                double la = Za[(m * i + r) * c + j] + Ba[r * c + j];
                if (la > mx)
                    mx = la;
                if (with_b) {
                    double lb = Zb[(m * (i - 1) + r) * c + j] + Bb[r * c + j];
                    if (lb > mx)
                        mx = lb;
                }
            }
            double den = 0.0, num = 0.0;
            for (int r = 0; r < m; r++) {
                double ea = exp(Za[(m * i + r) * c + j] + Ba[r * c + j] - mx);
                den += ea;
                num += ea * Ca[(m * i + r) * c + j];
                if (with_b) {
                    double eb = exp(Zb[(m * (i - 1) + r) * c + j] + Bb[r * c + j] - mx);
                    den += eb;
                    num += eb * Cb[(m * (i - 1) + r) * c + j];
                }
            }
            out[i * c + j] = num / den;
        }
    }
}

/* ------------------------------------------------------------- indexer --- */

/* Eq. 16: I[t][s] = sum_h wI[t][h] * max(0, qI[t][h] . kI[s]) for the
 * compressed entries visible to t; invisible entries get -inf. No scale and
 * no softmax. Batches b have their own keys kI[b] and queries. */
void oracle_indexer(const double *qI, const double *wI, const double *kI,
                    const int64_t *q_pos, int B, int64_t nq, int64_t E, int hI,
                    int cI, int m, double *scores)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t bt = 0; bt < (int64_t)B * nq; bt++) {
        int64_t b = bt / nq;
        int64_t V = oracle_visible(q_pos[bt], m, E);
        const double *q = qI + bt * hI * cI;
        for (int64_t s = 0; s < E; s++) {
            double acc = -INFINITY;
            if (s < V) {
                const double *k = kI + (b * E + s) * cI;
                acc = 0.0;
                for (int hh = 0; hh < hI; hh++) {
                    double dot = 0.0;
                    for (int x = 0; x < cI; x++)
                        dot += q[hh * cI + x] * k[x];
                    acc += wI[bt * hI + hh] * (dot > 0.0 ? dot : 0.0);
                }
            }
            scores[bt * E + s] = acc;
        }
    }
}

/* --------------------------------------------------------------- top-k --- */

typedef struct {
    double v;
    int32_t i;
} oracle_item;

static int by_score_then_index(const void *pa, const void *pb)
{
    const oracle_item *a = (const oracle_item *)pa, *b = (const oracle_item *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int ascending_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Eq. 17: the min(k, V) visible entries with the largest scores. Readings:
 * equal scores prefer the lower index (+0 and -0 are equal); the row lists
 * the chosen indices in ascending order, then -1 up to k. */
void oracle_topk(const double *scores, int64_t rows, int64_t E, int64_t ld,
                 const int64_t *q_pos, int m, int k, int32_t *idx)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < rows; r++) {
        int64_t V = oracle_visible(q_pos[r], m, E);
        oracle_item *it = (oracle_item *)malloc(sizeof(oracle_item) * (V > 0 ? V : 1));
        for (int64_t s = 0; s < V; s++) {
            it[s].v = scores[r * ld + s] + 0.0;   /* -0 -> +0 */
            it[s].i = (int32_t)s;
        }
        qsort(it, (size_t)V, sizeof(oracle_item), by_score_then_index);
        int64_t take = V < k ? V : k;
        int32_t *row = idx + r * k;
        for (int64_t j = 0; j < take; j++)
            row[j] = it[j].i;
        qsort(row, (size_t)take, sizeof(int32_t), ascending_int);
        for (int64_t j = take; j < k; j++)
            row[j] = -1;
        free(it);
    }
}

/* ----------------------------------------------------------- attention --- */

/* Eq. 18-19 with the window branch and the sink (Module D): every key is
 * also its own value. For query (b, t) the keys are
 *   - the selected entries entries[b][idx[bt][j]] (idx >= 0), or, when
 *     idx == NULL (HCA, Eq. 24-26), every visible entry s < V_t;
 *   - the raw window rows for positions max(0, t - n_win + 1) .. t, read
 *     from kwin[b][p - win_pos0[b]].
 * z_j = scale * q . key_j,  M = max(max_j z_j, z'_h),
 * o = sum_j e^{z_j - M} key_j / (sum_j e^{z_j - M} + e^{z'_h - M}),
 * lse = M + log(denominator). A sink of +inf gives o = 0; an empty key set
 * with a sink of -inf gives o = 0 and lse = -inf.
 * Returns 0, or -1 if an index or a window position is out of range. */
int oracle_attend(const double *q, const double *entries, int64_t E,
                  const int32_t *idx, int k, int m, const double *kwin,
                  int64_t wrows, const int64_t *win_pos0, int n_win,
                  const int64_t *q_pos, const double *sink, int B, int64_t nq,
                  int h, int c, double scale, double *out, double *lse)
{
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t bt = 0; bt < (int64_t)B * nq; bt++) {
        int64_t b = bt / nq, t = q_pos[bt];
        int64_t V = oracle_visible(t, m, E);
        int64_t nsel = idx ? k : V;
        int64_t w0 = t - n_win + 1 < 0 ? 0 : t - n_win + 1;
        int64_t nwin = n_win > 0 ? t - w0 + 1 : 0;
        const double **keys = (const double **)malloc(sizeof(double *) * (nsel + nwin + 1));
        double *z = (double *)malloc(sizeof(double) * (nsel + nwin + 1));
        int64_t nk = 0;
        for (int64_t j = 0; j < nsel; j++) {
            int64_t s = idx ? idx[bt * k + j] : j;
            if (s < 0)
                continue;
            if (s >= V) {
                bad = 1;
                continue;
            }
            keys[nk++] = entries + (b * E + s) * c;
        }
        for (int64_t p = w0; p < w0 + nwin; p++) {
            int64_t row = p - win_pos0[b];
            if (row < 0 || row >= wrows) {
                bad = 1;
                continue;
            }
            keys[nk++] = kwin + (b * wrows + row) * c;
        }
        for (int hh = 0; hh < h; hh++) {
            const double *qv = q + (bt * h + hh) * c;
            double *o = out + (bt * h + hh) * c;
            double zs = sink[hh], mx = zs;
            for (int64_t j = 0; j < nk; j++) {
                double d = 0.0;
                for (int x = 0; x < c; x++)
                    d += qv[x] * keys[j][x];
                z[j] = scale * d;
                if (z[j] > mx)
                    mx = z[j];
            }
            for (int x = 0; x < c; x++)
                o[x] = 0.0;
            if (zs == INFINITY) {
                lse[bt * h + hh] = INFINITY;
                continue;
            }
            if (mx == -INFINITY) {                 /* no keys, sink -inf */
                lse[bt * h + hh] = -INFINITY;
                continue;
            }
            double den = exp(zs - mx);
            for (int64_t j = 0; j < nk; j++) {
                double p = exp(z[j] - mx);
                den += p;
                for (int x = 0; x < c; x++)
                    o[x] += p * keys[j][x];
            }
            for (int x = 0; x < c; x++)
                o[x] /= den;
            lse[bt * h + hh] = mx + log(den);
        }
        free(keys);
        free(z);
    }
    return bad ? -1 : 0;
}

/* RMSNorm of one head vector, then partial RoPE on its last R dims (Module D:
 * "Q/KV normalisation" and "partial RoPE"). In place on rows x heads vectors
 * of c values:
 *   x <- x / sqrt(mean_j x_j^2 + eps) * gamma          (gamma [c], or NULL: 1)
 *   for pair p = 0 .. R/2-1 of the last R dims, at position pos[row]:
 *     phi = pos * base^(-2p/R),
 *     (a, b) <- (a cos phi - b sin phi, a sin phi + b cos phi)
 * Readings (the pages are silent): the RoFormer pairing of adjacent dims
 * (c-R+2p, c-R+2p+1); frequencies base^(-2p/R) over the rotated dims only;
 * normalise = 0 skips the RMSNorm (rotation alone). */
void oracle_norm_rope(double *x, int64_t rows, int heads, int c, int R, const int64_t *pos,
                      const double *gamma, int normalise, double eps, double base)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int h = 0; h < heads; h++) {
            double *v = x + (r * heads + h) * (int64_t)c;
            if (normalise) {
                double ss = 0.0;
                for (int j = 0; j < c; j++)
                    ss += v[j] * v[j];
                const double inv = 1.0 / sqrt(ss / c + eps);
                for (int j = 0; j < c; j++)
                    v[j] = v[j] * inv * (gamma ? gamma[j] : 1.0);
            }
            for (int p = 0; p < R / 2; p++) {
                const double phi = (double)pos[r] * pow(base, -2.0 * p / R);
                const double cs = cos(phi), sn = sin(phi);
                double *a = v + (c - R) + 2 * p;
                const double a0 = a[0], a1 = a[1];
                a[0] = a0 * cs - a1 * sn;
                a[1] = a0 * sn + a1 * cs;
            }
        }
    }
}
