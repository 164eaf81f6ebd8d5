/*
 * dq_oracle.c -- plain, slow CPU reference for row-wise INT4 quantization and the
 * INT4 embedding bag.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU
 * baseline may load this file's library. It shares no code, header, table or
 * constant with the CUDA path, and it includes nothing from it.
 *
 * What it computes follows "Post-Training 4-bit Quantization on Embedding Tables"
 * (Guan et al., 2019), review page, section 提出的方法 (proposed method): one uniform
 * 4-bit quantizer per embedding row, its clipping range found by a greedy search
 * that walks toward a local minimum of the squared error (bullet 1), and scale
 * and bias stored as FP16 (bullet 2; section 主要发现 / main findings, bullet 4).
 * The lookup is the sum-pooled embedding bag of "Deep Learning Recommendation
 * Model for Personalization and Recommendation Systems", section 提出的方法
 * (proposed method), bullet 1.
 *
 * The pages leave the details open. This library fixes them as follows, and the
 * oracle takes the steps in this order:
 *
 *   fl(.) is one IEEE binary32 operation rounded to nearest even; fma(a,b,c)
 *   rounds a*b+c once. h(.) is binary32 -> binary16 rounding to nearest even
 *   (subnormals kept, overflow to infinity); w(.) widens binary16 exactly.
 *
 *   Row x[0..d-1]:
 *   1. xmin = min x, xmax = max x, R = fl(xmax - xmin), step = fl(R / 200).
 *   2. Grid points lo(i) = fma(i, step, xmin), hi(j) = fma(-j, step, xmax).
 *   3. Loss L(i,j): s = fl(fl(hi - lo) / 15); for each k:
 *        q = clamp(rint(fl(fl(x_k - lo) / s)), 0, 15)   (q = 0 when s == 0)
 *        xhat = fma(q, s, lo), e = fl(x_k - xhat), c_k = fl(e * e);
 *      L = pairwise sum of c_0..c_{d-1} padded with +0 to the next power of two
 *      (sum(a[0:n]) = fl(sum(a[0:n/2]) + sum(a[n/2:n]))).
 *   4. Start at (i, j) = (0, 0) with best = (0, 0), Lbest = L(0, 0).
 *   5. While the clip width (200 - i - j) * step exceeds 0.16 * R, i.e. while
 *      i + j < 168: Ll = L(i+1, j), Lr = L(i, j+1); move right (j+1) if Lr < Ll,
 *      else left (i+1); if the new loss < Lbest, remember it. Exactly 168 moves.
 *   6. scale16 = h(fl(fl(hi* - lo*) / 15)), bias16 = h(lo*), S = w(scale16),
 *      B = w(bias16), q_k = clamp(rint(fl(fl(x_k - B) / S)), 0, 15) (0 when S == 0).
 *   7. Byte m of the code row = q_{2m} | q_{2m+1} << 4; odd d leaves the last high
 *      nibble 0. The plain min/max quantizer is step 5 skipped.
 *
 *   Dequantize: xhat_k = fma(q_k, S, B).
 *   Normalized l2 error of a row (the quality measure of "Post-Training 4-bit
 *   Quantization on Embedding Tables", 提出的方法 bullet 5; the pages do not define it,
 *   the reading taken is): sqrt(sum_k (x_k - xhat_k)^2) / sqrt(sum_k x_k^2), both sums
 *   in binary64 over the binary64 values of the binary32 x and xhat, in index order;
 *   a row with sum x^2 = 0 has error 0 if it is reconstructed exactly, else +inf.
 *   Embedding bag: out[b][t*d + k] = sum over the bag's ids p of xhat_{p,k}, summed
 *   in binary64 in index order and rounded once to binary32; an empty bag gives +0.
 *   Bag backward, SGD step and re-quantization of the touched rows (the training
 *   step of the DQRM repository page: embeddings trained at INT4 with quantization-
 *   aware training on binary32 masters; the pages fix no arithmetic for it, the
 *   reading taken is):
 *   a. Offsets must be a CSR array: offsets[0] = 0, nondecreasing, offsets[T*B] =
 *      the number of indices; otherwise nothing changes. Every position p of bag
 *      (t, b) with a valid id gives an entry (key = row_base[t] + id, p), row_base[t]
 *      = rows of the tables before t. Invalid ids give no entry.
 *   b. The entries are sorted by (key, p), so each row's entries are together, in
 *      the order of their positions in `indices`.
 *   c. Gradient of a row, element k: the plain binary64 sum, from +0, of
 *      g[b][t*d + k] over the row's entries in that order (one addition after the
 *      other), rounded once to binary32 (G_k). Any order gives a valid sum; this is
 *      the plainest one, and the CUDA path is compared with it within a stated
 *      tolerance rather than required to share its order.
 *   d. W[id][k] = fma(-lr, G_k, W[id][k]) (binary32, rounded once).
 *   e. Each touched row (one with at least one entry) is quantized again from its new
 *      master values by the quantizer above (greedy or min/max); other rows keep
 *      their codes.
 *   Codebook quantizer ("Post-Training 4-bit Quantization on Embedding Tables",
 *   提出的方法 bullet 3: codebook quantization by k-means, values mapped to a
 *   non-uniform set; 主要发现 bullet 3: the 18.8%-37.5% sizes fit 16 binary16 centroids
 *   per row). The pages fix no initialisation, iteration count or precision; the
 *   reading taken is one-dimensional Lloyd iterations in binary32:
 *   K1. c_j = fma(j, fl(R / 15), xmin), j = 0..15 (the min/max quantizer's levels).
 *   K2. `iters` times: a_k = the j minimising fl(|fl(x_k - c_j)|), ties to the lower j;
 *       then for every j with n_j > 0 members, c_j = the mean of its members: their
 *       values summed in binary64 from +0 in index order (one addition after the
 *       other), divided by n_j in binary64, the quotient rounded once to binary32; an
 *       empty cluster keeps its centroid. (The pages name the mean and no order; this
 *       is the plainest order, and where every partial sum is exact in binary64, as
 *       for most rows, the sum is the exact one and no order can change it.)
 *   K3. Stored centroids C_j = h(c_j); codes q_k = the j minimising fl(|fl(x_k - w(C_j))|),
 *       ties to the lower j; packed as above. Row loss: the pairwise sum of
 *       fl(fl(x_k - w(C_{q_k}))^2).
 *   Dequantize: w(C_{q_k}); the codebook bag sums those values like the bag above.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread
 * (no FMA contraction and no excess precision, so every C operator below is one
 * IEEE binary32 operation; fmaf() is the C library's correctly rounded FMA).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_GRID_STEPS 200.0f
#define ORACLE_MOVES 168          /* 200 - 0.16 * 200 */
#define ORACLE_LEVELS 15.0f       /* 2^4 - 1 */
#define ORACLE_MAX_D 1024

enum { ORACLE_GREEDY = 0, ORACLE_MINMAX = 1 };

/* ------------------------------------------------------------------------ */
/* binary16 conversions                                                     */
/* ------------------------------------------------------------------------ */

/* binary32 -> binary16, round to nearest, ties to even. The result's quantum is
 * 2^qe with qe = max(exponent - 10, -24); the significand is shifted right by the
 * difference of quanta and rounded on the dropped bits. A carry out of the
 * significand moves into the exponent field by itself, up to infinity. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    int ef = (int)((u >> 23) & 0xffu);
    uint32_t man = u & 0x7fffffu;
    if (ef == 0xff)                               /* infinity or NaN */
        return man ? (uint16_t)(sign | 0x7e00u | (man >> 13)) : (uint16_t)(sign | 0x7c00u);
    if (ef == 0)                                  /* |f| < 2^-126: rounds to zero */
        return sign;
    uint32_t m = man | 0x800000u;                 /* value = m * 2^(ef - 150) */
    int qe = ef - 127 - 10;                       /* quantum exponent of the result */
    if (qe < -24)
        qe = -24;
    int eh = qe + 25;                             /* biased binary16 exponent */
    if (eh > 30)
        return (uint16_t)(sign | 0x7c00u);
    int drop = qe - (ef - 150);                   /* >= 13 */
    uint32_t r = 0;
    if (drop < 25) {
        uint32_t rem = m & ((1u << drop) - 1u), half = 1u << (drop - 1);
        r = m >> drop;
        if (rem > half || (rem == half && (r & 1u)))
            r++;
    }
    return (uint16_t)(sign | (uint32_t)(((eh - 1) << 10) + (int)r));
}

/* binary16 -> binary32 (exact). */
float oracle_f16_to_f32(uint16_t h)
{
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    float v;
    if (e == 0x1f)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexpf((float)m, -24);
    else
        v = ldexpf((float)(1024 + m), e - 25);
    return (h & 0x8000) ? -v : v;
}

/* Element-wise conversion of n values (for the exhaustive checks). */
void oracle_f32_to_f16_array(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_f32_to_f16(in[i]);
}

void oracle_f16_to_f32_array(const uint16_t *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_f16_to_f32(in[i]);
}

/* ------------------------------------------------------------------------ */
/* the loss of one clip range                                               */
/* ------------------------------------------------------------------------ */

static int next_pow2(int d)
{
    int p = 1;
    while (p < d)
        p <<= 1;
    return p;
}

/* q = clamp(rint(fl(fl(x - lo) / s)), 0, 15); 0 when s == 0. rint rounds half to even. */
static float code_of(float x, float lo, float s)
{
    if (s == 0.0f)
        return 0.0f;
    float t = x - lo;
    float y = t / s;
    float q = nearbyintf(y);
    if (!(q > 0.0f))
        q = 0.0f;
    if (q > ORACLE_LEVELS)
        q = ORACLE_LEVELS;
    return q;
}

static float pairwise_sum(const float *c, int n)
{
    if (n == 1)
        return c[0];
    return pairwise_sum(c, n / 2) + pairwise_sum(c + n / 2, n / 2);
}

/* L for the clip range [lo, hi]; cbuf holds next_pow2(d) floats. */
static float loss_of(const float *x, int d, float lo, float hi, float *cbuf)
{
    float s = (hi - lo) / ORACLE_LEVELS;
    int p = next_pow2(d);
    for (int k = 0; k < d; k++) {
        float q = code_of(x[k], lo, s);
        float xhat = fmaf(q, s, lo);
        float e = x[k] - xhat;
        cbuf[k] = e * e;
    }
    for (int k = d; k < p; k++)
        cbuf[k] = 0.0f;
    return pairwise_sum(cbuf, p);
}

float oracle_row_loss(const float *x, int32_t d, float lo, float hi)
{
    float cbuf[ORACLE_MAX_D];
    if (d < 1 || d > ORACLE_MAX_D)
        return NAN;
    return loss_of(x, d, lo, hi, cbuf);
}

/* ------------------------------------------------------------------------ */
/* the greedy search of one row                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    float xmin, xmax, step;
    int bi, bj;
    float lbest;
} search_result;

static float grid_lo(float xmin, float step, int i) { return fmaf((float)i, step, xmin); }
static float grid_hi(float xmax, float step, int j) { return fmaf(-(float)j, step, xmax); }

/* Runs steps 1-5. When trace_* are given, records every evaluation in order
 * (eval 0 = (0,0); move m evaluates 2m+1 = (i+1, j) and 2m+2 = (i, j+1)) and the
 * position after every move. */
static search_result search_row(const float *x, int d, int mode, float *cbuf,
                                float *trace_lo, float *trace_hi, float *trace_loss,
                                int32_t *trace_i, int32_t *trace_j)
{
    search_result r;
    float xmin = x[0], xmax = x[0];
    for (int k = 1; k < d; k++) {
        if (x[k] < xmin)
            xmin = x[k];
        if (x[k] > xmax)
            xmax = x[k];
    }
    float range = xmax - xmin;
    float step = range / ORACLE_GRID_STEPS;
    r.xmin = xmin;
    r.xmax = xmax;
    r.step = step;
    r.bi = r.bj = 0;
    r.lbest = loss_of(x, d, xmin, xmax, cbuf);
    if (trace_loss) {
        trace_lo[0] = xmin;
        trace_hi[0] = xmax;
        trace_loss[0] = r.lbest;
    }
    if (mode != ORACLE_GREEDY)
        return r;
    int i = 0, j = 0;
    for (int mv = 0; i + j < ORACLE_MOVES; mv++) {
        float lo_l = grid_lo(xmin, step, i + 1), hi_l = grid_hi(xmax, step, j);
        float lo_r = grid_lo(xmin, step, i), hi_r = grid_hi(xmax, step, j + 1);
        float ll = loss_of(x, d, lo_l, hi_l, cbuf);
        float lr = loss_of(x, d, lo_r, hi_r, cbuf);
        float l;
        if (lr < ll) {
            j++;
            l = lr;
        } else {
            i++;
            l = ll;
        }
        if (l < r.lbest) {
            r.lbest = l;
            r.bi = i;
            r.bj = j;
        }
        if (trace_loss) {
            trace_lo[2 * mv + 1] = lo_l;
            trace_hi[2 * mv + 1] = hi_l;
            trace_loss[2 * mv + 1] = ll;
            trace_lo[2 * mv + 2] = lo_r;
            trace_hi[2 * mv + 2] = hi_r;
            trace_loss[2 * mv + 2] = lr;
            trace_i[mv] = i;
            trace_j[mv] = j;
        }
    }
    return r;
}

/* Steps 6-7 for one row. */
static void finish_row(const float *x, int d, const search_result *r, uint8_t *codes,
                       uint16_t *scale_bias)
{
    float lo = grid_lo(r->xmin, r->step, r->bi);
    float hi = grid_hi(r->xmax, r->step, r->bj);
    float s = (hi - lo) / ORACLE_LEVELS;
    uint16_t s16 = oracle_f32_to_f16(s);
    uint16_t b16 = oracle_f32_to_f16(lo);
    float S = oracle_f16_to_f32(s16);
    float B = oracle_f16_to_f32(b16);
    for (int m = 0; m < (d + 1) / 2; m++)
        codes[m] = 0;
    for (int k = 0; k < d; k++) {
        int q = (int)code_of(x[k], B, S);
        codes[k / 2] |= (uint8_t)(q << (4 * (k % 2)));
    }
    scale_bias[0] = s16;
    scale_bias[1] = b16;
}

/* Full trace of one row's search; each trace_* array holds 1 + 2*168 entries,
 * trace_i/trace_j hold 168. Returns Lbest and writes (i*, j*). */
float oracle_greedy_trace(const float *x, int32_t d, float *trace_lo, float *trace_hi,
                          float *trace_loss, int32_t *trace_i, int32_t *trace_j,
                          int32_t *best_ij)
{
    float cbuf[ORACLE_MAX_D];
    if (d < 1 || d > ORACLE_MAX_D)
        return NAN;
    search_result r = search_row(x, d, ORACLE_GREEDY, cbuf, trace_lo, trace_hi, trace_loss,
                                 trace_i, trace_j);
    best_ij[0] = r.bi;
    best_ij[1] = r.bj;
    return r.lbest;
}

/* ------------------------------------------------------------------------ */
/* codebook quantizer (per-row k-means, 16 centroids)                       */
/* ------------------------------------------------------------------------ */

/* argmin_j fl(|fl(x - c_j)|), ties to the lower j */
static int nearest(float x, const float *c)
{
    int best = 0;
    float bd = fabsf(x - c[0]);
    for (int j = 1; j < 16; j++) {
        float dj = fabsf(x - c[j]);
        if (dj < bd) {
            bd = dj;
            best = j;
        }
    }
    return best;
}

/* K2's update of the centroids c[16] from the assignment a[0..d-1]. */
static void kmeans_means(const float *x, const int32_t *a, int d, float *c)
{
    double s[16];
    int n[16];
    for (int j = 0; j < 16; j++) {
        s[j] = 0.0;
        n[j] = 0;
    }
    for (int k = 0; k < d; k++) {
        s[a[k]] += (double)x[k];
        n[a[k]] += 1;
    }
    for (int j = 0; j < 16; j++)
        if (n[j] > 0)
            c[j] = (float)(s[j] / (double)n[j]);
}

int32_t oracle_kmeans_means(const float *x, const int32_t *a, int32_t d, float *c)
{
    if (d < 1 || d > ORACLE_MAX_D)
        return -1;
    for (int k = 0; k < d; k++)
        if (a[k] < 0 || a[k] > 15)
            return -1;
    kmeans_means(x, a, d, c);
    return 0;
}

/* Steps K1-K3 for one row; cbuf holds next_pow2(d) floats. Writes the stored
 * centroids (binary16), the packed codes, and returns the row loss. */
static float kmeans_row(const float *x, int d, int iters, float *cbuf, uint8_t *codes, uint16_t *codebook)
{
    float xmin = x[0], xmax = x[0];
    for (int k = 1; k < d; k++) {
        xmin = fminf(xmin, x[k]);
        xmax = fmaxf(xmax, x[k]);
    }
    float step = (xmax - xmin) / ORACLE_LEVELS;
    float c[16];
    for (int j = 0; j < 16; j++)
        c[j] = fmaf((float)j, step, xmin);
    int P = next_pow2(d);
    int32_t a[ORACLE_MAX_D];
    for (int it = 0; it < iters; it++) {
        for (int k = 0; k < d; k++)
            a[k] = nearest(x[k], c);
        kmeans_means(x, a, d, c);
    }
    float C[16];
    for (int j = 0; j < 16; j++) {
        codebook[j] = oracle_f32_to_f16(c[j]);
        C[j] = oracle_f16_to_f32(codebook[j]);
    }
    for (int m = 0; m < (d + 1) / 2; m++)
        codes[m] = 0;
    for (int k = 0; k < P; k++)
        cbuf[k] = 0.0f;
    for (int k = 0; k < d; k++) {
        int q = nearest(x[k], C);
        codes[k / 2] |= (uint8_t)(q << (4 * (k % 2)));
        float e = x[k] - C[q];
        cbuf[k] = e * e;
    }
    return pairwise_sum(cbuf, P);
}

typedef struct {
    const float *x;
    int64_t n, ld;
    int d, iters;
    uint8_t *codes;
    int64_t codes_ld;
    uint16_t *codebook;
    float *loss;
    int64_t begin, end;
} kmeans_job;

static void *kmeans_worker(void *arg)
{
    kmeans_job *j = (kmeans_job *)arg;
    float cbuf[ORACLE_MAX_D];
    for (int64_t r = j->begin; r < j->end; r++) {
        float l = kmeans_row(j->x + r * j->ld, j->d, j->iters, cbuf, j->codes + r * j->codes_ld,
                             j->codebook + 16 * r);
        if (j->loss)
            j->loss[r] = l;
    }
    return NULL;
}

/* K1-K3 for n rows (codebook [n][16] binary16 patterns); threaded over rows. */
int32_t oracle_quantize_rows_kmeans(const float *x, int64_t n, int32_t d, int64_t ld, uint8_t *codes,
                                    int64_t codes_ld, uint16_t *codebook, float *loss, int32_t iters,
                                    int32_t nthreads);

/* xhat_k = w(C_{q_k}) for n rows. */
int32_t oracle_dequantize_rows_kmeans(const uint8_t *codes, int64_t codes_ld, const uint16_t *codebook, int64_t n,
                                      int32_t d, float *out, int64_t out_ld)
{
    if (n < 0 || d < 1 || d > ORACLE_MAX_D || out_ld < d || codes_ld < (d + 1) / 2)
        return -1;
    for (int64_t r = 0; r < n; r++)
        for (int k = 0; k < d; k++) {
            int q = (codes[r * codes_ld + k / 2] >> (4 * (k % 2))) & 15;
            out[r * out_ld + k] = oracle_f16_to_f32(codebook[16 * r + q]);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* threaded drivers                                                         */
/* ------------------------------------------------------------------------ */

static int resolve_threads(int32_t nthreads)
{
    if (nthreads > 0)
        return nthreads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

typedef struct {
    const float *x;
    int64_t n, ld;
    int d, mode;
    uint8_t *codes;
    int64_t codes_ld;
    uint16_t *scale_bias;
    float *loss;
    uint8_t *best_ij;
    int64_t begin, end;
} quant_job;

static void *quant_worker(void *arg)
{
    quant_job *j = (quant_job *)arg;
    float cbuf[ORACLE_MAX_D];
    for (int64_t row = j->begin; row < j->end; row++) {
        const float *x = j->x + row * j->ld;
        search_result r = search_row(x, j->d, j->mode, cbuf, NULL, NULL, NULL, NULL, NULL);
        finish_row(x, j->d, &r, j->codes + row * j->codes_ld, j->scale_bias + 2 * row);
        if (j->loss)
            j->loss[row] = r.lbest;
        if (j->best_ij) {
            j->best_ij[2 * row] = (uint8_t)r.bi;
            j->best_ij[2 * row + 1] = (uint8_t)r.bj;
        }
    }
    return NULL;
}

/* Quantizes n rows of x (row stride ld floats). codes: row stride codes_ld bytes;
 * scale_bias: [n][2] binary16 bit patterns; loss and best_ij may be NULL.
 * Returns 0, or -1 on bad arguments. */
int32_t oracle_quantize_rows(const float *x, int64_t n, int32_t d, int64_t ld, uint8_t *codes,
                             int64_t codes_ld, uint16_t *scale_bias, float *loss,
                             uint8_t *best_ij, int32_t mode, int32_t nthreads)
{
    if (n < 0 || d < 1 || d > ORACLE_MAX_D || ld < d || codes_ld < (d + 1) / 2)
        return -1;
    if (n == 0)
        return 0;
    int nt = resolve_threads(nthreads);
    if (nt > n)
        nt = (int)n;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    quant_job *jobs = (quant_job *)malloc(sizeof(quant_job) * (size_t)nt);
    for (int t = 0; t < nt; t++) {
        quant_job j = {x, n, ld, d, mode, codes, codes_ld, scale_bias, loss, best_ij,
                       n * t / nt, n * (t + 1) / nt};
        jobs[t] = j;
        pthread_create(&th[t], NULL, quant_worker, &jobs[t]);
    }
    for (int t = 0; t < nt; t++)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* xhat = fma(q, S, B) for n rows; out row stride out_ld floats. */
int32_t oracle_dequantize_rows(const uint8_t *codes, int64_t codes_ld, const uint16_t *scale_bias,
                               int64_t n, int32_t d, float *out, int64_t out_ld)
{
    if (n < 0 || d < 1 || d > ORACLE_MAX_D || out_ld < d || codes_ld < (d + 1) / 2)
        return -1;
    for (int64_t row = 0; row < n; row++) {
        float S = oracle_f16_to_f32(scale_bias[2 * row]);
        float B = oracle_f16_to_f32(scale_bias[2 * row + 1]);
        for (int k = 0; k < d; k++) {
            int q = (codes[row * codes_ld + k / 2] >> (4 * (k % 2))) & 0xf;
            out[row * out_ld + k] = fmaf((float)q, S, B);
        }
    }
    return 0;
}

/* Normalized l2 error of each of n rows (binary64); returns the sum over rows
 * (binary64, index order), or NAN on bad arguments. row_err may be NULL. */
double oracle_row_l2_error(const float *x, int64_t n, int32_t d, int64_t x_ld, const uint8_t *codes,
                           int64_t codes_ld, const uint16_t *scale_bias, double *row_err)
{
    if (n < 0 || d < 1 || d > ORACLE_MAX_D || x_ld < d || codes_ld < (d + 1) / 2)
        return NAN;
    double total = 0.0;
    for (int64_t row = 0; row < n; row++) {
        float S = oracle_f16_to_f32(scale_bias[2 * row]);
        float B = oracle_f16_to_f32(scale_bias[2 * row + 1]);
        double se = 0.0, sx = 0.0;
        for (int k = 0; k < d; k++) {
            int q = (codes[row * codes_ld + k / 2] >> (4 * (k % 2))) & 0xf;
            double xk = (double)x[row * x_ld + k];
            double e = xk - (double)fmaf((float)q, S, B);
            se += e * e;
            sx += xk * xk;
        }
        double err = sx > 0.0 ? sqrt(se / sx) : (se > 0.0 ? INFINITY : 0.0);
        if (row_err)
            row_err[row] = err;
        total += err;
    }
    return total;
}

typedef struct {
    const uint8_t *codes;
    const uint16_t *scale_bias;     /* uniform rows: {scale, bias} per row */
    int64_t n_rows;
    int64_t codes_ld;
    const uint16_t *codebook;       /* non-NULL: codebook rows, 16 binary16 centroids per row */
} oracle_table;

typedef struct {
    const oracle_table *tables;
    int T, d, B;
    const int32_t *indices;
    const int32_t *offsets;
    float *out;
    double *abs_sum;
    int64_t skipped;
    int64_t begin, end;
} bag_job;

static void *bag_worker(void *arg)
{
    bag_job *j = (bag_job *)arg;
    double acc[ORACLE_MAX_D], mag[ORACLE_MAX_D];
    int d = j->d;
    j->skipped = 0;
    for (int64_t g = j->begin; g < j->end; g++) {
        int t = (int)(g / j->B), b = (int)(g % j->B);
        const oracle_table *tab = &j->tables[t];
        for (int k = 0; k < d; k++)
            acc[k] = mag[k] = 0.0;
        int32_t p0 = j->offsets[g], p1 = j->offsets[g + 1];
        for (int32_t p = p0; p < p1; p++) {
            int32_t id = j->indices[p];
            if (id < 0 || (int64_t)id >= tab->n_rows) {
                j->skipped++;
                continue;
            }
            const uint8_t *row = tab->codes + (int64_t)id * tab->codes_ld;
            float S = 0.0f, Bv = 0.0f;
            if (!tab->codebook) {
                S = oracle_f16_to_f32(tab->scale_bias[2 * (int64_t)id]);
                Bv = oracle_f16_to_f32(tab->scale_bias[2 * (int64_t)id + 1]);
            }
            for (int k = 0; k < d; k++) {
                int q = (row[k / 2] >> (4 * (k % 2))) & 0xf;
                float xhat = tab->codebook ? oracle_f16_to_f32(tab->codebook[16 * (int64_t)id + q])
                                           : fmaf((float)q, S, Bv);
                acc[k] += (double)xhat;
                mag[k] += fabs((double)xhat);
            }
        }
        if (p1 < p0)
            j->skipped++;
        float *o = j->out + (int64_t)b * j->T * d + (int64_t)t * d;
        for (int k = 0; k < d; k++)
            o[k] = (float)acc[k];
        if (j->abs_sum) {
            double *m = j->abs_sum + (int64_t)b * j->T * d + (int64_t)t * d;
            for (int k = 0; k < d; k++)
                m[k] = mag[k];
        }
    }
    return NULL;
}

typedef struct {
    uint32_t key;
    int32_t bag;
    int64_t pos;
} bwd_entry;

static int entry_cmp(const void *pa, const void *pb)
{
    const bwd_entry *a = (const bwd_entry *)pa, *b = (const bwd_entry *)pb;
    if (a->key != b->key)
        return a->key < b->key ? -1 : 1;
    return a->pos < b->pos ? -1 : (a->pos > b->pos ? 1 : 0);
}

/* key in the ascending array sample[0..n)? */
static int in_sample(const uint32_t *sample, int64_t n, uint32_t key)
{
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        if (sample[mid] < key)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo < n && sample[lo] == key;
}

/* Steps a-e of the bag backward on T tables sharing d: masters W[t] (row stride
 * w_ld[t]) and packed tables codes[t]/scale_bias[t] (code row stride codes_ld[t]),
 * n_rows[t] rows each; grad is [B][T*d]. With sample_keys (ascending global keys), steps
 * c-e are applied to those rows only. Returns the number of invalid ids, -2 if the
 * offsets are not a CSR array (nothing changed), -1 on bad arguments. */
int64_t oracle_embbag_bwd_sgd(float *const *W, const int64_t *w_ld, uint8_t *const *codes,
                              const int64_t *codes_ld, uint16_t *const *scale_bias,
                              const int64_t *n_rows, int32_t T, int32_t d, const int32_t *indices,
                              const int32_t *offsets, int32_t B, int64_t n_indices, const float *grad,
                              float lr, int32_t mode, const uint32_t *sample_keys, int64_t n_sample)
{
    if (T < 1 || d < 1 || d > ORACLE_MAX_D || B < 0 || n_indices < 0)
        return -1;
    int64_t G = (int64_t)T * B;
    if (offsets[0] != 0 || offsets[G] != n_indices)
        return -2;
    for (int64_t g = 0; g < G; g++)
        if (offsets[g + 1] < offsets[g])
            return -2;
    /* a. entries */
    int64_t *row_base = (int64_t *)malloc(sizeof(int64_t) * (size_t)T);
    int64_t total = 0;
    for (int t = 0; t < T; t++) {
        row_base[t] = total;
        total += n_rows[t];
    }
    bwd_entry *e = (bwd_entry *)malloc(sizeof(bwd_entry) * (size_t)(n_indices > 0 ? n_indices : 1));
    int64_t ne = 0, invalid = 0;
    for (int64_t g = 0; g < G; g++) {
        int t = (int)(g / (B > 0 ? B : 1));
        for (int64_t p = offsets[g]; p < offsets[g + 1]; p++) {
            int32_t id = indices[p];
            if (id < 0 || (int64_t)id >= n_rows[t]) {
                invalid++;
                continue;
            }
            e[ne].key = (uint32_t)(row_base[t] + id);
            e[ne].bag = (int32_t)g;
            e[ne].pos = p;
            ne++;
        }
    }
    /* b. sort by (key, p) */
    qsort(e, (size_t)ne, sizeof(bwd_entry), entry_cmp);
    double *sum = (double *)malloc(sizeof(double) * (size_t)d);
    float cbuf[ORACLE_MAX_D];
    for (int64_t s0 = 0; s0 < ne;) {
        int64_t s1 = s0;
        while (s1 < ne && e[s1].key == e[s0].key)
            s1++;
        if (sample_keys && !in_sample(sample_keys, n_sample, e[s0].key)) {
            s0 = s1;  /* steps c-e only for the sampled rows */
            continue;
        }
        int t = 0;
        while (t + 1 < T && (int64_t)e[s0].key >= row_base[t + 1])
            t++;
        int64_t id = (int64_t)e[s0].key - row_base[t];
        /* c. the row's gradient: one binary64 sum over its entries, in list order */
        for (int k = 0; k < d; k++)
            sum[k] = 0.0;
        for (int64_t i = s0; i < s1; i++) {
            int64_t b = e[i].bag - (int64_t)t * B;
            const float *gr = grad + b * (int64_t)T * d + (int64_t)t * d;
            for (int k = 0; k < d; k++)
                sum[k] = sum[k] + (double)gr[k];
        }
        /* d. SGD step */
        float *w = W[t] + id * w_ld[t];
        for (int k = 0; k < d; k++)
            w[k] = fmaf(-lr, (float)sum[k], w[k]);
        /* e. re-quantize the row */
        search_result r = search_row(w, d, mode, cbuf, NULL, NULL, NULL, NULL, NULL);
        finish_row(w, d, &r, codes[t] + id * codes_ld[t], scale_bias[t] + 2 * id);
        s0 = s1;
    }
    free(sum);
    free(e);
    free(row_base);
    return invalid;
}

/* Sum-pooled lookup over T packed tables sharing d. indices/offsets as the CUDA
 * entry point takes them (offsets [T*B+1], table-major). out [B][T*d] float;
 * abs_sum (nullable) [B][T*d] double gets the sum of |xhat| per output element.
 * Out-of-range ids are skipped and decreasing offsets give an empty bag; the
 * return value is the number of such skips, or -1 on bad arguments. */
int64_t oracle_embbag(const oracle_table *tables, int32_t T, int32_t d, const int32_t *indices,
                      const int32_t *offsets, int32_t B, float *out, double *abs_sum,
                      int32_t nthreads)
{
    if (T < 1 || d < 1 || d > ORACLE_MAX_D || B < 0)
        return -1;
    int64_t G = (int64_t)T * B;
    if (G == 0)
        return 0;
    int nt = resolve_threads(nthreads);
    if (nt > G)
        nt = (int)G;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    bag_job *jobs = (bag_job *)malloc(sizeof(bag_job) * (size_t)nt);
    for (int t = 0; t < nt; t++) {
        bag_job j = {tables, T, d, B, indices, offsets, out, abs_sum, 0, G * t / nt, G * (t + 1) / nt};
        jobs[t] = j;
        pthread_create(&th[t], NULL, bag_worker, &jobs[t]);
    }
    int64_t skipped = 0;
    for (int t = 0; t < nt; t++) {
        pthread_join(th[t], NULL);
        skipped += jobs[t].skipped;
    }
    free(th);
    free(jobs);
    return skipped;
}

int32_t oracle_quantize_rows_kmeans(const float *x, int64_t n, int32_t d, int64_t ld, uint8_t *codes,
                                    int64_t codes_ld, uint16_t *codebook, float *loss, int32_t iters,
                                    int32_t nthreads)
{
    if (n < 0 || d < 1 || d > ORACLE_MAX_D || ld < d || codes_ld < (d + 1) / 2 || iters < 0)
        return -1;
    if (n == 0)
        return 0;
    int nt = resolve_threads(nthreads);
    if (nt > n)
        nt = (int)n;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    kmeans_job *jobs = (kmeans_job *)malloc(sizeof(kmeans_job) * (size_t)nt);
    for (int t = 0; t < nt; t++) {
        kmeans_job j = {x, n, ld, d, iters, codes, codes_ld, codebook, loss, n * t / nt, n * (t + 1) / nt};
        jobs[t] = j;
        pthread_create(&th[t], NULL, kmeans_worker, &jobs[t]);
    }
    for (int t = 0; t < nt; t++)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}
