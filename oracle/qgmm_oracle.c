/*
 * qgmm_oracle.c -- plain CPU oracle for the fused int8 GroupedMatmul +
 * MoeFinalizeRouting op.  TEST INFRASTRUCTURE ONLY: the tests, the package's
 * smoke check and the benchmark's CPU-baseline leg call it; the product path
 * never does.  It shares no code with the CUDA library.
 *
 * What it follows (pages as printed, by title and section):
 *  - "aclnnGroupedMatmulFinalizeRoutingWeightNzV2", function description: a
 *    grouped matmul whose output rows are combined into the output by index;
 *    parameter constraints: groupList type 0 is non-negative and monotone
 *    non-decreasing (cumulative ends), type 1 is non-negative (per-group
 *    counts); x2 is (e, k, n), or int32 (e, k, n/8) holding int4 values;
 *    scale is (e, 1, n); pertokenScale is (m); sharedInput rows land at
 *    sharedInputOffset with offset + bsdp <= outputBS; optional inputs may be
 *    absent.
 *  - "matmul支持pertoken量化模式", 计算示例: out[i][j] = (sum_k x[i][k] w[k][j])
 *    * deqScale[j] * perTokenScale[i], int8 inputs, exact integer products.
 *  - PTOAS issue 1568 (per_token_cast), 背景: the quantised value is the input
 *    multiplied by a precomputed inverse scale.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - bias is added after the two dequant scales and before the routing weight:
 *    y = ((acc * scale[g][j]) * pts[i] + bias[g][j]) * logit[i];
 *  - sharedInput is added unweighted; rows outside its range start at 0;
 *  - rows at or past the groups' total are ignored;
 *  - the combine sums, per output element, the shared value first and then the
 *    contributions in ascending source row order;
 *  - int4: the lowest nibble of each int32 word is the lowest n index, two's
 *    complement (values -8..7);
 *  - per-token quant: a = max |x|, pts = a/127, inv = 127/a (0 for a zero row),
 *    q = round-half-even(x * inv) clamped to [-127, 127]; non-finite inputs as
 *    IEEE f32 has them (NaN skipped by the absmax), a NaN product gives 0;
 *  - a BF16 scale (page 1, parameter notes: scaleOptional is FLOAT or BF16 on
 *    A2/A3) is widened to f32, which is exact, and then enters the same f32
 *    dequant as a FLOAT scale (qo_bf16_to_f32).
 *
 * Precision: integer accumulation is exact (int64, checked to fit int32).
 * Two float forms of the dequant+combine are provided:
 *  - qo_finalize_f64: every step in double -- the value the op approximates;
 *  - qo_finalize_f32: every step in IEEE single precision in the order above
 *    (compiled with -ffp-contract=off, no fast-math) -- what an f32 device
 *    computes when it keeps that order.
 * The per-token quant decides integers from floats, so it runs in f32.
 *
 * Parallelism: independent destination rows are split across POSIX threads;
 * each element's arithmetic is the same as in the single-threaded loop.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

float qo_e4m3_decode(uint8_t c);
double qo_e2m1_decode(uint8_t nibble);
double qo_e8m0_decode(uint8_t c);

enum {
    QO_OK = 0,
    QO_ERR_NEGATIVE_COUNT = 1,
    QO_ERR_NOT_MONOTONE = 2,
    QO_ERR_TOTAL_GT_M = 3,
    QO_ERR_BAD_ROW_INDEX = 4,
    QO_ERR_ACC_OVERFLOW = 5,
    QO_ERR_ARG = 6,
};

/* ---- groupList -> row offsets (parameter constraints of page 1) -------- */
int qo_group_offsets(const int64_t *group_list, int64_t e, int group_list_type,
                     int64_t m, int64_t *off /* [e+1] */)
{
    if (!group_list || !off || e < 1) return QO_ERR_ARG;
    off[0] = 0;
    for (int64_t g = 0; g < e; ++g) {
        int64_t v = group_list[g];
        if (v < 0) return QO_ERR_NEGATIVE_COUNT;
        if (group_list_type == 0) {
            if (v < off[g]) return QO_ERR_NOT_MONOTONE;
            off[g + 1] = v;
        } else if (group_list_type == 1) {
            off[g + 1] = off[g] + v;
        } else {
            return QO_ERR_ARG;
        }
    }
    if (off[e] > m) return QO_ERR_TOTAL_GT_M;
    return QO_OK;
}

/* weight value W(g, kk, j) of the int8 or the int32-packed int4 layout */
static inline int32_t weight_at(const void *x2, int weight_type, int64_t k, int64_t n,
                                int64_t g, int64_t kk, int64_t j)
{
    if (weight_type == 0) {
        const int8_t *w = (const int8_t *)x2;
        return (int32_t)w[(g * k + kk) * n + j];
    } else {
        const int32_t *w = (const int32_t *)x2;
        uint32_t word = (uint32_t)w[(g * k + kk) * (n / 8) + j / 8];
        int32_t nib = (int32_t)((word >> (4 * (j % 8))) & 0xFu);
        return nib >= 8 ? nib - 16 : nib;
    }
}

static int64_t group_of_row(const int64_t *off, int64_t e, int64_t i)
{
    for (int64_t g = 0; g < e; ++g)
        if (i >= off[g] && i < off[g + 1]) return g;
    return -1;
}

/* FLOAT8 E4M3 operands (weight_type 2, page 1: x1 and x2 both FLOAT8_E4M3FN in the
 * Atlas 350 per-token / per-channel mode): acc[j] = sum_kk x1[i][kk] * x2[g][kk][j]
 * over the values the codes stand for, in double.  Exact: every product of two
 * E4M3 values is a multiple of 2^-18 below 2^18, so a sum of at most 65536 of them
 * needs under 53 significant bits.  mag[j] = sum_kk |x1[i][kk] * x2[g][kk][j]|. */
static void accum_row_f8(const int8_t *x1, const void *x2, int64_t k, int64_t n, int64_t g, int64_t i,
                         double *acc, double *mag)
{
    const uint8_t *a = (const uint8_t *)x1 + i * k;
    for (int64_t j = 0; j < n; ++j) acc[j] = mag[j] = 0.0;
    for (int64_t kk = 0; kk < k; ++kk) {
        double av = (double)qo_e4m3_decode(a[kk]);
        if (av == 0.0) continue;
        const uint8_t *wrow = (const uint8_t *)x2 + (g * k + kk) * n;
        for (int64_t j = 0; j < n; ++j) {
            double p = av * (double)qo_e4m3_decode(wrow[j]);
            acc[j] += p;
            mag[j] += fabs(p);
        }
    }
}

/* MxA8W4 (weight_type 3, page 1's Atlas 350 MxA8W4 mode): x1 is FLOAT8 E4M3 [m, k]
 * with one E8M0 scale per 32 k-elements, sfa [m, k/32] (pertokenScale, shape
 * (m, ceil(k/64), 2)); the weights are FP4 E2M1, transposed (e, n, k) as page 1
 * requires for this mode, two per byte with the lower k in the low nibble (a
 * reading), (e, n, k/2) bytes, with one E8M0 scale per 32 k-elements, sfb
 * [e, n, k/32] (scale, shape (e, n, ceil(k/64), 2)).  A block's products are
 * summed, then multiplied by both of the block's scales:
 *   acc[j] = sum_b 2^(sfa[i][b] - 127) * 2^(sfb[g][j][b] - 127) * sum_{kk in b} x1[i][kk] * W(g, j, kk)
 * in double; mag[j] is the same sum of |scaled products|. */
static void accum_row_mx(const uint8_t *x1, const uint8_t *sfa, const uint8_t *w, const uint8_t *sfb, int64_t k,
                         int64_t n, int64_t g, int64_t i, double *acc, double *mag, double *xrow)
{
    const int64_t nb = k / 32;
    for (int64_t kk = 0; kk < k; ++kk) xrow[kk] = (double)qo_e4m3_decode(x1[i * k + kk]);
    for (int64_t j = 0; j < n; ++j) {
        const uint8_t *wr = w + (g * n + j) * (k / 2);
        double a = 0.0, am = 0.0;
        for (int64_t b = 0; b < nb; ++b) {
            double sum = 0.0, sabs = 0.0;
            for (int64_t kk = b * 32; kk < b * 32 + 32; ++kk) {
                const uint8_t byte = wr[kk / 2];
                const double p = xrow[kk] * qo_e2m1_decode((kk & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF));
                sum += p;
                sabs += fabs(p);
            }
            const double sc = qo_e8m0_decode(sfa[i * nb + b]) * qo_e8m0_decode(sfb[(g * n + j) * nb + b]);
            a += sc * sum;
            am += sc * sabs;
        }
        acc[j] = a;
        mag[j] = am;
    }
}

/* acc[j] = sum_kk x1[i][kk] * W(g, kk, j), exact; returns 0 or overflow code */
static int accum_row(const int8_t *x1, const void *x2, int weight_type, int64_t k, int64_t n,
                     int64_t g, int64_t i, int64_t *acc64 /* [n] scratch */, int32_t *acc)
{
    for (int64_t j = 0; j < n; ++j) acc64[j] = 0;
    for (int64_t kk = 0; kk < k; ++kk) {
        int64_t a = (int64_t)x1[i * k + kk];
        if (a == 0) continue;
        if (weight_type == 0) {
            const int8_t *wrow = (const int8_t *)x2 + (g * k + kk) * n;
            for (int64_t j = 0; j < n; ++j) acc64[j] += a * (int64_t)wrow[j];
        } else {
            for (int64_t j = 0; j < n; ++j) acc64[j] += a * (int64_t)weight_at(x2, 1, k, n, g, kk, j);
        }
    }
    int rc = QO_OK;
    for (int64_t j = 0; j < n; ++j) {
        if (acc64[j] > INT32_MAX || acc64[j] < INT32_MIN) rc = QO_ERR_ACC_OVERFLOW;
        acc[j] = (int32_t)acc64[j];
    }
    return rc;
}

/* ---- parallel-for over a list of items ---------------------------------- */
typedef struct {
    void (*fn)(void *ctx, int64_t item, int64_t *s64, int32_t *s32, double *sd, int *rc);
    void *ctx;
    int64_t nitems, n;
    int nthreads, tid;
    int rc;
} job_t;

static void *job_main(void *p)
{
    job_t *j = (job_t *)p;
    int64_t *s64 = (int64_t *)malloc(sizeof(int64_t) * (size_t)j->n);
    int32_t *s32 = (int32_t *)malloc(sizeof(int32_t) * (size_t)j->n);
    double *sd = (double *)malloc(sizeof(double) * (2 * (size_t)j->n + 65536));   /* + one decoded x1 row */
    if (!s64 || !s32 || !sd) { j->rc = QO_ERR_ARG; free(s64); free(s32); free(sd); return NULL; }
    for (int64_t it = j->tid; it < j->nitems; it += j->nthreads) j->fn(j->ctx, it, s64, s32, sd, &j->rc);
    free(s64);
    free(s32);
    free(sd);
    return NULL;
}

static int run_parallel(void (*fn)(void *, int64_t, int64_t *, int32_t *, double *, int *), void *ctx,
                        int64_t nitems, int64_t n, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    job_t jobs[256];
    pthread_t th[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn; jobs[t].ctx = ctx; jobs[t].nitems = nitems; jobs[t].n = n;
        jobs[t].nthreads = nthreads; jobs[t].tid = t; jobs[t].rc = QO_OK;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, job_main, &jobs[t]);
    job_main(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    int rc = QO_OK;
    for (int t = 0; t < nthreads; ++t) if (jobs[t].rc != QO_OK) rc = jobs[t].rc;
    return rc;
}

/* ---- exact int32 accumulators for chosen source rows ------------------- */
typedef struct {
    const int8_t *x1; const void *x2; int weight_type; int64_t k, n, e;
    const int64_t *off; const int64_t *rows; int32_t *acc_out;
} accum_ctx;

static void accum_item(void *p, int64_t it, int64_t *s64, int32_t *s32, double *sd, int *rc)
{
    accum_ctx *c = (accum_ctx *)p;
    (void)s32;
    (void)sd;
    int64_t i = c->rows ? c->rows[it] : it;
    int32_t *dst = c->acc_out + it * c->n;
    int64_t g = group_of_row(c->off, c->e, i);
    if (g < 0) { memset(dst, 0, sizeof(int32_t) * (size_t)c->n); return; }
    int r = accum_row(c->x1, c->x2, c->weight_type, c->k, c->n, g, i, s64, dst);
    if (r != QO_OK) *rc = r;
}

/* acc_out[r][j] for source rows rows[0..nrows) (rows == NULL: rows 0..nrows-1).
 * Rows that belong to no group (at or past the total) come back as zeros. */
int qo_accum(const int8_t *x1, const void *x2, int weight_type, int64_t m, int64_t k, int64_t n,
             int64_t e, const int64_t *group_list, int group_list_type,
             const int64_t *rows, int64_t nrows, int32_t *acc_out, int nthreads)
{
    if (!x1 || !x2 || !acc_out || k < 1 || n < 1 || (weight_type == 1 && n % 8)) return QO_ERR_ARG;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(e + 1));
    if (!off) return QO_ERR_ARG;
    int rc = qo_group_offsets(group_list, e, group_list_type, m, off);
    if (rc == QO_OK) {
        accum_ctx c = {x1, x2, weight_type, k, n, e, off, rows, acc_out};
        rc = run_parallel(accum_item, &c, nrows, n, nthreads);
    }
    free(off);
    return rc;
}

/* FP8 accumulators acc_out[r][j] (double, exact) and mag_out[r][j] (sum of
 * |products|, may be NULL) for source rows rows[0..nrows); rows past the total
 * come back as zeros. */
typedef struct {
    const int8_t *x1; const void *x2; int64_t k, n, e;
    const int64_t *off; const int64_t *rows; double *acc_out, *mag_out;
} accum_f8_ctx;

static void accum_f8_item(void *p, int64_t it, int64_t *s64, int32_t *s32, double *sd, int *rc)
{
    accum_f8_ctx *c = (accum_f8_ctx *)p;
    (void)s64; (void)s32; (void)rc;
    int64_t i = c->rows ? c->rows[it] : it;
    double *dst = c->acc_out + it * c->n;
    double *mag = c->mag_out ? c->mag_out + it * c->n : sd + c->n;
    int64_t g = group_of_row(c->off, c->e, i);
    if (g < 0) {
        for (int64_t j = 0; j < c->n; ++j) dst[j] = mag[j] = 0.0;
        return;
    }
    accum_row_f8(c->x1, c->x2, c->k, c->n, g, i, dst, mag);
}

int qo_accum_f8(const int8_t *x1, const void *x2, int64_t m, int64_t k, int64_t n, int64_t e,
                const int64_t *group_list, int group_list_type, const int64_t *rows, int64_t nrows,
                double *acc_out, double *mag_out, int nthreads)
{
    if (!x1 || !x2 || !acc_out || k < 1 || n < 1) return QO_ERR_ARG;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(e + 1));
    if (!off) return QO_ERR_ARG;
    int rc = qo_group_offsets(group_list, e, group_list_type, m, off);
    if (rc == QO_OK) {
        accum_f8_ctx c = {x1, x2, k, n, e, off, rows, acc_out, mag_out};
        rc = run_parallel(accum_f8_item, &c, nrows, n, nthreads);
    }
    free(off);
    return rc;
}

/* ---- dequant + combine -------------------------------------------------- */
typedef struct {
    const int8_t *x1; const void *x2; int weight_type; int64_t m, k, n, e;
    const int64_t *off; int64_t total;
    const float *scale, *pts, *logit, *bias;
    const void *row_index; int row_index_type;
    const uint16_t *shared; int64_t shared_bs, shared_offset, output_bs;
    const int64_t *dest_rows;
    double *out64; double *sabs64; float *out32;
    const uint8_t *sfa, *sfb;   /* weight_type 3 only */
} fin_ctx;

static inline float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static inline int64_t dest_of(const fin_ctx *c, int64_t i)
{
    if (!c->row_index) return i;
    if (c->row_index_type == 0) return ((const int64_t *)c->row_index)[i];
    return (int64_t)((const int32_t *)c->row_index)[i];
}

static void fin_item(void *p, int64_t it, int64_t *s64, int32_t *acc, double *sd, int *rc)
{
    fin_ctx *c = (fin_ctx *)p;
    const int64_t n = c->n;
    int64_t r = c->dest_rows ? c->dest_rows[it] : it;
    double *o64 = c->out64 ? c->out64 + it * n : NULL;
    double *a64 = c->sabs64 ? c->sabs64 + it * n : NULL;
    float *o32 = c->out32 ? c->out32 + it * n : NULL;

    /* initial value: the sharedInput row landing here, else zero */
    int in_shared = c->shared && r >= c->shared_offset && r < c->shared_offset + c->shared_bs;
    for (int64_t j = 0; j < n; ++j) {
        float s = in_shared ? bf16_to_f32(c->shared[(r - c->shared_offset) * n + j]) : 0.0f;
        if (o64) o64[j] = (double)s;
        if (a64) a64[j] = fabs((double)s);
        if (o32) o32[j] = s;
    }
    /* contributions in ascending source row order */
    for (int64_t i = 0; i < c->total; ++i) {
        int64_t d = dest_of(c, i);
        if (d < 0 || d >= c->output_bs) { *rc = QO_ERR_BAD_ROW_INDEX; continue; }
        if (d != r) continue;
        int64_t g = group_of_row(c->off, c->e, i);
        const int f8 = c->weight_type == 2 || c->weight_type == 3;
        double *accd = sd, *mag = sd + n;       /* FP8 / MX: the sums and sums of |products| */
        if (c->weight_type == 3) {
            accum_row_mx((const uint8_t *)c->x1, c->sfa, (const uint8_t *)c->x2, c->sfb, c->k, n, g, i, accd, mag,
                         sd + 2 * n);
        } else if (f8) {
            accum_row_f8(c->x1, c->x2, c->k, n, g, i, accd, mag);
        } else {
            int ar = accum_row(c->x1, c->x2, c->weight_type, c->k, n, g, i, s64, acc);
            if (ar != QO_OK) *rc = ar;
        }
        const float pts = c->pts ? c->pts[i] : 1.0f;
        const float lg = c->logit ? c->logit[i] : 1.0f;
        for (int64_t j = 0; j < n; ++j) {
            const float sc = c->scale ? c->scale[g * n + j] : 1.0f;
            const float bs = c->bias ? c->bias[g * n + j] : 0.0f;
            const double av = f8 ? accd[j] : (double)acc[j];
            if (o64 || a64) {
                double y = ((av * (double)sc) * (double)pts + (double)bs) * (double)lg;
                if (o64) o64[j] += y;
                /* the rounding of (acc*scale*pts + bias)*logit in any f32 order is bounded by a
                   few ulp of the summands' magnitudes, taken before the bias can cancel; for FP8
                   operands the accumulation itself rounds, so its terms are sum |products| */
                const double am = f8 ? mag[j] : fabs(av);
                if (a64) a64[j] += (am * fabs((double)sc * (double)pts) + fabs((double)bs)) * fabs((double)lg);
            }
            if (o32) {
                float y = (float)av;            /* round to nearest even (FP8: of the exact sum) */
                y = y * sc;
                y = y * pts;
                y = y + bs;
                y = y * lg;
                o32[j] = o32[j] + y;
            }
        }
    }
}

/*
 * Output rows dest_rows[0..ndest) (dest_rows == NULL: rows 0..ndest-1) of the
 * op.  out64/sabs64 (double, may be NULL): value in double, and the magnitude
 * that bounds f32 rounding error in each element: |initial value| plus, per
 * contribution, (|acc*scale*pts| + |bias|) * |logit|.
 * out32 (may be NULL): the same in f32 in the fixed order.  scale, pts, logit,
 * bias, row_index, shared may be NULL (1, 1, 1, 0, identity, absent).
 */
int qo_finalize(const int8_t *x1, const void *x2, int weight_type, int64_t m, int64_t k, int64_t n,
                int64_t e, const int64_t *group_list, int group_list_type,
                const float *scale, const float *pts, const float *logit, const float *bias,
                const void *row_index, int row_index_type,
                const uint16_t *shared, int64_t shared_bs, int64_t shared_offset, int64_t output_bs,
                const int64_t *dest_rows, int64_t ndest,
                double *out64, double *sabs64, float *out32, int nthreads)
{
    if (!x1 || !x2 || k < 1 || n < 1 || output_bs < 1 || (weight_type == 1 && n % 8) || weight_type < 0 ||
        weight_type > 2)
        return QO_ERR_ARG;
    if (shared && (shared_offset < 0 || shared_offset + shared_bs > output_bs)) return QO_ERR_ARG;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(e + 1));
    if (!off) return QO_ERR_ARG;
    int rc = qo_group_offsets(group_list, e, group_list_type, m, off);
    if (rc == QO_OK) {
        fin_ctx c = {x1, x2, weight_type, m, k, n, e, off, off[e], scale, pts, logit, bias,
                     row_index, row_index_type, shared, shared_bs, shared_offset, output_bs,
                     dest_rows, out64, sabs64, out32, NULL, NULL};
        rc = run_parallel(fin_item, &c, ndest, n, nthreads);
    }
    free(off);
    return rc;
}

/*
 * MxA8W4 (accum_row_mx): x1 E4M3 [m, k] with sfa E8M0 [m, k/32]; weights E2M1
 * (e, n, k/2) bytes with sfb E8M0 [e, n, k/32]; k % 32 == 0, k <= 65536.  The
 * output is (acc + bias) * logit combined as in qo_finalize (the block scales
 * take the place of scale and pertokenScale); the arguments after sfb are those
 * of qo_finalize.
 */
int qo_finalize_mx(const uint8_t *x1, const uint8_t *sfa, const uint8_t *x2, const uint8_t *sfb, int64_t m,
                   int64_t k, int64_t n, int64_t e, const int64_t *group_list, int group_list_type,
                   const float *logit, const float *bias, const void *row_index, int row_index_type,
                   const uint16_t *shared, int64_t shared_bs, int64_t shared_offset, int64_t output_bs,
                   const int64_t *dest_rows, int64_t ndest, double *out64, double *sabs64, float *out32,
                   int nthreads)
{
    if (!x1 || !sfa || !x2 || !sfb || k < 32 || k % 32 || k > 65536 || n < 1 || output_bs < 1) return QO_ERR_ARG;
    if (shared && (shared_offset < 0 || shared_offset + shared_bs > output_bs)) return QO_ERR_ARG;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(e + 1));
    if (!off) return QO_ERR_ARG;
    int rc = qo_group_offsets(group_list, e, group_list_type, m, off);
    if (rc == QO_OK) {
        fin_ctx c = {(const int8_t *)x1, x2, 3, m, k, n, e, off, off[e], NULL, NULL, logit, bias,
                     row_index, row_index_type, shared, shared_bs, shared_offset, output_bs,
                     dest_rows, out64, sabs64, out32, sfa, sfb};
        rc = run_parallel(fin_item, &c, ndest, n, nthreads);
    }
    free(off);
    return rc;
}

/* MxA8W4 accumulators (accum_row_mx) for source rows rows[0..nrows) (NULL: all);
 * rows past the total come back as zeros. */
typedef struct {
    const uint8_t *x1, *sfa, *x2, *sfb; int64_t k, n, e;
    const int64_t *off; const int64_t *rows; double *acc_out, *mag_out;
} accum_mx_ctx;

static void accum_mx_item(void *p, int64_t it, int64_t *s64, int32_t *s32, double *sd, int *rc)
{
    accum_mx_ctx *c = (accum_mx_ctx *)p;
    (void)s64; (void)s32; (void)rc;
    int64_t i = c->rows ? c->rows[it] : it;
    double *dst = c->acc_out + it * c->n;
    double *mag = c->mag_out ? c->mag_out + it * c->n : sd + c->n;
    int64_t g = group_of_row(c->off, c->e, i);
    if (g < 0) {
        for (int64_t j = 0; j < c->n; ++j) dst[j] = mag[j] = 0.0;
        return;
    }
    accum_row_mx(c->x1, c->sfa, c->x2, c->sfb, c->k, c->n, g, i, dst, mag, sd + 2 * c->n);
}

int qo_accum_mx(const uint8_t *x1, const uint8_t *sfa, const uint8_t *x2, const uint8_t *sfb, int64_t m,
                int64_t k, int64_t n, int64_t e, const int64_t *group_list, int group_list_type,
                const int64_t *rows, int64_t nrows, double *acc_out, double *mag_out, int nthreads)
{
    if (!x1 || !sfa || !x2 || !sfb || !acc_out || k < 32 || k % 32 || k > 65536 || n < 1) return QO_ERR_ARG;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(e + 1));
    if (!off) return QO_ERR_ARG;
    int rc = qo_group_offsets(group_list, e, group_list_type, m, off);
    if (rc == QO_OK) {
        accum_mx_ctx c = {x1, sfa, x2, sfb, k, n, e, off, rows, acc_out, mag_out};
        rc = run_parallel(accum_mx_item, &c, nrows, n, nthreads);
    }
    free(off);
    return rc;
}

/* ---- bf16 -> f32 widening (a BF16 scale; exact) ------------------------- */
int qo_bf16_to_f32(const uint16_t *in, int64_t count, float *out)
{
    if ((!in || !out) && count > 0) return QO_ERR_ARG;
    for (int64_t i = 0; i < count; ++i) out[i] = bf16_to_f32(in[i]);
    return QO_OK;
}

/* ---- per-token quantisation (f32; the decision is an integer) -----------
 * Non-finite inputs (a reading; the pages do not mention them) keep IEEE f32
 * semantics: a NaN element is not larger than anything, so the absmax skips
 * it; an infinite element makes a = inf, pts = inf and inv = 127/inf = 0.  A
 * product x*inv that is NaN (a NaN element, or an infinite one times the zero
 * inverse) has no integer code and quantises to 0; an infinite product would
 * saturate like any value past 127. */
int qo_per_token_quant(const uint16_t *x_bf16, int64_t rows, int64_t k, int8_t *q, float *pts)
{
    if (!x_bf16 || !q || !pts || rows < 0 || k < 1) return QO_ERR_ARG;
    for (int64_t i = 0; i < rows; ++i) {
        float a = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            float v = fabsf(bf16_to_f32(x_bf16[i * k + j]));
            if (v > a) a = v;               /* false for NaN: skipped */
        }
        pts[i] = a / 127.0f;
        float inv = a > 0.0f ? 127.0f / a : 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            float t = bf16_to_f32(x_bf16[i * k + j]) * inv;
            if (isnan(t)) {
                q[i * k + j] = 0;
                continue;
            }
            float r = rintf(t);                 /* default mode: half to even */
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[i * k + j] = (int8_t)r;
        }
    }
    return QO_OK;
}

/* ---- per-32-group FP8 E4M3 cast ------------------------------------------
 * "PTOAS issue 1568", 背景: per_token_cast multiplies each bf16 value by an
 * inverse scale factor broadcast over its group of 32 elements (a 256-element
 * tile uses sf_inv[row, tile*8 .. tile*8+7]) and converts the product to
 * FLOAT8 E4M3FN; the scale factors are packed ("packed SF").  The page does
 * not say how a scale factor is chosen.  Reading (the block format that
 * per-32 FP8 groups with packed one-byte scale factors belong to, and the one
 * page 1's MxA8W4 mode consumes): an E8M0 power of two per group, whose
 * exponent places the group's largest magnitude in E4M3's top binade:
 *     amax = max |x| over the group's 32 elements (NaN skipped, as above)
 *     sf   = max(0, biased f32 exponent of amax - 8)         (E8M0 code)
 *     inv  = 2^(127 - sf)                                     (exact)
 *     q    = E4M3(x * inv), round to nearest even, magnitudes past 448
 *            (and infinities) saturate to 448, NaN gives 0x7F
 * so x ~= q * 2^(sf - 127).  (amax 0 or an f32-subnormal amax gives sf = 0.)
 * x * inv is exact in f32 except where it falls below 2^-126, far under
 * E4M3's smallest subnormal 2^-9, so the one rounding is the E4M3 one. */

/* E4M3FN from its definition: sign, 4 exponent bits (bias 7), 3 fraction bits;
 * exponent 0 holds subnormals m * 2^-9; S.1111.111 is NaN; no infinities; the
 * largest finite magnitude is 1.75 * 2^8 = 448 (S.1111.110). */
uint8_t qo_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (a >= 448.0f) return sign | 0x7E;
    if (a < 0.015625f) {                       /* below 2^-6: subnormal grid m * 2^-9 */
        float m = rintf(a * 512.0f);           /* exact product; m = 8 is 2^-6, code 8 */
        return sign | (uint8_t)m;
    }
    int e = ilogbf(a);                         /* -6 .. 8 */
    float frac = ldexpf(a, -e) - 1.0f;         /* [0, 1), exact */
    int m = (int)rintf(frac * 8.0f);           /* exact product, then half to even */
    if (m == 8) { m = 0; e += 1; }
    int code = ((e + 7) << 3) | m;
    if (code > 0x7E) code = 0x7E;              /* the tie at 464 rounds up: saturate */
    return sign | (uint8_t)code;
}

/* the value an E4M3FN code stands for (NaN for S.1111.111) */
float qo_e4m3_decode(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    float s = (c & 0x80) ? -1.0f : 1.0f;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return s * ldexpf((float)m, -9);
    return s * ldexpf(1.0f + (float)m / 8.0f, e - 7);
}

int qo_per_token_quant_mxfp8(const uint16_t *x_bf16, int64_t rows, int64_t k, uint8_t *q, uint8_t *sf)
{
    if (!x_bf16 || !q || !sf || rows < 0 || k < 32 || k % 32) return QO_ERR_ARG;
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t g = 0; g < k / 32; ++g) {
            const uint16_t *x = x_bf16 + i * k + g * 32;
            float a = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float v = fabsf(bf16_to_f32(x[j]));
                if (v > a) a = v;               /* false for NaN: skipped */
            }
            uint32_t bits;
            memcpy(&bits, &a, sizeof bits);
            int biased = (int)((bits >> 23) & 0xFF);
            int code = biased - 8 > 0 ? biased - 8 : 0;
            float inv = ldexpf(1.0f, 127 - code);
            sf[i * (k / 32) + g] = (uint8_t)code;
            for (int j = 0; j < 32; ++j) q[i * k + g * 32 + j] = qo_e4m3_encode(bf16_to_f32(x[j]) * inv);
        }
    }
    return QO_OK;
}

/* FP4 E2M1 from its definition: sign (bit 3), 2 exponent bits (bias 1), 1 fraction
 * bit; exponent 0 holds the subnormal m * 0.5.  Values 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double qo_e2m1_decode(uint8_t nibble)
{
    const int e = (nibble >> 1) & 3, m = nibble & 1;
    const double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (nibble & 8) ? -v : v;
}

/* E8M0 scale from its definition: 2^(c - 127); 0xFF is NaN. */
double qo_e8m0_decode(uint8_t c)
{
    return c == 0xFF ? NAN : ldexp(1.0, (int)c - 127);
}
