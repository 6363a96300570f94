/*
 * kq_oracle.c -- plain, slow fp64 CPU oracle for the fused Kronecker-factored
 * transform + per-token INT4 quantiser.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *   - Kronecker product (Kronecker Product page, "Definition", entrywise
 *     formula and block form) and the vectorisation identity
 *     vec(V)(P1 (x) P2) = vec(P1^T V P2) (same page, "Why It Matters for LLM
 *     Quantization"; FlatQuant page, "Kronecker factorization").  A token row
 *     x of length n = n1*n2 is read row-major as X~[a][b] = x[a*n2 + b] and
 *     the transform is Y~ = P1^T X~ P2, stored back row-major:
 *     y[i*n2 + j] = Y~[i][j].  This equals x (P1 (x) P2) (row-vector
 *     convention; checked against an explicit Kronecker matrix by the tests).
 *   - Per-channel scaling diag(c) applied before the transform (FlatQuant
 *     page, "Per-channel scaling and learnable clipping"); the path is given
 *     cinv = 1/c and uses x' = x * cinv.
 *   - Clipping after the transform with ratio alpha in (0, 1] (same section),
 *     quantiser Q onto 4-bit integer points with step s (FlatQuant page,
 *     "Symbol Map"): one scale per token, s = alpha * max|y| / 7,
 *     q = clamp(round-half-to-even(y / s), -8, 7).
 *   - Inverse: (P1 (x) P2)^-1 = P1^-1 (x) P2^-1 (FlatQuant page, "Kronecker
 *     factorization", equation for Q(XP)Q(P^-1 W^T)); x^ = (P1^-T Y^ P2^-1) * c.
 *
 * Arithmetic: every input is widened exactly to double (bf16 -> float ->
 * double, float -> double); all sums are plain fp64 loops in the order of the
 * definition: first Z = X~' P2 (sum over b), then Y~ = P1^T Z (sum over a).
 * Rounding uses nearbyint() under the default round-to-nearest-even mode.
 *
 * Threads: tokens are independent, so token ranges are split over pthreads.
 * That is the only parallelism; there is no blocking or reordering.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared kq_oracle.c -lpthread -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KQO_OK 0
#define KQO_ERR_ARG -1
#define KQO_ERR_NOMEM -2

/* bf16 bit pattern -> double, exact (bf16 is the top half of a float). */
static double bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* x' = x * cinv, then Z = X~' P2, then Y~ = P1^T Z, for one token. */
static void transform_token(const uint16_t *x, const double *P1, const double *P2,
                            const float *cinv, int n1, int n2,
                            double *xs, double *Z, double *y)
{
    int n = n1 * n2;
    for (int k = 0; k < n; ++k)
        xs[k] = bf16_to_double(x[k]) * (cinv ? (double)cinv[k] : 1.0);
    /* Right contraction: Z[a][j] = sum_b X~'[a][b] P2[b][j]. */
    for (int a = 0; a < n1; ++a)
        for (int j = 0; j < n2; ++j) {
            double acc = 0.0;
            for (int b = 0; b < n2; ++b)
                acc += xs[a * n2 + b] * P2[b * n2 + j];
            Z[a * n2 + j] = acc;
        }
    /* Left contraction: Y~[i][j] = sum_a P1[a][i] Z[a][j]  (P1 transposed). */
    for (int i = 0; i < n1; ++i)
        for (int j = 0; j < n2; ++j) {
            double acc = 0.0;
            for (int a = 0; a < n1; ++a)
                acc += P1[a * n1 + i] * Z[a * n2 + j];
            y[i * n2 + j] = acc;
        }
}

/*
 * Per-token symmetric INT4 quantiser with clip ratio alpha.
 * codes[k] in [-8, 7]; packed byte k holds code 2k in the low nibble and code
 * 2k+1 in the high nibble (two's complement).  dist[k] = distance of y/s to
 * the nearest rounding boundary (a half-integer); for s == 0 it is 0.5.
 */
static void quantize_token(const double *y, int n, double alpha, int8_t *codes,
                           uint8_t *packed, double *scale64, float *scale32,
                           double *dist)
{
    double m = 0.0;
    for (int k = 0; k < n; ++k) {
        double a = fabs(y[k]);
        if (a > m)
            m = a;
    }
    double s = alpha * m / 7.0;
    if (scale64)
        *scale64 = s;
    if (scale32)
        *scale32 = (float)s;
    for (int k = 0; k < n; ++k) {
        int q = 0;
        double d = 0.5;
        if (s > 0.0) {
            double r = y[k] / s;
            double rq = nearbyint(r);
            if (rq > 7.0)
                rq = 7.0;
            if (rq < -8.0)
                rq = -8.0;
            q = (int)rq;
            d = fabs(fabs(r - floor(r)) - 0.5);
        }
        if (codes)
            codes[k] = (int8_t)q;
        if (dist)
            dist[k] = d;
        if (packed) {
            uint8_t nib = (uint8_t)(q & 0xF);
            if (k & 1)
                packed[k >> 1] = (uint8_t)(packed[k >> 1] | (nib << 4));
            else
                packed[k >> 1] = nib;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Thread plumbing: split [0, T) into contiguous ranges.                  */

typedef struct {
    int op; /* 0 transform, 1 quantize, 2 transform+quant, 3 dequant+inverse */
    int64_t t0, t1;
    int n1, n2;
    const uint16_t *x;
    const double *P1, *P2;
    const float *cinv;
    double alpha;
    const double *y_in;
    double *y_out;
    uint8_t *packed;
    int8_t *codes;
    double *scale64;
    float *scale32;
    double *dist;
    const uint8_t *q_in;
    const float *scale_in;
    const double *P1inv, *P2inv;
    const double *c;
    int status;
} job_t;

static void dequant_inverse_token(const uint8_t *q, float scale, const double *P1inv,
                                  const double *P2inv, const double *c, int n1, int n2,
                                  double *yq, double *W, double *xhat)
{
    int n = n1 * n2;
    for (int k = 0; k < n; ++k) {
        uint8_t byte = q[k >> 1];
        int nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
        int code = nib >= 8 ? nib - 16 : nib;
        yq[k] = (double)code * (double)scale;
    }
    /* x^~ = P1^-T Y^ P2^-1: first W = Y^ P2inv, then P1inv^T W. */
    for (int a = 0; a < n1; ++a)
        for (int j = 0; j < n2; ++j) {
            double acc = 0.0;
            for (int b = 0; b < n2; ++b)
                acc += yq[a * n2 + b] * P2inv[b * n2 + j];
            W[a * n2 + j] = acc;
        }
    for (int i = 0; i < n1; ++i)
        for (int j = 0; j < n2; ++j) {
            double acc = 0.0;
            for (int a = 0; a < n1; ++a)
                acc += P1inv[a * n1 + i] * W[a * n2 + j];
            xhat[i * n2 + j] = acc * (c ? c[i * n2 + j] : 1.0);
        }
}

static void *run_job(void *arg)
{
    job_t *jb = (job_t *)arg;
    int n = jb->n1 * jb->n2;
    double *buf = (double *)malloc(sizeof(double) * (size_t)n * 3);
    if (!buf) {
        jb->status = KQO_ERR_NOMEM;
        return NULL;
    }
    double *xs = buf, *Z = buf + n, *y = buf + 2 * (size_t)n;
    for (int64_t t = jb->t0; t < jb->t1; ++t) {
        size_t off = (size_t)t * (size_t)n;
        switch (jb->op) {
        case 0:
            transform_token(jb->x + off, jb->P1, jb->P2, jb->cinv, jb->n1, jb->n2, xs, Z,
                            jb->y_out + off);
            break;
        case 1:
            quantize_token(jb->y_in + off, n, jb->alpha, jb->codes ? jb->codes + off : NULL,
                           jb->packed ? jb->packed + off / 2 : NULL,
                           jb->scale64 ? jb->scale64 + t : NULL,
                           jb->scale32 ? jb->scale32 + t : NULL,
                           jb->dist ? jb->dist + off : NULL);
            break;
        case 2:
            transform_token(jb->x + off, jb->P1, jb->P2, jb->cinv, jb->n1, jb->n2, xs, Z, y);
            quantize_token(y, n, jb->alpha, jb->codes ? jb->codes + off : NULL,
                           jb->packed ? jb->packed + off / 2 : NULL,
                           jb->scale64 ? jb->scale64 + t : NULL,
                           jb->scale32 ? jb->scale32 + t : NULL,
                           jb->dist ? jb->dist + off : NULL);
            break;
        default:
            dequant_inverse_token(jb->q_in + off / 2, jb->scale_in[t], jb->P1inv, jb->P2inv,
                                  jb->c, jb->n1, jb->n2, xs, Z, jb->y_out + off);
            break;
        }
    }
    free(buf);
    jb->status = KQO_OK;
    return NULL;
}

static int run_threads(job_t proto, int64_t T, int nthreads)
{
    if (T <= 0)
        return KQO_OK;
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > T)
        nthreads = (int)T;
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return KQO_ERR_NOMEM;
    }
    int64_t per = T / nthreads, rem = T % nthreads, start = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = proto;
        jobs[i].t0 = start;
        start += per + (i < rem ? 1 : 0);
        jobs[i].t1 = start;
        jobs[i].status = KQO_ERR_ARG;
    }
    int launched = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, run_job, &jobs[i]) != 0)
            break;
        launched = i;
    }
    run_job(&jobs[0]);
    for (int i = 1; i <= launched; ++i)
        pthread_join(th[i], NULL);
    /* Ranges whose thread could not be created run here. */
    for (int i = launched + 1; i < nthreads; ++i)
        run_job(&jobs[i]);
    int st = KQO_OK;
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status != KQO_OK)
            st = jobs[i].status;
    free(jobs);
    free(th);
    return st;
}

static double *widen_factor(const uint16_t *P, int k)
{
    double *d = (double *)malloc(sizeof(double) * (size_t)k * (size_t)k);
    if (d)
        for (int i = 0; i < k * k; ++i)
            d[i] = bf16_to_double(P[i]);
    return d;
}

static int check_shape(int64_t T, int n1, int n2)
{
    if (T < 0 || n1 <= 0 || n2 <= 0 || ((int64_t)n1 * n2) % 2 != 0)
        return KQO_ERR_ARG;
    return KQO_OK;
}

/* y[T, n] (fp64) = transform of x[T, n] (bf16 bits). */
int kqo_transform(const uint16_t *x, const uint16_t *P1, const uint16_t *P2, const float *cinv,
                  int64_t T, int n1, int n2, double *y, int nthreads)
{
    if (check_shape(T, n1, n2) || (T > 0 && (!x || !P1 || !P2 || !y)))
        return KQO_ERR_ARG;
    double *p1 = widen_factor(P1, n1), *p2 = widen_factor(P2, n2);
    if (!p1 || !p2) {
        free(p1);
        free(p2);
        return KQO_ERR_NOMEM;
    }
    job_t jb;
    memset(&jb, 0, sizeof jb);
    jb.op = 0;
    jb.n1 = n1;
    jb.n2 = n2;
    jb.x = x;
    jb.P1 = p1;
    jb.P2 = p2;
    jb.cinv = cinv;
    jb.y_out = y;
    int st = run_threads(jb, T, nthreads);
    free(p1);
    free(p2);
    return st;
}

/* Quantise fp64 rows y[T, n].  Any output pointer may be NULL. */
int kqo_quantize(const double *y, int64_t T, int n, float alpha, int8_t *codes, uint8_t *packed,
                 double *scale64, float *scale32, double *dist, int nthreads)
{
    if (T < 0 || n <= 0 || n % 2 || (T > 0 && !y))
        return KQO_ERR_ARG;
    job_t jb;
    memset(&jb, 0, sizeof jb);
    jb.op = 1;
    jb.n1 = 1;
    jb.n2 = n;
    jb.alpha = (double)alpha;
    jb.y_in = y;
    jb.codes = codes;
    jb.packed = packed;
    jb.scale64 = scale64;
    jb.scale32 = scale32;
    jb.dist = dist;
    return run_threads(jb, T, nthreads);
}

/* Transform + quantise token by token without storing y. */
int kqo_transform_quant(const uint16_t *x, const uint16_t *P1, const uint16_t *P2,
                        const float *cinv, float alpha, int64_t T, int n1, int n2,
                        uint8_t *packed, float *scale32, int8_t *codes, double *scale64,
                        double *dist, int nthreads)
{
    if (check_shape(T, n1, n2) || (T > 0 && (!x || !P1 || !P2)))
        return KQO_ERR_ARG;
    double *p1 = widen_factor(P1, n1), *p2 = widen_factor(P2, n2);
    if (!p1 || !p2) {
        free(p1);
        free(p2);
        return KQO_ERR_NOMEM;
    }
    job_t jb;
    memset(&jb, 0, sizeof jb);
    jb.op = 2;
    jb.n1 = n1;
    jb.n2 = n2;
    jb.x = x;
    jb.P1 = p1;
    jb.P2 = p2;
    jb.cinv = cinv;
    jb.alpha = (double)alpha;
    jb.packed = packed;
    jb.scale32 = scale32;
    jb.codes = codes;
    jb.scale64 = scale64;
    jb.dist = dist;
    int st = run_threads(jb, T, nthreads);
    free(p1);
    free(p2);
    return st;
}

/* x^[T, n] = ((q * s) (P1^-1 (x) P2^-1)) * c, with fp64 inverse factors. */
int kqo_dequant_inverse(const uint8_t *q, const float *scale, const double *P1inv,
                        const double *P2inv, const double *c, int64_t T, int n1, int n2,
                        double *xhat, int nthreads)
{
    if (check_shape(T, n1, n2) || (T > 0 && (!q || !scale || !P1inv || !P2inv || !xhat)))
        return KQO_ERR_ARG;
    job_t jb;
    memset(&jb, 0, sizeof jb);
    jb.op = 3;
    jb.n1 = n1;
    jb.n2 = n2;
    jb.q_in = q;
    jb.scale_in = scale;
    jb.P1inv = P1inv;
    jb.P2inv = P2inv;
    jb.c = c;
    jb.y_out = xhat;
    return run_threads(jb, T, nthreads);
}
