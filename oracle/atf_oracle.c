/*
 * atf_oracle.c -- plain fp64 CPU oracle for causal (GQA) attention with a
 * distance window per RoPE frequency pair.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
 * the benchmark's CPU-baseline leg load this file.  It shares no code, header,
 * table or helper with the CUDA library; it is deliberately slow and written
 * to be checked by eye against the method's definition.
 *
 * Source of the method:
 *   "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent"
 *   (sudo-ai.de), section "Was ATFlash anders macht": RoPE encodes position as
 *   2-D rotations at several frequencies; every frequency pair gets its own
 *   distance window derived from its wavelength, beyond which that pair's
 *   query-key products are left out, so a far key stays reachable through the
 *   slow (low-frequency) pairs.  Section "Die Zahlen - und ihre Grenze": the
 *   online-softmax recurrence is left unchanged.
 *
 * Definition computed here (the reading of "a proportional distance" that
 * this library implements):
 *   omega_i = theta^(-2i/d),  lambda_i = 2*pi/omega_i,  W_i = ceil(alpha*lambda_i)
 *   s(m,n)  = (1/sqrt d) * sum_{i : m-n <= W_i} (q~_{2i} k~_{2i} + q~_{2i+1} k~_{2i+1})
 *   an empty sum gives the logit 0 (kept in the softmax, not masked);
 *   out_m   = sum_{n<=m} softmax_n(s(m,.)) v_n.
 * q~, k~ are q, k rotated by RoPE at their absolute positions.  Pair i is the
 * two dimensions (a_i, b_i): (2i, 2i+1) in the interleaved convention the
 * method's formula is written in, (i, i + d/2) in the rotate-half convention
 * (the one of NeoX-style checkpoints such as the Qwen2.5 family the pages
 * measure on), `pairing` 0 and 1 below:
 *   x~_{a_i} = x_{a_i} cos(p omega_i) - x_{b_i} sin(p omega_i)
 *   x~_{b_i} = x_{a_i} sin(p omega_i) + x_{b_i} cos(p omega_i)
 * and the pair product in the logit is q~_{a_i} k~_{a_i} + q~_{b_i} k~_{b_i}.
 * GQA: query head h reads key/value head floor(h / (Hq/Hkv)).
 * alpha = +inf gives W_i = INT64_MAX (plain causal RoPE attention).
 *
 * Inputs may be fp32 or bf16 (raw 16-bit patterns); both are widened to fp64
 * exactly before any arithmetic.  All arithmetic is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_F32 1
#define ORACLE_BF16 0

static double widen(const void *base, long long idx, int dtype) {
    if (dtype == ORACLE_F32) return (double)((const float *)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* omega_i and W_i for i < d/2. */
void oracle_windows(int d, double theta, double alpha, long long *W, double *omega) {
    const double two_pi = 6.283185307179586476925286766559;
    for (int i = 0; i < d / 2; ++i) {
        double om = pow(theta, -2.0 * (double)i / (double)d);
        if (omega) omega[i] = om;
        if (isinf(alpha)) {
            W[i] = INT64_MAX;
        } else {
            double lambda = two_pi / om;
            double w = ceil(alpha * lambda);
            W[i] = (w >= 9.2e18) ? INT64_MAX : (long long)w;
        }
    }
}

/* The two dimensions of frequency pair i. */
static int pair_a(int i, int d, int pairing) { return pairing ? i : 2 * i; }
static int pair_b(int i, int d, int pairing) { return pairing ? i + d / 2 : 2 * i + 1; }

/* RoPE of one head vector x (length d) at position p, into y. */
static void rope_vec(const double *x, double *y, long long p, const double *omega, int d, int pairing) {
    for (int i = 0; i < d / 2; ++i) {
        const int a = pair_a(i, d, pairing), b = pair_b(i, d, pairing);
        double phi = (double)p * omega[i];
        double c = cos(phi), s = sin(phi);
        y[a] = x[a] * c - x[b] * s;
        y[b] = x[a] * s + x[b] * c;
    }
}

/* Rotate x[b][t][h][d] (dtype) at positions pos0 + t; y is fp64, same layout. */
void oracle_rope(const void *x, int dtype, double *y, int batch, int seq, int heads, int d,
                 long long pos0, double theta, int pairing) {
    double *omega = malloc(sizeof(double) * (size_t)(d / 2));
    long long *W = malloc(sizeof(long long) * (size_t)(d / 2));
    double *xv = malloc(sizeof(double) * (size_t)d);
    oracle_windows(d, theta, INFINITY, W, omega);
    for (int b = 0; b < batch; ++b)
        for (int t = 0; t < seq; ++t)
            for (int h = 0; h < heads; ++h) {
                long long base = (((long long)b * seq + t) * heads + h) * d;
                for (int e = 0; e < d; ++e) xv[e] = widen(x, base + e, dtype);
                rope_vec(xv, y + base, pos0 + t, omega, d, pairing);
            }
    free(omega);
    free(W);
    free(xv);
}

/* ------------------------------------------------------------------------- */
/* Prefill: rows m = q_offset + t for t in [0, q_len); keys n in [0, m].      */

typedef struct {
    const void *q, *k, *v;
    int dtype;
    double *out;
    int batch, q_len, kv_len, Hq, Hkv, d;
    long long q_offset;
    const long long *W;
    const double *omega;
    int pairing;     /* 0: pairs (2i, 2i+1); 1: pairs (i, i + d/2) */
    const int *rows; /* NULL: all t */
    int n_rows;
    const double *k64;  /* keys rotated once up front (fp64), or NULL: k is already rotated */
    long long next;     /* work counter */
    pthread_mutex_t lock;
    unsigned long long skipped;
} job_t;

static void one_row(job_t *J, int b, int h, int t, double *qt, double *kt, double *logit,
                    unsigned long long *skipped) {
    const int d = J->d, G = J->Hq / J->Hkv, hk = h / G;
    const long long m = J->q_offset + t;
    double *qraw = malloc(sizeof(double) * (size_t)d);
    long long qbase = (((long long)b * J->q_len + t) * J->Hq + h) * d;
    for (int e = 0; e < d; ++e) qraw[e] = widen(J->q, qbase + e, J->dtype);
    rope_vec(qraw, qt, m, J->omega, d, J->pairing);
    free(qraw);

    long long nmax = m;
    if (nmax > J->kv_len - 1) nmax = J->kv_len - 1;
    double mx = -INFINITY;
    for (long long n = 0; n <= nmax; ++n) {
        long long kbase = (((long long)b * J->kv_len + n) * J->Hkv + hk) * d;
        if (J->k64) {
            for (int e = 0; e < d; ++e) kt[e] = J->k64[kbase + e];
        } else {
            for (int e = 0; e < d; ++e) kt[e] = widen(J->k, kbase + e, J->dtype);
        }
        long long delta = m - n;
        double acc = 0.0;
        for (int i = 0; i < d / 2; ++i) {
            const int a = pair_a(i, d, J->pairing), bb = pair_b(i, d, J->pairing);
            if (delta <= J->W[i])
                acc += qt[a] * kt[a] + qt[bb] * kt[bb];
            else
                *skipped += 1;
        }
        logit[n] = acc / sqrt((double)d);
        if (logit[n] > mx) mx = logit[n];
    }
    double *o = J->out + (((long long)b * J->q_len + t) * J->Hq + h) * d;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    double den = 0.0;
    for (long long n = 0; n <= nmax; ++n) {
        double p = exp(logit[n] - mx);
        den += p;
        long long vbase = (((long long)b * J->kv_len + n) * J->Hkv + hk) * d;
        for (int e = 0; e < d; ++e) o[e] += p * widen(J->v, vbase + e, J->dtype);
    }
    for (int e = 0; e < d; ++e) o[e] /= den;
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    const int d = J->d;
    double *qt = malloc(sizeof(double) * (size_t)d);
    double *kt = malloc(sizeof(double) * (size_t)d);
    double *logit = malloc(sizeof(double) * (size_t)(J->kv_len > 0 ? J->kv_len : 1));
    unsigned long long skipped = 0;
    const long long rows_per_bh = J->rows ? J->n_rows : J->q_len;
    const long long total = (long long)J->batch * J->Hq * rows_per_bh;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        long long w = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (w >= total) break;
        int r = (int)(w % rows_per_bh);
        int h = (int)((w / rows_per_bh) % J->Hq);
        int b = (int)(w / rows_per_bh / J->Hq);
        int t = J->rows ? J->rows[r] : r;
        one_row(J, b, h, t, qt, kt, logit, &skipped);
    }
    pthread_mutex_lock(&J->lock);
    J->skipped += skipped;
    pthread_mutex_unlock(&J->lock);
    free(qt);
    free(kt);
    free(logit);
    return NULL;
}

static unsigned long long run_jobs(job_t *J, int nthreads) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    pthread_mutex_init(&J->lock, NULL);
    J->next = 0;
    J->skipped = 0;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->skipped;
}

/*
 * Prefill oracle.  q: [batch][q_len][Hq][d], k, v: [batch][kv_len][Hkv][d],
 * out: fp64 [batch][q_len][Hq][d] (rows not in `rows` are left untouched).
 * Query t sits at absolute position q_offset + t; key n at position n.
 * Returns the number of (query head, query, key, pair) quadruples whose pair
 * was outside its window, over the rows computed.
 */
unsigned long long oracle_prefill(const void *q, const void *k, const void *v, int dtype, double *out,
                                  int batch, int q_len, int kv_len, long long q_offset, int Hq, int Hkv,
                                  int d, double theta, double alpha, const int *rows, int n_rows,
                                  int nthreads, int pairing) {
    long long *W = malloc(sizeof(long long) * (size_t)(d / 2));
    double *omega = malloc(sizeof(double) * (size_t)(d / 2));
    oracle_windows(d, theta, alpha, W, omega);
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dtype = dtype; J.out = out;
    J.batch = batch; J.q_len = q_len; J.kv_len = kv_len; J.Hq = Hq; J.Hkv = Hkv; J.d = d;
    J.q_offset = q_offset; J.W = W; J.omega = omega; J.rows = rows; J.n_rows = n_rows;
    J.pairing = pairing;
    /* keys are rotated once, at their absolute positions 0..kv_len-1 */
    double *k64 = malloc(sizeof(double) * (size_t)batch * (size_t)kv_len * (size_t)Hkv * (size_t)d);
    oracle_rope(k, dtype, k64, batch, kv_len, Hkv, d, 0, theta, pairing);
    J.k64 = k64;
    unsigned long long s = run_jobs(&J, nthreads);
    free(k64);
    free(W);
    free(omega);
    return s;
}

/*
 * Decode oracle: one new query per sequence.  q: raw (unrotated) [batch][Hq][d];
 * k_rot: keys ALREADY rotated (same pairing), [batch][n_cache][Hkv][d]; v: [batch][n_cache][Hkv][d];
 * kv_len[b] <= n_cache keys are live; the query sits at position kv_len[b]-1.
 * out: fp64 [batch][Hq][d].  Returns the skipped pair count.
 */
unsigned long long oracle_decode(const void *q, const void *k_rot, const void *v, int dtype, double *out,
                                 int batch, long long n_cache, const long long *kv_len, int Hq, int Hkv,
                                 int d, double theta, double alpha, int nthreads, int pairing) {
    long long *W = malloc(sizeof(long long) * (size_t)(d / 2));
    double *omega = malloc(sizeof(double) * (size_t)(d / 2));
    oracle_windows(d, theta, alpha, W, omega);
    unsigned long long total = 0;
    const int esz = dtype == ORACLE_F32 ? 4 : 2;
    for (int b = 0; b < batch; ++b) {
        job_t J;
        memset(&J, 0, sizeof J);
        /* one sequence at a time, as a one-row prefill whose query sits at kv_len-1 */
        J.q = (const char *)q + (size_t)b * Hq * d * esz;
        J.k = (const char *)k_rot + (size_t)b * n_cache * Hkv * d * esz;
        J.v = (const char *)v + (size_t)b * n_cache * Hkv * d * esz;
        J.dtype = dtype;
        J.out = out + (size_t)b * Hq * d;
        J.batch = 1; J.q_len = 1; J.kv_len = (int)kv_len[b]; J.Hq = Hq; J.Hkv = Hkv; J.d = d;
        J.q_offset = kv_len[b] - 1; J.W = W; J.omega = omega; J.rows = NULL; J.n_rows = 0;
        J.k64 = NULL;
        J.pairing = pairing;
        total += run_jobs(&J, nthreads);
    }
    free(W);
    free(omega);
    return total;
}
