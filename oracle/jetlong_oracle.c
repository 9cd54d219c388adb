/*
 * jetlong_oracle.c -- TEST INFRASTRUCTURE ONLY (not part of the product path).
 *
 * A plain, slow, fp64 CPU oracle for Jet-Long's dynamic bifocal RoPE causal
 * attention.  Only the test suite, the package smoke check and the bench's
 * CPU-baseline leg may load this file's library.  It shares no code, header,
 * table or constant with the CUDA library: it is written from the method's
 * statement alone, with one explicit rotation per (query, key) pair.
 *
 * Sources (page: "Jet-Long: Efficient Long-Context Extension with Dynamic
 * Bifocal RoPE", gist.science/it/paper/2607.07740):
 *   - Metodologia, 1 "RoPE Bifocale Dinamico": a local window of size w0 keeps
 *     classic RoPE; positions beyond it use f(x) = floor(x / G) with
 *     G = max(1, ceil(L / w_pretrained)) from the current length L
 *     (display equation for G; the floor-division sentence after it).
 *   - Metodologia, 2 "Meccanismi di Efficienza dell'Inferenza": RoPE rotations
 *     compose additively; the inclusion-exclusion merge yields the exact
 *     distance-routed output (one softmax over all routed pairs).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - local iff i - j < w0 (i - j == w0 is remote);
 *   - the remote branch uses exactly f(i) and f(j), no extra offset;
 *   - RoPE frequencies theta_m = rope_theta^(-2m/d), m < d/2, half-split
 *     pairing (m, m + d/2) as in the Qwen3 models the pages evaluate;
 *   - grouped-query mapping: q head h reads kv head h / (Hq / Hkv);
 *   - softmax(scale * logit) in base e, scale given by the caller.
 *
 * Everything is fp64.  Inputs are widened exactly from bf16 bits or fp32.
 * cos/sin of (position * theta_m) may be cached per position (the values are
 * the same libm results as an uncached call); the rotation itself is applied
 * explicitly for every (i, j) pair.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define JLO_IN_BF16 0
#define JLO_IN_FP32 1

/* G = max(1, ceil(L / w_pretrained)); page 1, Metodologia 1, display eq. */
int64_t jlo_group_size(int64_t L, int64_t w_pretrained)
{
    if (L < 0 || w_pretrained < 1) return -1;
    int64_t g = L / w_pretrained;
    if (g * w_pretrained < L) g += 1; /* ceiling */
    if (g < 1) g = 1;
    return g;
}

/* f(x) = floor(x / G) for x >= 0, G >= 1; page 1, Metodologia 1. */
int64_t jlo_remote_position(int64_t x, int64_t G)
{
    return x / G;
}

/* theta_m = rope_theta^(-2m/d) (standard RoPE frequency; reading c3). */
static double inv_freq(int m, int d, double rope_theta)
{
    return pow(rope_theta, -2.0 * (double)m / (double)d);
}

/* Rotate one d-vector to position p, half-split pairing (m, m + d/2):
 *   y_m       = x_m cos(p theta_m) - x_{m+d/2} sin(p theta_m)
 *   y_{m+d/2} = x_m sin(p theta_m) + x_{m+d/2} cos(p theta_m)          */
void jlo_rotate(const double* x, double* y, int d, int64_t p, double rope_theta)
{
    int h = d / 2;
    for (int m = 0; m < h; ++m) {
        double phi = (double)p * inv_freq(m, d, rope_theta);
        double c = cos(phi), s = sin(phi);
        double a = x[m], b = x[m + h];
        y[m] = a * c - b * s;
        y[m + h] = a * s + b * c;
    }
}

/* Unscaled logit of one (query at i, key at j) pair, routed by distance:
 * local (i - j < w0) -> classic RoPE at i and j; remote -> RoPE at f(i), f(j). */
double jlo_pair_logit(const double* q, const double* k, int d, int64_t i, int64_t j,
                      int64_t w0, int64_t G, double rope_theta)
{
    double qr[512], kr[512];
    if (d > 512) return NAN;
    int64_t pq, pk;
    if (i - j < w0) { pq = i; pk = j; }
    else { pq = jlo_remote_position(i, G); pk = jlo_remote_position(j, G); }
    jlo_rotate(q, qr, d, pq, rope_theta);
    jlo_rotate(k, kr, d, pk, rope_theta);
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += qr[t] * kr[t];
    return acc;
}

static double widen(const void* base, int dtype, size_t idx)
{
    if (dtype == JLO_IN_FP32) return (double)((const float*)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* One routed attention row.                                                 */

typedef struct {
    /* geometry */
    int d, w0;
    int64_t G;
    double scale;
    int in_dtype;
    /* cos/sin cache for positions [0, npos): cs[(p * h + m) * 2 + {0,1}] */
    const double* cs;
    int64_t npos;
    /* 1: key rows are stored already rotated to their exact positions j (a
     * standard RoPE cache); 0: raw key rows */
    int rope_cache;
} row_ctx;

static void rotate_cached(const row_ctx* c, const double* x, double* y, int64_t p)
{
    int h = c->d / 2;
    const double* t = c->cs + (size_t)p * h * 2;
    for (int m = 0; m < h; ++m) {
        double cc = t[2 * m], ss = t[2 * m + 1];
        double a = x[m], b = x[m + h];
        y[m] = a * cc - b * ss;
        y[m + h] = a * ss + b * cc;
    }
}

/* Rotation by -p (the inverse of the rotation to p): cos(-a) = cos a,
 * sin(-a) = -sin a. */
static void unrotate_cached(const row_ctx* c, const double* x, double* y, int64_t p)
{
    int h = c->d / 2;
    const double* t = c->cs + (size_t)p * h * 2;
    for (int m = 0; m < h; ++m) {
        double cc = t[2 * m], ss = t[2 * m + 1];
        double a = x[m], b = x[m + h];
        y[m] = a * cc + b * ss;
        y[m + h] = -a * ss + b * cc;
    }
}

/* q: pointer to the raw query row; keys/values: base of this kv head, row j
 * at element offset j * d.  Query position i, keys j in [0, i].          */
static void attend_row(const row_ctx* c, const void* q, size_t q_off,
                       const void* kbase, const void* vbase, size_t kv_off,
                       int64_t i, double* logit, double* out, double* lse)
{
    int d = c->d;
    double qraw[512], qe[512], qm[512], kraw[512], kr[512];
    for (int t = 0; t < d; ++t) qraw[t] = widen(q, c->in_dtype, q_off + t);
    rotate_cached(c, qraw, qe, i);                               /* exact  */
    rotate_cached(c, qraw, qm, jlo_remote_position(i, c->G));    /* remote */

    double mx = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
        size_t off = kv_off + (size_t)j * d;
        for (int t = 0; t < d; ++t) kraw[t] = widen(kbase, c->in_dtype, off + t);
        const double* qq;
        if (i - j < (int64_t)c->w0) {                  /* local branch  */
            if (c->rope_cache) memcpy(kr, kraw, sizeof(double) * (size_t)d);  /* already at j */
            else rotate_cached(c, kraw, kr, j);
            qq = qe;
        } else {                                       /* remote branch */
            int64_t fj = jlo_remote_position(j, c->G);
            /* a key stored at j moves to f(j) by the extra rotation
             * f(j) - j <= 0 (rotations compose additively) */
            if (c->rope_cache) unrotate_cached(c, kraw, kr, j - fj);
            else rotate_cached(c, kraw, kr, fj);
            qq = qm;
        }
        double a = 0.0;
        for (int t = 0; t < d; ++t) a += qq[t] * kr[t];
        logit[j] = c->scale * a;
        if (logit[j] > mx) mx = logit[j];
    }
    double sum = 0.0;
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int64_t j = 0; j <= i; ++j) {
        double p = exp(logit[j] - mx);
        sum += p;
        size_t off = kv_off + (size_t)j * d;
        for (int t = 0; t < d; ++t) out[t] += p * widen(vbase, c->in_dtype, off + t);
    }
    for (int t = 0; t < d; ++t) out[t] /= sum;
    /* log of the softmax denominator: log sum_j exp(scale * a_ij) */
    if (lse) *lse = mx + log(sum);
}

/* cos/sin of p * theta_m for positions [0, npos): the same libm values as
 * jlo_rotate computes for each position (theta_m evaluated once per m, the
 * product and cos/sin once per (p, m)).  Filled by the host's threads over
 * disjoint position ranges; each entry is computed exactly as a serial loop
 * would compute it. */
typedef struct {
    double* cs;
    const double* freq;
    int h;
    int64_t p0, p1;
} cs_part;

static void* fill_cs(void* arg)
{
    cs_part* P = (cs_part*)arg;
    for (int64_t p = P->p0; p < P->p1; ++p)
        for (int m = 0; m < P->h; ++m) {
            double phi = (double)p * P->freq[m];
            P->cs[((size_t)p * P->h + m) * 2] = cos(phi);
            P->cs[((size_t)p * P->h + m) * 2 + 1] = sin(phi);
        }
    return NULL;
}

static double* build_cs_threads(int d, int64_t npos, double rope_theta, int nthreads)
{
    int h = d / 2;
    double freq[256];
    for (int m = 0; m < h; ++m) freq[m] = inv_freq(m, d, rope_theta);
    double* cs = (double*)malloc(sizeof(double) * 2 * (size_t)h * (size_t)(npos > 0 ? npos : 1));
    if (!cs) return NULL;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads * 1024 > npos) nthreads = (int)(npos / 1024) + 1;
    cs_part part[256];
    pthread_t th[256];
    int started[256] = {0};
    for (int t = 0; t < nthreads; ++t) {
        part[t].cs = cs; part[t].freq = freq; part[t].h = h;
        part[t].p0 = npos * t / nthreads;
        part[t].p1 = npos * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t) started[t] = pthread_create(&th[t], NULL, fill_cs, &part[t]) == 0;
    fill_cs(&part[0]);
    for (int t = 1; t < nthreads; ++t) {
        if (started[t]) pthread_join(th[t], NULL);
        else fill_cs(&part[t]);
    }
    return cs;
}

static double* build_cs(int d, int64_t npos, double rope_theta)
{
    return build_cs_threads(d, npos, rope_theta, 0);
}

/* ------------------------------------------------------------------------ */
/* Threaded drivers.                                                         */

typedef struct {
    row_ctx c;
    const void *q, *k, *v;
    int B, Hq, Hkv, L, Lkv; /* Lkv: row stride (in rows) of the key/value arrays */
    int q_is_decode;        /* 1: q is [B,Hq,d] and the query sits at i = L-1 */
    const int32_t* rows;    /* n triples (b, h, i) */
    int64_t n;
    double* out;
    double* lse;  /* optional: one log-sum-exp per row */
    int64_t next; /* work counter */
    int status;
} job_t;

static void* worker(void* arg)
{
    job_t* J = (job_t*)arg;
    int d = J->c.d;
    double* logit = (double*)malloc(sizeof(double) * ((size_t)J->L + 1));
    if (!logit) { __atomic_store_n(&J->status, -2, __ATOMIC_RELAXED); return NULL; }
    int group = J->Hq / J->Hkv;
    for (;;) {
        int64_t r = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (r >= J->n) break;
        int b = J->rows[3 * r], h = J->rows[3 * r + 1];
        int64_t i = J->rows[3 * r + 2];
        int kvh = h / group;
        size_t q_off = J->q_is_decode ? ((size_t)b * J->Hq + h) * d
                                      : (((size_t)b * J->Hq + h) * J->L + i) * d;
        size_t kv_off = ((size_t)b * J->Hkv + kvh) * (size_t)J->Lkv * d;
        attend_row(&J->c, J->q, q_off, J->k, J->v, kv_off, i, logit, J->out + (size_t)r * d,
                   J->lse ? J->lse + r : NULL);
    }
    free(logit);
    return NULL;
}

static int run_job(job_t* J, int nthreads)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if ((int64_t)nthreads > J->n) nthreads = J->n > 0 ? (int)J->n : 1;
    pthread_t th[1024];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, worker, J) == 0) started = t; else break;
    worker(J);
    for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
    return J->status;
}

static int check_common(int B, int Hq, int Hkv, int L, int d, int w0, int w_pretrained,
                        double rope_theta, int in_dtype)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || d < 2 || d > 512 || (d & 1)) return -1;
    if (Hq % Hkv) return -1;
    if (w0 < 0 || w_pretrained < 1 || !(rope_theta > 0.0)) return -1;
    if (in_dtype != JLO_IN_BF16 && in_dtype != JLO_IN_FP32) return -1;
    return 0;
}

/* Prefill rows: out[r, :] = routed attention output of query (b, h, i) for
 * the n triples in rows; q [B,Hq,L,d], k/v [B,Hkv,L,d], one G for the call
 * computed from L.  Returns 0 on success. */
int jlo_prefill_rows_lse(const void* q, const void* k, const void* v, int in_dtype,
                         int B, int Hq, int Hkv, int L, int d, int w0, int w_pretrained,
                         double rope_theta, double scale,
                         const int32_t* rows, int64_t n, double* out, double* lse, int nthreads);

int jlo_prefill_rows(const void* q, const void* k, const void* v, int in_dtype,
                     int B, int Hq, int Hkv, int L, int d, int w0, int w_pretrained,
                     double rope_theta, double scale,
                     const int32_t* rows, int64_t n, double* out, int nthreads)
{
    return jlo_prefill_rows_lse(q, k, v, in_dtype, B, Hq, Hkv, L, d, w0, w_pretrained, rope_theta,
                                scale, rows, n, out, NULL, nthreads);
}

/* The same rows plus lse[r] = log sum_j exp(scale * a_ij) of each row (the
 * statistic the pages' inclusion-exclusion merge combines, Metodologia 2). */
int jlo_prefill_rows_lse(const void* q, const void* k, const void* v, int in_dtype,
                         int B, int Hq, int Hkv, int L, int d, int w0, int w_pretrained,
                         double rope_theta, double scale,
                         const int32_t* rows, int64_t n, double* out, double* lse, int nthreads)
{
    if (check_common(B, Hq, Hkv, L, d, w0, w_pretrained, rope_theta, in_dtype)) return -1;
    for (int64_t r = 0; r < n; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= Hq ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= L)
            return -1;
    /* every position a row reaches (i, j <= i and their aliases) is <= the
     * largest query position asked for */
    int64_t npos = 1;
    for (int64_t r = 0; r < n; ++r)
        if ((int64_t)rows[3 * r + 2] + 1 > npos) npos = (int64_t)rows[3 * r + 2] + 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.c.d = d; J.c.w0 = w0; J.c.G = jlo_group_size(L, w_pretrained);
    J.c.scale = scale; J.c.in_dtype = in_dtype; J.c.npos = npos;
    J.c.cs = build_cs_threads(d, npos, rope_theta, nthreads);
    if (!J.c.cs) return -2;
    J.q = q; J.k = k; J.v = v; J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.L = L; J.Lkv = L;
    J.rows = rows; J.n = n; J.out = out; J.lse = lse;
    int st = run_job(&J, nthreads);
    free((void*)J.c.cs);
    return st;
}

static int decode_impl(const void* q, const void* kcache, const void* vcache, int in_dtype,
                       int B, int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
                       double rope_theta, double scale, double* out, int nthreads, int rope_cache);

/* Decode: one new query per (b, h) at position i = L - 1 attending keys
 * [0, L) of caches [B,Hkv,Lcap,d] holding raw key rows; G from this L.
 * out is [B,Hq,d]. */
int jlo_decode(const void* q, const void* kcache, const void* vcache, int in_dtype,
               int B, int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
               double rope_theta, double scale, double* out, int nthreads)
{
    return decode_impl(q, kcache, vcache, in_dtype, B, Hq, Hkv, L, Lcap, d, w0, w_pretrained,
                       rope_theta, scale, out, nthreads, 0);
}

/* The same decode over a standard RoPE cache: row j of kcache holds the key
 * already rotated to its exact position j.  Page 1, Metodologia 2: the cache
 * keeps the base rotation; a remote key is moved to f(j) by the rotation
 * f(j) - j (rotations compose additively), a local key is used as stored. */
int jlo_decode_rope_cache(const void* q, const void* kcache, const void* vcache, int in_dtype,
                          int B, int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
                          double rope_theta, double scale, double* out, int nthreads)
{
    return decode_impl(q, kcache, vcache, in_dtype, B, Hq, Hkv, L, Lcap, d, w0, w_pretrained,
                       rope_theta, scale, out, nthreads, 1);
}

/* Rotate every row j of x [nplanes][nrows][d] to position j (fp64 out):
 * builds a standard RoPE key cache from raw keys. */
int jlo_rotate_rows(const void* x, int in_dtype, int64_t nplanes, int64_t nrows, int d,
                    double rope_theta, double* out)
{
    if (nplanes < 1 || nrows < 1 || d < 2 || d > 512 || (d & 1) || !(rope_theta > 0.0)) return -1;
    if (in_dtype != JLO_IN_BF16 && in_dtype != JLO_IN_FP32) return -1;
    /* per-position cos/sin, computed once (the same libm values as jlo_rotate) */
    row_ctx c;
    memset(&c, 0, sizeof c);
    c.d = d;
    c.npos = nrows;
    c.cs = build_cs(d, nrows, rope_theta);
    if (!c.cs) return -2;
    double xr[512];
    for (int64_t pl = 0; pl < nplanes; ++pl)
        for (int64_t j = 0; j < nrows; ++j) {
            size_t off = ((size_t)pl * (size_t)nrows + (size_t)j) * (size_t)d;
            for (int t = 0; t < d; ++t) xr[t] = widen(x, in_dtype, off + (size_t)t);
            rotate_cached(&c, xr, out + off, j);
        }
    free((void*)c.cs);
    return 0;
}

static int decode_impl(const void* q, const void* kcache, const void* vcache, int in_dtype,
                       int B, int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
                       double rope_theta, double scale, double* out, int nthreads, int rope_cache)
{
    if (check_common(B, Hq, Hkv, L, d, w0, w_pretrained, rope_theta, in_dtype)) return -1;
    if (Lcap < L) return -1;
    int64_t n = (int64_t)B * Hq;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * 3 * (size_t)n);
    if (!rows) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t r = (size_t)b * Hq + h;
            rows[3 * r] = b; rows[3 * r + 1] = h; rows[3 * r + 2] = L - 1;
        }
    job_t J;
    memset(&J, 0, sizeof J);
    J.c.d = d; J.c.w0 = w0; J.c.G = jlo_group_size(L, w_pretrained);
    J.c.scale = scale; J.c.in_dtype = in_dtype; J.c.npos = L; J.c.rope_cache = rope_cache;
    J.c.cs = build_cs_threads(d, L, rope_theta, nthreads);
    if (!J.c.cs) { free(rows); return -2; }
    J.q = q; J.k = kcache; J.v = vcache; J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.L = L; J.Lkv = Lcap;
    J.q_is_decode = 1; J.rows = rows; J.n = n; J.out = out;
    int st = run_job(&J, nthreads);
    free((void*)J.c.cs);
    free(rows);
    return st;
}
