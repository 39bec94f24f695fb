/*
 * Plain fp64 CPU oracle for SANA's multi-head ReLU linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no source, header, table or
 * helper with the CUDA library; the two meet only through seeded inputs.
 *
 * What it computes (and where each step is stated):
 *
 *   Eq. (1), "Sana: Efficient High-Resolution Image Synthesis with Linear
 *   Diffusion Transformers", section 2.1 (linear attention):
 *
 *       O_i = ReLU(Q_i) (sum_j ReLU(K_j)^T V_j) / (ReLU(Q_i) sum_j ReLU(K_j)^T)
 *
 *   with the sums over all N tokens (non-causal), and the remark right after
 *   Eq. (1) of the same section that the two sums are formed once and then
 *   reused by every query token, which is what makes the cost O(N).
 *
 *   QK-Norm, "SANA 1.5: Efficient Scaling of Training-Time and
 *   Inference-Time Compute in Linear Diffusion Transformer", section
 *   "Model architecture", QK Norm bullet: an RMSNorm on the queries and keys
 *   of the linear self-attention, placed before the ReLU feature map.
 *
 * Readings taken where the pages leave a step open:
 *   - phi(x) = ReLU(g * x / sqrt(mean(x^2) + eps)), the mean taken over the
 *     D channels of one head (per-head RMSNorm), g a per-channel gain of
 *     length C = H*D.  With the norm switched off phi(x) = ReLU(x).
 *     An optional full-channel scope (mean over all C channels of a token)
 *     exists for comparison only.
 *   - The same eps is added to the scalar denominator of Eq. (1) after the
 *     dot product:  O = num / (den + eps).
 *   - Layout (B, N, C) row-major, channel c = h*D + d.
 *
 * Arithmetic is fp64 throughout, in the order the formulas are written;
 * the only parallelism is independent (b, h) pairs or tokens on pthreads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_NORM_OFF 0
#define ORACLE_NORM_PER_HEAD 1
#define ORACLE_NORM_FULL_C 2

/* ---------------------------------------------------------------------- */
/* Feature map phi: RMSNorm (optional) -> gain -> ReLU, one token.         */
/* ---------------------------------------------------------------------- */

/* phi of head h of one token: x and g hold the token's C values and gains,
 * out receives the head's D values.  norm selects the RMSNorm scope: the mean
 * square is taken over the head's D channels, or over all C channels of the
 * token for the full-channel comparison scope. */
static void phi_head(const double* x, const double* g, double* out,
                     int C, int H, int h, double eps, int norm)
{
    const int D = C / H;
    const double* xh = x + (size_t)h * D;
    if (norm == ORACLE_NORM_OFF) {
        for (int d = 0; d < D; ++d) out[d] = xh[d] > 0.0 ? xh[d] : 0.0;
        return;
    }
    double ss = 0.0;
    double r;
    if (norm == ORACLE_NORM_FULL_C) {
        for (int c = 0; c < C; ++c) ss += x[c] * x[c];
        r = 1.0 / sqrt(ss / (double)C + eps);
    } else {
        for (int d = 0; d < D; ++d) ss += xh[d] * xh[d];
        r = 1.0 / sqrt(ss / (double)D + eps);
    }
    for (int d = 0; d < D; ++d) {
        const double y = g[h * D + d] * (xh[d] * r);
        out[d] = y > 0.0 ? y : 0.0;
    }
}

/* phi of every head of one token (C values in, C values out). */
static void phi_token(const double* x, const double* g, double* out,
                      int C, int H, double eps, int norm)
{
    const int D = C / H;
    for (int h = 0; h < H; ++h) phi_head(x, g, out + (size_t)h * D, C, H, h, eps, norm);
}

/* ---------------------------------------------------------------------- */
/* Thread pool helper: run fn(i, ctx) for i in [0, n) on nthreads threads. */
/* ---------------------------------------------------------------------- */

typedef void (*work_fn)(int64_t i, void* ctx);

typedef struct {
    work_fn fn;
    void* ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
} pool_t;

static void* pool_worker(void* arg)
{
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        const int64_t i = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (i >= p->n) break;
        p->fn(i, p->ctx);
    }
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, work_fn fn, void* ctx)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if ((int64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    pool_t p;
    p.fn = fn; p.ctx = ctx; p.n = n; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    if (nthreads == 1) {
        pool_worker(&p);
    } else {
        pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
        int started = 0;
        for (int t = 0; t < nthreads; ++t)
            if (pthread_create(&th[t], NULL, pool_worker, &p) == 0) ++started;
        if (started == 0) pool_worker(&p);
        for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
        free(th);
    }
    pthread_mutex_destroy(&p.mu);
}

/* ---------------------------------------------------------------------- */
/* Public entry points (called from oracle/oracle.py through ctypes).      */
/* ---------------------------------------------------------------------- */

/* phi of every token: x (T, C) -> out (T, C).  g may be NULL only when
 * norm == ORACLE_NORM_OFF. */
typedef struct {
    const double* x; const double* g; double* out;
    int C, H; double eps; int norm;
} phi_ctx;

static void phi_row(int64_t t, void* vctx)
{
    phi_ctx* c = (phi_ctx*)vctx;
    phi_token(c->x + (size_t)t * c->C, c->g, c->out + (size_t)t * c->C,
              c->C, c->H, c->eps, c->norm);
}

int oracle_phi_f64(const double* x, const double* g, double* out,
                   int64_t T, int C, int H, double eps, int norm, int nthreads)
{
    if (C <= 0 || H <= 0 || C % H != 0 || T < 0) return -1;
    if (norm != ORACLE_NORM_OFF && g == NULL) return -1;
    phi_ctx c = { x, g, out, C, H, eps, norm };
    parallel_for(T, nthreads, phi_row, &c);
    return 0;
}

/* The per-head state of Eq. (1):
 *   S[b][h][d][e] = sum_n phi(K)[b,n,h,d] * V[b,n,h,e]   (e < D)
 *   S[b][h][d][D] = sum_n phi(K)[b,n,h,d]                (the normaliser)
 * k, v: (B, N, C).  S: (B, H, D, D+1). */
typedef struct {
    const double* k; const double* v; const double* gk; double* S;
    int64_t B, N; int C, H; double eps; int norm;
} kv_ctx;

static void kv_one(int64_t bh, void* vctx)
{
    kv_ctx* c = (kv_ctx*)vctx;
    const int D = c->C / c->H;
    const int64_t b = bh / c->H;
    const int h = (int)(bh % c->H);
    double* S = c->S + (size_t)bh * D * (D + 1);
    double* kk = (double*)malloc(sizeof(double) * (size_t)D);
    memset(S, 0, sizeof(double) * (size_t)D * (D + 1));
    for (int64_t n = 0; n < c->N; ++n) {
        const size_t row = ((size_t)b * c->N + n) * c->C;
        phi_head(c->k + row, c->gk, kk, c->C, c->H, h, c->eps, c->norm);
        const double* vv = c->v + row + (size_t)h * D;
        for (int d = 0; d < D; ++d) {
            for (int e = 0; e < D; ++e) S[d * (D + 1) + e] += kk[d] * vv[e];
            S[d * (D + 1) + D] += kk[d];
        }
    }
    free(kk);
}

int oracle_kv_state_f64(const double* k, const double* v, const double* gk,
                        double* S, int64_t B, int64_t N, int C, int H,
                        double eps, int norm, int nthreads)
{
    if (B < 0 || N < 0 || C <= 0 || H <= 0 || C % H != 0) return -1;
    if (norm != ORACLE_NORM_OFF && gk == NULL) return -1;
    kv_ctx c = { k, v, gk, S, B, N, C, H, eps, norm };
    parallel_for(B * H, nthreads, kv_one, &c);
    return 0;
}

/* Apply Eq. (1) with a given state:
 *   num[e] = sum_d phi(Q)[d] S[d][e],  den = sum_d phi(Q)[d] S[d][D],
 *   O[e]   = num[e] / (den + eps).
 * q: (B, N, C); S: (B, H, D, D+1).  tok (optional, length T) lists flat
 * token indices b*N + n to evaluate; out has T rows of C.  With tok == NULL
 * every token is evaluated and out is (B, N, C). */
typedef struct {
    const double* q; const double* gq; const double* S; double* out;
    const int64_t* tok; int64_t N; int C, H; double eps; int norm;
} ap_ctx;

static void apply_one(int64_t i, void* vctx)
{
    ap_ctx* c = (ap_ctx*)vctx;
    const int D = c->C / c->H;
    const int64_t t = c->tok ? c->tok[i] : i;
    const int64_t b = t / c->N;
    double* phiq = (double*)malloc(sizeof(double) * (size_t)c->C);
    phi_token(c->q + (size_t)t * c->C, c->gq, phiq, c->C, c->H, c->eps, c->norm);
    double* o = c->out + (size_t)i * c->C;
    for (int h = 0; h < c->H; ++h) {
        const double* S = c->S + ((size_t)b * c->H + h) * D * (D + 1);
        const double* qq = phiq + (size_t)h * D;
        double den = 0.0;
        for (int d = 0; d < D; ++d) den += qq[d] * S[d * (D + 1) + D];
        for (int e = 0; e < D; ++e) {
            double num = 0.0;
            for (int d = 0; d < D; ++d) num += qq[d] * S[d * (D + 1) + e];
            o[h * D + e] = num / (den + c->eps);
        }
    }
    free(phiq);
}

int oracle_apply_f64(const double* q, const double* gq, const double* S,
                     double* out, const int64_t* tok, int64_t T,
                     int64_t B, int64_t N, int C, int H, double eps, int norm,
                     int nthreads)
{
    if (B < 0 || N < 0 || C <= 0 || H <= 0 || C % H != 0) return -1;
    if (norm != ORACLE_NORM_OFF && gq == NULL) return -1;
    if (tok) {
        for (int64_t i = 0; i < T; ++i)
            if (tok[i] < 0 || tok[i] >= B * N) return -1;
    } else {
        T = B * N;
    }
    ap_ctx c = { q, gq, S, out, tok, N, C, H, eps, norm };
    parallel_for(T, nthreads, apply_one, &c);
    return 0;
}

/* The whole op: state, then apply.  out: (B, N, C). */
int oracle_forward_f64(const double* q, const double* k, const double* v,
                       const double* gq, const double* gk, double* out,
                       int64_t B, int64_t N, int C, int H, double eps,
                       int norm, int nthreads)
{
    if (B < 0 || N < 0 || C <= 0 || H <= 0 || C % H != 0) return -1;
    const int D = C / H;
    double* S = (double*)malloc(sizeof(double) * (size_t)(B * H) * D * (D + 1) + 1);
    if (!S) return -2;
    int rc = oracle_kv_state_f64(k, v, gk, S, B, N, C, H, eps, norm, nthreads);
    if (rc == 0)
        rc = oracle_apply_f64(q, gq, S, out, NULL, 0, B, N, C, H, eps, norm, nthreads);
    free(S);
    return rc;
}

/* The prefix (causal) form: "Sana ..." notes describe linear attention as a
 * cumulative prefix sum (the explainer page's O(N) prefix form).  Token n only
 * sees keys j <= n:
 *   S_n[d][e] = sum_{j <= n} phi(K_j)[d] V_j[e],  S_n[d][D] = sum_{j <= n} phi(K_j)[d],
 *   O_n[e]    = (sum_d phi(Q_n)[d] S_n[d][e]) / (sum_d phi(Q_n)[d] S_n[d][D] + eps).
 * Written as the running sum over tokens, one (b, h) at a time.  out: (B, N, C). */
typedef struct {
    const double* q; const double* k; const double* v;
    const double* gq; const double* gk; double* out;
    int64_t N; int C, H; double eps; int norm;
} causal_ctx;

static void causal_one(int64_t bh, void* vctx)
{
    causal_ctx* c = (causal_ctx*)vctx;
    const int D = c->C / c->H;
    const int64_t b = bh / c->H;
    const int h = (int)(bh % c->H);
    double* run = (double*)calloc((size_t)D * (D + 1), sizeof(double));   /* S_n */
    double* fk = (double*)malloc(sizeof(double) * (size_t)D);
    double* fq = (double*)malloc(sizeof(double) * (size_t)D);
    for (int64_t t = 0; t < c->N; ++t) {              /* tokens in order */
        const size_t at = ((size_t)b * c->N + t) * c->C;
        /* S_n = S_{n-1} + phi(K_n)^T [V_n | 1] */
        phi_head(c->k + at, c->gk, fk, c->C, c->H, h, c->eps, c->norm);
        const double* vn = c->v + at + (size_t)h * D;
        for (int i = 0; i < D; ++i) {
            for (int j = 0; j < D; ++j) run[i * (D + 1) + j] += fk[i] * vn[j];
            run[i * (D + 1) + D] += fk[i];
        }
        /* O_n = phi(Q_n) S_n[:, :D] / (phi(Q_n) S_n[:, D] + eps) */
        phi_head(c->q + at, c->gq, fq, c->C, c->H, h, c->eps, c->norm);
        double dn = 0.0;
        for (int i = 0; i < D; ++i) dn += fq[i] * run[i * (D + 1) + D];
        double* on = c->out + at + (size_t)h * D;
        for (int j = 0; j < D; ++j) {
            double nm = 0.0;
            for (int i = 0; i < D; ++i) nm += fq[i] * run[i * (D + 1) + j];
            on[j] = nm / (dn + c->eps);
        }
    }
    free(run);
    free(fk);
    free(fq);
}

int oracle_causal_forward_f64(const double* q, const double* k, const double* v,
                              const double* gq, const double* gk, double* out,
                              int64_t B, int64_t N, int C, int H, double eps,
                              int norm, int nthreads)
{
    if (B < 0 || N < 0 || C <= 0 || H <= 0 || C % H != 0) return -1;
    if (norm != ORACLE_NORM_OFF && (gq == NULL || gk == NULL)) return -1;
    causal_ctx c = { q, k, v, gq, gk, out, N, C, H, eps, norm };
    parallel_for(B * H, nthreads, causal_one, &c);
    return 0;
}
