/*
 * gdr_oracle.c -- fp64 CPU oracle of the gated delta-rule layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code with the CUDA library.
 *
 * Everything is plain, slow and written to be checked by eye against the
 * pages that describe the layer:
 *
 *  [P2] "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型" (kongchang.com),
 *       section 注意力层的细节: 16 key heads / 48 value heads, head dim 128,
 *       a kernel-4 causal conv in front, gated RMSNorm, fp32 recurrent state;
 *       box 门控 delta rule: the forget-gated variant of the delta rule.
 *  [P3] "33B 只做 18 层：Agnes 3.0 Flash 靠「小身材」杀进轻量模型第一梯队？"
 *       (yfxerp.com), §1.2: beta = sigmoid(b),
 *       g = -exp(A_log) * softplus(a + dt_bias) in fp32, q/k L2-normalised
 *       inside the recurrence, chunk 64 prefill and single-step decode said to
 *       be interchangeable.
 *  [P4] "Sapiens AI 发布 Agnes-3.0-Flash：以 Apache 2.0 开源的 33B 多模态模型"
 *       (gpts24.com), section "delta 规则循环层究竟怎么运作": new state =
 *       old state x (I - beta k k^T) + beta v k^T, beta a per-token strength.
 *  [P5] "33B 只做 18 层 ..." (mhpq.cn), §2.1 源码层的架构印证: the model
 *       source has a single-step causal conv, a chunk-64 loop and a
 *       per-token loop.
 *
 * The gated recurrence in full (per value head, state S of size dv x dk):
 *     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = scale * S_t q_t.
 * This file stores the state transposed, H = S^T with shape [dk][dv], which
 * is the layout the CUDA library uses as well.
 *
 * Readings of points the pages leave open (listed in the design notes):
 *  - L2 norm: x / sqrt(sum x^2 + 1e-6).
 *  - softplus follows torch's default (beta 1, threshold 20).
 *  - value head h reads key head h / (hv / hk) (contiguous grouping).
 *  - conv: y_t = SiLU(sum_j w[c][j] x_{t-3+j}), w[c][3] hits the current
 *    token; positions before a sequence start come from the conv state
 *    ([3][C], oldest first) or are zero.
 *  - gated RMSNorm: y = o / sqrt(mean(o^2) + eps) * w * SiLU(z).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

#define EXPORT __attribute__((visibility("default")))

EXPORT int oracle_abi_version(void) { return 1; }

/* ------------------------------------------------------------------------ */
/* bf16 rounding of an fp64 value, round to nearest, ties to even.           */
/* A bf16 keeps the sign, the 8-bit exponent and 7 fraction bits of fp32.    */
/* Rounding straight from fp64 (not through fp32) avoids double rounding.    */
/* ------------------------------------------------------------------------ */
EXPORT uint16_t oracle_round_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    double ax = fabs(x);
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (ax == 0.0) return sign;
    if (isinf(x)) return sign | 0x7F80;
    int e;
    double m = frexp(ax, &e);        /* ax = m * 2^e, m in [0.5, 1) */
    int exp32 = e - 1;               /* ax = (2m) * 2^(e-1), 2m in [1,2) */
    double q;                        /* quantum at this magnitude */
    if (exp32 < -126) {
        q = ldexp(1.0, -126 - 7);    /* subnormal bf16 spacing */
    } else {
        q = ldexp(1.0, exp32 - 7);   /* 8 significant bits */
    }
    double n = ax / q;               /* exact: power-of-two scaling */
    double fl = floor(n);
    double frac = n - fl;
    double r;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double v = r * q;
    if (v >= ldexp(1.0, 128)) return sign | 0x7F80;   /* overflow to inf */
    float f = (float)v;               /* exact: v has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16) | sign;
}

EXPORT void oracle_round_bf16_array(const double *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Gates [P3 §1.2]                                                           */
/* ------------------------------------------------------------------------ */
EXPORT double oracle_softplus(double x)
{
    /* torch.nn.functional.softplus default: beta 1, threshold 20 */
    if (x > 20.0) return x;
    return log1p(exp(x));
}

EXPORT double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* g[t][h] = -exp(A_log[h]) * softplus(a[t][h] + dt_bias[h]);
 * beta[t][h] = sigmoid(b[t][h]).   a, b: [T][hv]. */
EXPORT void oracle_gates(const double *a, const double *b, const float *A_log,
                         const float *dt_bias, int64_t T, int hv, double *g, double *beta)
{
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < hv; ++h) {
            int64_t i = t * hv + h;
            g[i] = -exp((double)A_log[h]) * oracle_softplus(a[i] + (double)dt_bias[h]);
            beta[i] = oracle_sigmoid(b[i]);
        }
}

/* ------------------------------------------------------------------------ */
/* small thread pool over independent (sequence, value head) units           */
/* ------------------------------------------------------------------------ */
typedef void (*unit_fn)(void *ctx, int unit);
typedef struct { unit_fn fn; void *ctx; int n_units; int next; } pool_t;

static void *pool_worker(void *p_)
{
    pool_t *p = (pool_t *)p_;
    for (;;) {
        int u = __atomic_fetch_add(&p->next, 1, __ATOMIC_RELAXED);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static void run_units(unit_fn fn, void *ctx, int n_units, int nthreads)
{
    pool_t p = {fn, ctx, n_units, 0};
    if (nthreads <= 1 || n_units <= 1) { pool_worker(&p); return; }
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 0; i < nthreads - 1; ++i)
        if (pthread_create(&th[started], NULL, pool_worker, &p) == 0) ++started;
    pool_worker(&p);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------ */
/* The recurrence, token by token [P4 delta 规则循环层究竟怎么运作; P3 §1.2]   */
/* ------------------------------------------------------------------------ */
typedef struct {
    int hk, hv, dk, dv;
    const double *q, *k, *v, *g, *beta;
    double scale;
    int use_l2norm;
    double l2eps;
    const int32_t *cu;
    const double *h0;
    double *o, *hT;
    const int32_t *head_mask;
    int chunk;               /* chunked form only */
} core_ctx;

static void l2_normalise(const double *x, int d, int use, double eps, double *out)
{
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += x[i] * x[i];
    double r = use ? 1.0 / sqrt(s + eps) : 1.0;
    for (int i = 0; i < d; ++i) out[i] = x[i] * r;
}

static void stepwise_unit(void *ctx_, int unit)
{
    const core_ctx *c = (const core_ctx *)ctx_;
    const int hv = c->hv, hk = c->hk, dk = c->dk, dv = c->dv;
    const int n = unit / hv, h = unit % hv;
    if (c->head_mask && !c->head_mask[h]) return;
    const int kh = h / (hv / hk);
    double *H = (double *)malloc(sizeof(double) * dk * dv);
    double *qn = (double *)malloc(sizeof(double) * dk);
    double *kn = (double *)malloc(sizeof(double) * dk);
    double *u = (double *)malloc(sizeof(double) * dv);
    double *acc = (double *)malloc(sizeof(double) * dv);
    const size_t soff = ((size_t)n * hv + h) * dk * dv;
    for (int e = 0; e < dk * dv; ++e) H[e] = c->h0 ? c->h0[soff + e] : 0.0;

    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        l2_normalise(c->q + ((size_t)t * hk + kh) * dk, dk, c->use_l2norm, c->l2eps, qn);
        l2_normalise(c->k + ((size_t)t * hk + kh) * dk, dk, c->use_l2norm, c->l2eps, kn);
        const double *vt = c->v + ((size_t)t * hv + h) * dv;
        const double decay = exp(c->g[(size_t)t * hv + h]);
        const double bt = c->beta[(size_t)t * hv + h];
        /* H' = exp(g) H */
        for (int e = 0; e < dk * dv; ++e) H[e] *= decay;
        /* u = beta (v - H'^T k) */
        for (int j = 0; j < dv; ++j) acc[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) acc[j] += H[i * dv + j] * kn[i];
        for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - acc[j]);
        /* H = H' + k u^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) H[i * dv + j] += kn[i] * u[j];
        /* o = scale H^T q */
        for (int j = 0; j < dv; ++j) acc[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) acc[j] += H[i * dv + j] * qn[i];
        double *ot = c->o + ((size_t)t * hv + h) * dv;
        for (int j = 0; j < dv; ++j) ot[j] = c->scale * acc[j];
    }
    if (c->hT) memcpy(c->hT + soff, H, sizeof(double) * dk * dv);
    free(H); free(qn); free(kn); free(u); free(acc);
}

/*
 * Stepwise recurrence over packed sequences.
 *   q, k: [T][hk][dk]   v: [T][hv][dv]   g, beta: [T][hv]
 *   cu: [n_seqs+1] token offsets, h0: [n_seqs][hv][dk][dv] or NULL (zeros)
 *   o: [T][hv][dv]      hT: [n_seqs][hv][dk][dv] or NULL
 *   head_mask: [hv] or NULL; heads with mask 0 are skipped (outputs untouched)
 */
EXPORT int oracle_gdr_stepwise(int hk, int hv, int dk, int dv,
                               const double *q, const double *k, const double *v,
                               const double *g, const double *beta, double scale,
                               int use_l2norm, double l2eps,
                               const int32_t *cu, int n_seqs, const double *h0,
                               double *o, double *hT, const int32_t *head_mask,
                               int nthreads)
{
    if (hk <= 0 || hv <= 0 || hv % hk || dk <= 0 || dv <= 0 || n_seqs < 0) return -1;
    core_ctx c = {hk, hv, dk, dv, q, k, v, g, beta, scale, use_l2norm, l2eps,
                  cu, h0, o, hT, head_mask, 0};
    run_units(stepwise_unit, &c, n_seqs * hv, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The chunked form, used only to cross-check the stepwise one.              */
/* [P3 §1.2] names a chunk-64 path and says it is interchangeable with the    */
/* per-token path.  Unrolling the recurrence inside a chunk of length L with */
/* cumulative log-decay gamma_i = g_1 + ... + g_i gives                       */
/*   A_ij = beta_i exp(gamma_i - gamma_j) k_i.k_j        (j < i)              */
/*   T    = (I + A)^-1                                                        */
/*   W    = T diag(beta exp(gamma)) K,   Ut = T diag(beta) V                  */
/*   U    = Ut - W H0                                                         */
/*   O    = scale (diag(exp(gamma)) Q H0 + (Q K^T . M) U),                    */
/*          M_ij = exp(gamma_i - gamma_j) for j <= i, else 0                  */
/*   H_L  = exp(gamma_L) H0 + K^T diag(exp(gamma_L - gamma)) U                */
/* ------------------------------------------------------------------------ */
static void chunked_unit(void *ctx_, int unit)
{
    const core_ctx *c = (const core_ctx *)ctx_;
    const int hv = c->hv, hk = c->hk, dk = c->dk, dv = c->dv, C = c->chunk;
    const int n = unit / hv, h = unit % hv;
    if (c->head_mask && !c->head_mask[h]) return;
    const int kh = h / (hv / hk);
    double *H = malloc(sizeof(double) * dk * dv);
    double *Kn = malloc(sizeof(double) * C * dk), *Qn = malloc(sizeof(double) * C * dk);
    double *V = malloc(sizeof(double) * C * dv);
    double *gam = malloc(sizeof(double) * C), *bt = malloc(sizeof(double) * C);
    double *A = malloc(sizeof(double) * C * C), *Tm = malloc(sizeof(double) * C * C);
    double *W = malloc(sizeof(double) * C * dk), *U = malloc(sizeof(double) * C * dv);
    double *Hn = malloc(sizeof(double) * dk * dv);
    const size_t soff = ((size_t)n * hv + h) * dk * dv;
    for (int e = 0; e < dk * dv; ++e) H[e] = c->h0 ? c->h0[soff + e] : 0.0;

    for (int64_t s = c->cu[n]; s < c->cu[n + 1]; s += C) {
        int L = (int)((c->cu[n + 1] - s) < C ? (c->cu[n + 1] - s) : C);
        double run = 0.0;
        for (int i = 0; i < L; ++i) {
            size_t t = (size_t)(s + i);
            l2_normalise(c->q + (t * hk + kh) * dk, dk, c->use_l2norm, c->l2eps, Qn + i * dk);
            l2_normalise(c->k + (t * hk + kh) * dk, dk, c->use_l2norm, c->l2eps, Kn + i * dk);
            memcpy(V + i * dv, c->v + (t * hv + h) * dv, sizeof(double) * dv);
            run += c->g[t * hv + h];
            gam[i] = run;
            bt[i] = c->beta[t * hv + h];
        }
        /* A (strictly lower) */
        for (int i = 0; i < L; ++i)
            for (int j = 0; j < L; ++j) {
                double a = 0.0;
                if (j < i) {
                    double d = 0.0;
                    for (int x = 0; x < dk; ++x) d += Kn[i * dk + x] * Kn[j * dk + x];
                    a = bt[i] * exp(gam[i] - gam[j]) * d;
                }
                A[i * C + j] = a;
            }
        /* T = (I + A)^-1 by forward substitution, one column at a time */
        for (int col = 0; col < L; ++col)
            for (int i = 0; i < L; ++i) {
                double x = (i == col) ? 1.0 : 0.0;
                for (int j = 0; j < i; ++j) x -= A[i * C + j] * Tm[j * C + col];
                Tm[i * C + col] = x;
            }
        /* W = T diag(beta e^gamma) K ;  U = T diag(beta) V - W H0 */
        for (int i = 0; i < L; ++i) {
            for (int x = 0; x < dk; ++x) {
                double sacc = 0.0;
                for (int j = 0; j < L; ++j) sacc += Tm[i * C + j] * bt[j] * exp(gam[j]) * Kn[j * dk + x];
                W[i * dk + x] = sacc;
            }
            for (int y = 0; y < dv; ++y) {
                double sacc = 0.0;
                for (int j = 0; j < L; ++j) sacc += Tm[i * C + j] * bt[j] * V[j * dv + y];
                for (int x = 0; x < dk; ++x) sacc -= W[i * dk + x] * H[x * dv + y];
                U[i * dv + y] = sacc;
            }
        }
        /* O */
        for (int i = 0; i < L; ++i) {
            double *ot = c->o + ((size_t)(s + i) * hv + h) * dv;
            double ei = exp(gam[i]);
            for (int y = 0; y < dv; ++y) {
                double inter = 0.0, intra = 0.0;
                for (int x = 0; x < dk; ++x) inter += Qn[i * dk + x] * H[x * dv + y];
                for (int j = 0; j <= i; ++j) {
                    double qk = 0.0;
                    for (int x = 0; x < dk; ++x) qk += Qn[i * dk + x] * Kn[j * dk + x];
                    intra += qk * exp(gam[i] - gam[j]) * U[j * dv + y];
                }
                ot[y] = c->scale * (ei * inter + intra);
            }
        }
        /* H_L */
        double eL = exp(gam[L - 1]);
        for (int x = 0; x < dk; ++x)
            for (int y = 0; y < dv; ++y) {
                double sacc = eL * H[x * dv + y];
                for (int j = 0; j < L; ++j) sacc += Kn[j * dk + x] * exp(gam[L - 1] - gam[j]) * U[j * dv + y];
                Hn[x * dv + y] = sacc;
            }
        memcpy(H, Hn, sizeof(double) * dk * dv);
    }
    if (c->hT) memcpy(c->hT + soff, H, sizeof(double) * dk * dv);
    free(H); free(Kn); free(Qn); free(V); free(gam); free(bt); free(A); free(Tm);
    free(W); free(U); free(Hn);
}

EXPORT int oracle_gdr_chunked(int hk, int hv, int dk, int dv,
                              const double *q, const double *k, const double *v,
                              const double *g, const double *beta, double scale,
                              int use_l2norm, double l2eps,
                              const int32_t *cu, int n_seqs, const double *h0,
                              double *o, double *hT, const int32_t *head_mask,
                              int chunk, int nthreads)
{
    if (hk <= 0 || hv <= 0 || hv % hk || dk <= 0 || dv <= 0 || chunk <= 0 || n_seqs < 0) return -1;
    core_ctx c = {hk, hv, dk, dv, q, k, v, g, beta, scale, use_l2norm, l2eps,
                  cu, h0, o, hT, head_mask, chunk};
    run_units(chunked_unit, &c, n_seqs * hv, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Depthwise causal conv, kernel 4, SiLU [P2 注意力层的细节; P5 §2.1]          */
/* ------------------------------------------------------------------------ */
static double silu(double x) { return x / (1.0 + exp(-x)); }

/*
 * x: [T][C], w: [C][4], conv_state: [n_seqs][3][C] (oldest first) or NULL.
 * y: [T][C]; if round_y, every y is rounded to bf16 (the conv output is a
 * bf16 tensor).  conv_state_out ([n_seqs][3][C], may be NULL) receives the
 * last three inputs of each sequence (older ones from conv_state if the
 * sequence is shorter than three).
 */
EXPORT void oracle_causal_conv(const double *x, const double *w, const double *conv_state,
                               const int32_t *cu, int n_seqs, int C, double *y,
                               double *conv_state_out, int round_y)
{
    for (int n = 0; n < n_seqs; ++n) {
        int64_t s = cu[n], e = cu[n + 1];
        for (int64_t t = s; t < e; ++t)
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int j = 0; j < 4; ++j) {
                    int64_t p = t - 3 + j;          /* input position */
                    double xv;
                    if (p >= s) xv = x[p * C + c];
                    else {
                        int64_t back = s - p;       /* 1..3 positions before start */
                        xv = conv_state ? conv_state[((size_t)n * 3 + (3 - back)) * C + c] : 0.0;
                    }
                    acc += w[(size_t)c * 4 + j] * xv;
                }
                double r = silu(acc);
                if (round_y) {
                    uint16_t bits = oracle_round_bf16(r);
                    uint32_t u = (uint32_t)bits << 16;
                    float f;
                    memcpy(&f, &u, 4);
                    r = f;
                }
                y[t * C + c] = r;
            }
        if (conv_state_out)
            for (int slot = 0; slot < 3; ++slot) {
                int64_t p = e - 3 + slot;
                for (int c = 0; c < C; ++c) {
                    double xv;
                    if (p >= s) xv = x[p * C + c];
                    else {
                        int64_t back = s - p;
                        xv = conv_state ? conv_state[((size_t)n * 3 + (3 - back)) * C + c] : 0.0;
                    }
                    conv_state_out[((size_t)n * 3 + slot) * C + c] = xv;
                }
            }
    }
}

/*
 * Single-step form of the same conv, as used by decode [P5 §2.1, the
 * single-step conv of the model source]: for each of B sequences,
 * y = SiLU(w0 s0 + w1 s1 + w2 s2 + w3 x), then the state rolls to (s1, s2, x).
 * x: [B][C], conv_state: [B][3][C] in/out, y: [B][C] (not rounded).
 */
EXPORT void oracle_conv_step(const double *x, const double *w, double *conv_state,
                             int B, int C, double *y)
{
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < C; ++c) {
            double *s = conv_state + (size_t)b * 3 * C;
            double s0 = s[c], s1 = s[C + c], s2 = s[2 * C + c], xv = x[(size_t)b * C + c];
            const double *wc = w + (size_t)c * 4;
            y[(size_t)b * C + c] = silu(wc[0] * s0 + wc[1] * s1 + wc[2] * s2 + wc[3] * xv);
            s[c] = s1; s[C + c] = s2; s[2 * C + c] = xv;
        }
}

/* ------------------------------------------------------------------------ */
/* Gated RMSNorm over rows of d [P2 注意力层的细节; P3 §2 table: z of width   */
/* 6144 = 48 x 128]:  y = o / sqrt(mean(o^2) + eps) * w * SiLU(z)            */
/* ------------------------------------------------------------------------ */
EXPORT void oracle_gated_rmsnorm(const double *o, const double *z, const double *w,
                                 double eps, int64_t rows, int d, double *y)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double *orow = o + r * d, *zrow = z + r * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += orow[j] * orow[j];
        double inv = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j)
            y[r * d + j] = orow[j] * inv * (w ? w[j] : 1.0) * silu(zrow[j]);
    }
}

/* ------------------------------------------------------------------------ */
/* Chunk table of packed sequences: chunks of `chunk` tokens restart at each  */
/* sequence start; the last chunk of a sequence may be shorter.  Returns the */
/* number of chunks, or -1 if cu is not a valid offset array or the table    */
/* does not fit in max_chunks entries.                                       */
/* ------------------------------------------------------------------------ */
EXPORT int oracle_prepare_chunks(const int32_t *cu, int n_seqs, int chunk,
                                 int32_t *chunk_seq, int32_t *chunk_start, int32_t *chunk_len,
                                 int max_chunks)
{
    if (n_seqs < 0 || chunk <= 0 || cu[0] != 0) return -1;
    int m = 0;
    for (int n = 0; n < n_seqs; ++n) {
        if (cu[n + 1] < cu[n]) return -1;
        for (int64_t t = cu[n]; t < cu[n + 1]; ++t) {
            if ((t - cu[n]) % chunk == 0) {          /* a chunk starts here */
                if (m >= max_chunks) return -1;
                chunk_seq[m] = n;
                chunk_start[m] = (int32_t)t;
                chunk_len[m] = 0;
                ++m;
            }
            chunk_len[m - 1] += 1;                    /* token t joins the open chunk */
        }
    }
    return m;
}
