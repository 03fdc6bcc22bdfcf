/*
 * fp64 CPU oracle for causal linear attention in its plain, gated, DeltaNet and
 * Gated DeltaNet forms.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the benchmark's CPU-baseline leg use it; no product code links it.  It
 * shares no code, header or table with the CUDA library.
 *
 * Sources (page title, section):
 *  - "混合注意力学习(1): 线性注意力" (jsqmd.com), section "Fast Weight Programmers与
 *    DeltaNet": the state is a key->value associative memory updated once per
 *    token; the delta rule reads the value currently bound to k, blends it with
 *    the new v through the learning rate beta and writes the difference back.
 *  - same page, section "Gated DeltaNet": Mamba2-style scalar decay alpha_t of
 *    the whole state, combined with the delta rule.
 *  - "【CS336】lecture4 线性注意力|Mamba|GDN|DSA" (wsisp.com), sections
 *    "朴素线性注意力" and "继续改进：GDN": the recurrent form accumulates k_t v_t^T
 *    into S_t, reads the output from S_t and q_t, and the erase factor
 *    (I - beta_t k_t k_t^T) is applied by computing k^T S first (O(d^2)/token).
 *  - "LinearAttention 概述" (razer666.cn), section "Lightning Attention": position
 *    t sees positions 1..t inclusive (Output_1 = q_1 (k_1^T v_1)), i.e. the
 *    output is read from the state AFTER the current token's write.
 *
 * Conventions (the pages print the exact equations only partly; the readings
 * taken are stated here):
 *  - Per head the state S is stored dk x dv (row j = key coordinate, column c =
 *    value coordinate).  In this layout the Gated DeltaNet step
 *        S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *    (value-by-key orientation) becomes
 *        u_t = beta_t (v_t - alpha_t S_{t-1}^T k_t)
 *        S_t = alpha_t S_{t-1} + k_t u_t^T
 *        o_t = S_t^T (scale * q_t)
 *  - Without beta (plain / gated linear attention): S_t = alpha_t S_{t-1} + k_t v_t^T.
 *  - Without g: alpha_t = 1.  With g: alpha_t = exp(g_t) (g is log-alpha).
 *  - Vector-valued gates (one log-decay per key coordinate, g_t in R^dk; the
 *    GLA-style variant next to the scalar gate flag): alpha_t = exp(g_t)
 *    elementwise decays row j of S by alpha_t[j]:
 *        u_t = beta_t (v_t - (diag(alpha_t) S_{t-1})^T k_t)
 *        S_t = diag(alpha_t) S_{t-1} + k_t u_t^T
 *    i.e. S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
 *
 * Everything is IEEE double, no fast-math; heads run on plain pthreads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* o = S^T (scale q): the read-out of a dk x dv state.                        */
static void read_out(const double *S, const double *q, double scale, long dk, long dv, double *o)
{
    for (long c = 0; c < dv; ++c) o[c] = 0.0;
    for (long j = 0; j < dk; ++j) {
        const double qj = scale * q[j];
        for (long c = 0; c < dv; ++c) o[c] += S[j * dv + c] * qj;
    }
}

/* ------------------------------------------------------------------------- */
/* One token of the recurrence for one head (the definition above).          */
/* S: dk x dv row-major, updated in place.  o: dv outputs.  sk: dv scratch.   */
static void token_step(double *S, const double *q, const double *k, const double *v,
                       const double *beta, const double *g, double scale,
                       long dk, long dv, double *o, double *sk)
{
    const double alpha = g ? exp(*g) : 1.0;
    if (beta) {
        /* read: the value the memory currently returns for key k (decayed) */
        for (long c = 0; c < dv; ++c) sk[c] = 0.0;
        for (long j = 0; j < dk; ++j)
            for (long c = 0; c < dv; ++c) sk[c] += S[j * dv + c] * k[j];
        /* blend/write amount: u = beta (v - alpha S^T k) */
        for (long c = 0; c < dv; ++c) sk[c] = (*beta) * (v[c] - alpha * sk[c]);
    } else {
        for (long c = 0; c < dv; ++c) sk[c] = v[c];
    }
    for (long j = 0; j < dk; ++j)
        for (long c = 0; c < dv; ++c) S[j * dv + c] = alpha * S[j * dv + c] + k[j] * sk[c];
    /* output from the state after this token's write */
    read_out(S, q, scale, dk, dv, o);
}

/* ------------------------------------------------------------------------- */
/* One token with a vector-valued gate gv (dk log-decays, one per key row).  */
/* S: dk x dv, in place.  sk: dv scratch, a: dk scratch.                      */
static void token_step_vg(double *S, const double *q, const double *k, const double *v,
                          const double *beta, const double *gv, double scale,
                          long dk, long dv, double *o, double *sk, double *a)
{
    for (long j = 0; j < dk; ++j) a[j] = gv ? exp(gv[j]) : 1.0;
    /* decay first: row j of the state by alpha[j] */
    for (long j = 0; j < dk; ++j)
        for (long c = 0; c < dv; ++c) S[j * dv + c] *= a[j];
    if (beta) {
        /* read the decayed memory at key k (column by column), then u = beta (v - read) */
        for (long col = 0; col < dv; ++col) {
            double rd = 0.0;
            for (long row = 0; row < dk; ++row) rd += k[row] * S[row * dv + col];
            sk[col] = (*beta) * (v[col] - rd);
        }
    } else {
        memcpy(sk, v, sizeof(double) * (size_t)dv);
    }
    for (long row = 0; row < dk; ++row)
        for (long col = 0; col < dv; ++col) S[row * dv + col] += sk[col] * k[row];
    read_out(S, q, scale, dk, dv, o);
}

/* ------------------------------------------------------------------------- */
/* Thread pool over independent heads.                                       */
typedef void (*head_fn)(void *ctx, long head, double *scratch);

typedef struct {
    head_fn fn;
    void *ctx;
    long nheads;
    long next;
    long scratch_len;
    pthread_mutex_t mu;
} pool_t;

static void *pool_worker(void *arg)
{
    pool_t *p = (pool_t *)arg;
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(p->scratch_len > 0 ? p->scratch_len : 1));
    for (;;) {
        pthread_mutex_lock(&p->mu);
        long h = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (h >= p->nheads) break;
        p->fn(p->ctx, h, scratch);
    }
    free(scratch);
    return NULL;
}

static void run_heads(head_fn fn, void *ctx, long nheads, long scratch_len, int nthreads)
{
    pool_t p;
    p.fn = fn; p.ctx = ctx; p.nheads = nheads; p.next = 0; p.scratch_len = scratch_len;
    pthread_mutex_init(&p.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nheads) nthreads = (int)(nheads > 0 ? nheads : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
    pool_worker(&p);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------------- */
/* Prefill: token-by-token recurrence over (B*H) heads.                       */
typedef struct {
    const double *q, *k, *v, *beta, *g, *s0;
    double *o, *s_final;
    long L, dk, dv;
    double scale;
} fwd_ctx;

static void fwd_head(void *vctx, long h, double *scratch)
{
    fwd_ctx *c = (fwd_ctx *)vctx;
    const long L = c->L, dk = c->dk, dv = c->dv;
    double *S = scratch, *sk = scratch + dk * dv;
    if (c->s0) memcpy(S, c->s0 + h * dk * dv, sizeof(double) * (size_t)(dk * dv));
    else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
    for (long t = 0; t < L; ++t) {
        const long r = h * L + t;
        token_step(S, c->q + r * dk, c->k + r * dk, c->v + r * dv,
                   c->beta ? c->beta + r : NULL, c->g ? c->g + r : NULL, c->scale,
                   dk, dv, c->o + r * dv, sk);
    }
    if (c->s_final) memcpy(c->s_final + h * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
}

/* q,k: (BH, L, dk); v: (BH, L, dv); beta, g: (BH, L) or NULL; s0: (BH, dk, dv)
 * or NULL (zero state); o: (BH, L, dv); s_final: (BH, dk, dv) or NULL.  */
int oracle_recurrent_fwd(const double *q, const double *k, const double *v,
                         const double *beta, const double *g, const double *s0,
                         double *o, double *s_final, long BH, long L, long dk, long dv,
                         double scale, int nthreads)
{
    if (BH < 0 || L < 0 || dk < 1 || dv < 1) return 1;
    fwd_ctx c = {q, k, v, beta, g, s0, o, s_final, L, dk, dv, scale};
    run_heads(fwd_head, &c, BH, dk * dv + dv, nthreads);
    return 0;
}

/* Prefill with vector-valued gates: g (BH, L, dk) or NULL; the rest as above. */
static void fwd_head_vg(void *vctx, long h, double *scratch)
{
    fwd_ctx *c = (fwd_ctx *)vctx;
    const long L = c->L, dk = c->dk, dv = c->dv;
    double *S = scratch, *sk = scratch + dk * dv, *a = sk + dv;
    if (c->s0) memcpy(S, c->s0 + h * dk * dv, sizeof(double) * (size_t)(dk * dv));
    else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
    for (long t = 0; t < L; ++t) {
        const long r = h * L + t;
        token_step_vg(S, c->q + r * dk, c->k + r * dk, c->v + r * dv,
                      c->beta ? c->beta + r : NULL, c->g ? c->g + r * dk : NULL, c->scale,
                      dk, dv, c->o + r * dv, sk, a);
    }
    if (c->s_final) memcpy(c->s_final + h * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
}

int oracle_recurrent_fwd_vg(const double *q, const double *k, const double *v,
                            const double *beta, const double *g, const double *s0,
                            double *o, double *s_final, long BH, long L, long dk, long dv,
                            double scale, int nthreads)
{
    if (BH < 0 || L < 0 || dk < 1 || dv < 1) return 1;
    fwd_ctx c = {q, k, v, beta, g, s0, o, s_final, L, dk, dv, scale};
    run_heads(fwd_head_vg, &c, BH, dk * dv + dv + dk, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Decode: one token for each of NH independent heads, state in place.       */
typedef struct {
    const double *q, *k, *v, *beta, *g;
    double *state, *o;
    long dk, dv;
    double scale;
} dec_ctx;

static void dec_head(void *vctx, long h, double *scratch)
{
    dec_ctx *c = (dec_ctx *)vctx;
    token_step(c->state + h * c->dk * c->dv, c->q + h * c->dk, c->k + h * c->dk,
               c->v + h * c->dv, c->beta ? c->beta + h : NULL, c->g ? c->g + h : NULL,
               c->scale, c->dk, c->dv, c->o + h * c->dv, scratch);
}

int oracle_decode_step(const double *q, const double *k, const double *v,
                       const double *beta, const double *g, double *state, double *o,
                       long NH, long dk, long dv, double scale, int nthreads)
{
    if (NH < 0 || dk < 1 || dv < 1) return 1;
    dec_ctx c = {q, k, v, beta, g, state, o, dk, dv, scale};
    run_heads(dec_head, &c, NH, dv, nthreads);
    return 0;
}

/* Decode with vector-valued gates: g (NH, dk) or NULL. */
static void dec_head_vg(void *vctx, long h, double *scratch)
{
    dec_ctx *c = (dec_ctx *)vctx;
    token_step_vg(c->state + h * c->dk * c->dv, c->q + h * c->dk, c->k + h * c->dk,
                  c->v + h * c->dv, c->beta ? c->beta + h : NULL, c->g ? c->g + h * c->dk : NULL,
                  c->scale, c->dk, c->dv, c->o + h * c->dv, scratch, scratch + c->dv);
}

int oracle_decode_step_vg(const double *q, const double *k, const double *v,
                          const double *beta, const double *g, double *state, double *o,
                          long NH, long dk, long dv, double scale, int nthreads)
{
    if (NH < 0 || dk < 1 || dv < 1) return 1;
    dec_ctx c = {q, k, v, beta, g, state, o, dk, dv, scale};
    run_heads(dec_head_vg, &c, NH, dv + dk, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Chunkwise re-derivation (test-only cross-check of the chunk algebra).
 *
 * "LinearAttention 概述", section "FLASH": the chunkwise-parallel form is exact,
 * C = 1 is the recurrent form and C = L the parallel form.  "混合注意力学习(1)",
 * sections "DeltaNet 分块并行机制", "重新定义降低内存占用" and "HouseHolder变换和WY表示":
 * the per-chunk pseudo-values are rebuilt by induction from the chunk's own keys
 * so no intermediate state is stored (the WY / UT form).
 *
 * For a chunk of n rows starting from state S (dk x dv), with G_r the inclusive
 * within-chunk cumulative sum of g, gamma_r = exp(G_r):
 *   A_rs = beta_r exp(G_r - G_s) k_r.k_s   (s < r),  T = (I + A)^-1 (forward substitution)
 *   W    = T diag(beta*gamma) K,   U = T diag(beta) V,   Ut = U - W S
 *   O    = diag(gamma) Q S + (Q K^T o Gamma) Ut,   Gamma_rs = exp(G_r - G_s) (s <= r)
 *   S'   = gamma_n S + sum_s exp(G_n - G_s) k_s Ut_s^T
 * Without beta the pseudo-values are V itself (Ut = V).                      */
typedef struct {
    const double *q, *k, *v, *beta, *g, *s0;
    double *o, *s_final;
    long L, dk, dv, C;
    double scale;
} chk_ctx;

static void chunk_head(void *vctx, long h, double *scratch)
{
    chk_ctx *c = (chk_ctx *)vctx;
    const long L = c->L, dk = c->dk, dv = c->dv, C = c->C;
    double *S = scratch;                 /* dk*dv */
    double *G = S + dk * dv;             /* C */
    double *A = G + C;                   /* C*C, then T in place */
    double *W = A + C * C;               /* C*dk */
    double *Ut = W + C * dk;             /* C*dv */
    double *S2 = Ut + C * dv;            /* dk*dv */
    if (c->s0) memcpy(S, c->s0 + h * dk * dv, sizeof(double) * (size_t)(dk * dv));
    else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
    for (long t0 = 0; t0 < L; t0 += C) {
        const long n = (L - t0 < C) ? (L - t0) : C;
        const double *Q = c->q + (h * L + t0) * dk, *K = c->k + (h * L + t0) * dk;
        const double *V = c->v + (h * L + t0) * dv;
        const double *bt = c->beta ? c->beta + h * L + t0 : NULL;
        const double *gg = c->g ? c->g + h * L + t0 : NULL;
        double acc = 0.0;
        for (long r = 0; r < n; ++r) { acc += gg ? gg[r] : 0.0; G[r] = acc; }
        if (bt) {
            /* A (strictly lower), then T = (I + A)^-1 by forward substitution,
             * solved column by column: T_rj = [r==j] - sum_{j<=s<r} A_rs T_sj */
            for (long r = 0; r < n; ++r)
                for (long s = 0; s < n; ++s) {
                    double kk = 0.0;
                    for (long j = 0; j < dk; ++j) kk += K[r * dk + j] * K[s * dk + j];
                    A[r * C + s] = (s < r) ? bt[r] * exp(G[r] - G[s]) * kk : 0.0;
                }
            double *T = (double *)malloc(sizeof(double) * (size_t)(n * n));
            for (long jc = 0; jc < n; ++jc)
                for (long r = 0; r < n; ++r) {
                    double x = (r == jc) ? 1.0 : 0.0;
                    for (long s = jc; s < r; ++s) x -= A[r * C + s] * T[s * n + jc];
                    T[r * n + jc] = (r < jc) ? 0.0 : x;
                }
            /* W = T diag(beta gamma) K ; U = T diag(beta) V ; Ut = U - W S */
            for (long r = 0; r < n; ++r) {
                for (long j = 0; j < dk; ++j) {
                    double w = 0.0;
                    for (long s = 0; s < n; ++s) w += T[r * n + s] * bt[s] * exp(G[s]) * K[s * dk + j];
                    W[r * dk + j] = w;
                }
                for (long cc = 0; cc < dv; ++cc) {
                    double u = 0.0;
                    for (long s = 0; s < n; ++s) u += T[r * n + s] * bt[s] * V[s * dv + cc];
                    double ws = 0.0;
                    for (long j = 0; j < dk; ++j) ws += W[r * dk + j] * S[j * dv + cc];
                    Ut[r * dv + cc] = u - ws;
                }
            }
            free(T);
        } else {
            for (long r = 0; r < n; ++r)
                for (long cc = 0; cc < dv; ++cc) Ut[r * dv + cc] = V[r * dv + cc];
        }
        /* O = diag(gamma) Q S + (Q K^T o Gamma) Ut */
        for (long r = 0; r < n; ++r) {
            double *orow = c->o + (h * L + t0 + r) * dv;
            for (long cc = 0; cc < dv; ++cc) {
                double inter = 0.0;
                for (long j = 0; j < dk; ++j) inter += c->scale * Q[r * dk + j] * S[j * dv + cc];
                double intra = 0.0;
                for (long s = 0; s <= r; ++s) {
                    double qk = 0.0;
                    for (long j = 0; j < dk; ++j) qk += c->scale * Q[r * dk + j] * K[s * dk + j];
                    intra += qk * exp(G[r] - G[s]) * Ut[s * dv + cc];
                }
                orow[cc] = exp(G[r]) * inter + intra;
            }
        }
        /* S' = gamma_n S + sum_s exp(G_n - G_s) k_s Ut_s^T */
        for (long j = 0; j < dk; ++j)
            for (long cc = 0; cc < dv; ++cc) {
                double x = exp(G[n - 1]) * S[j * dv + cc];
                for (long s = 0; s < n; ++s) x += exp(G[n - 1] - G[s]) * K[s * dk + j] * Ut[s * dv + cc];
                S2[j * dv + cc] = x;
            }
        memcpy(S, S2, sizeof(double) * (size_t)(dk * dv));
    }
    if (c->s_final) memcpy(c->s_final + h * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
}

int oracle_chunked_fwd(const double *q, const double *k, const double *v,
                       const double *beta, const double *g, const double *s0,
                       double *o, double *s_final, long BH, long L, long dk, long dv,
                       long C, double scale, int nthreads)
{
    if (BH < 0 || L < 0 || dk < 1 || dv < 1 || C < 1) return 1;
    chk_ctx c = {q, k, v, beta, g, s0, o, s_final, L, dk, dv, C, scale};
    run_heads(chunk_head, &c, BH, 2 * dk * dv + C + C * C + C * dk + C * dv, nthreads);
    return 0;
}

/* The UT factor of one chunk (test-only): T = (I + A)^-1 with
 * A_rs = beta_r exp(G_r - G_s) k_r.k_s for s < r.  K: n x dk; T: n x n.      */
int oracle_ut_transform(const double *K, const double *beta, const double *g,
                        double *T, long n, long dk)
{
    if (n < 1 || dk < 1) return 1;
    double *G = (double *)malloc(sizeof(double) * (size_t)n);
    double acc = 0.0;
    for (long r = 0; r < n; ++r) { acc += g ? g[r] : 0.0; G[r] = acc; }
    for (long jc = 0; jc < n; ++jc)
        for (long r = 0; r < n; ++r) {
            double x = (r == jc) ? 1.0 : 0.0;
            for (long s = jc; s < r; ++s) {
                double kk = 0.0;
                for (long j = 0; j < dk; ++j) kk += K[r * dk + j] * K[s * dk + j];
                x -= beta[r] * exp(G[r] - G[s]) * kk * T[s * n + jc];
            }
            T[r * n + jc] = (r < jc) ? 0.0 : x;
        }
    free(G);
    return 0;
}
