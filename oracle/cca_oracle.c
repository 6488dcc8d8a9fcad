/*
 * CCA-Attention CPU oracle (fp64): test infrastructure only.
 *
 * Source of the method: the write-up "ICML 2025 | 全局池化+局部保留，
 * CCA-Attention为LLM长文本建模带来突破性进展" of "Core Context Aware
 * Transformers for Long Context Language Modeling".  Its formulas were lost
 * when the page was extracted; the prose of each section is restated at the
 * function that follows it, and the readings taken where the prose leaves a
 * step open are stated there too.
 *
 * Plain loops, no blocking, no online softmax, no fusion: every output is
 * computed directly from its definition.  OpenMP parallelises over
 * independent outputs only, so the arithmetic of each output is serial and
 * in a fixed order.
 */
#include "cca_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0;

int cca_oracle_set_threads(int n)
{
    if (n > 0) g_threads = n;
    return cca_oracle_threads();
}

int cca_oracle_threads(void)
{
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Local window (write-up, section 局部保留模块 "locality-preserving module"):
 * every token sees at least the w raw tokens before it, and the window is
 * aligned to the group size so that no token is lost when the sequence
 * length is not a multiple of g.
 *
 * Reading taken (the window formula itself was lost): the window of query t
 * is [ws, t] with ws the largest multiple of g that is <= max(t - w, 0).
 * It is the smallest group-aligned window that holds t and its w
 * predecessors (all of them when t < w).
 */
long cca_oracle_window_start(long t, long g, long w)
{
    long lo = t - w;
    if (lo < 0) lo = 0;
    return (lo / g) * g;
}

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += a[i] * b[i];
    return s;
}

/* Softmax of x[0..n) in place (max subtracted first). */
static void softmax_inplace(double *x, long n)
{
    double mx = -INFINITY;
    for (long i = 0; i < n; ++i)
        if (x[i] > mx) mx = x[i];
    double sum = 0.0;
    for (long i = 0; i < n; ++i) {
        x[i] = exp(x[i] - mx);
        sum += x[i];
    }
    for (long i = 0; i < n; ++i) x[i] /= sum;
}

/*
 * Globally-aware pooling (write-up, section 全局感知池化): the sequence is
 * split into non-overlapping groups of g tokens; in group j the query of the
 * group's last token scores every key of the group, the scores are
 * normalised with a softmax, and the group's tokens are averaged with these
 * importance weights into one core token.  The core keys and values are the
 * core tokens projected by the shared W_K, W_V; since the projection is
 * linear, this equals pooling the projected keys and values K, V with the
 * same weights, which is what is computed here.
 *
 * Readings taken: the score of key i is q_last . k_i / sqrt(d) (the scaled
 * dot product of ordinary attention); a trailing partial group gets no core
 * token; with grouped-query attention (r = Hq/Hkv > 1, not covered by the
 * pages, whose model has r = 1) each key/value head has one core token whose
 * weights are the mean of the r softmax vectors of its query heads.
 */
int cca_oracle_pool(const double *Q, const double *K, const double *V,
                    double *Kc, double *Vc, double *A, int B, int Hq, int Hkv,
                    long T, int d, int g)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T < 0 || d <= 0 || g <= 0)
        return CCA_ORACLE_EINVAL;
    const int r = Hq / Hkv;
    const long m = T / g;
    const double scale = 1.0 / sqrt((double)d);

#pragma omp parallel num_threads(cca_oracle_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)g);
        double *a = (double *)malloc(sizeof(double) * (size_t)g);
#pragma omp for collapse(3) schedule(static)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hkv; ++h)
                for (long j = 0; j < m; ++j) {
                    const long first = j * g, last = j * g + g - 1;
                    const double *Kh = K + ((size_t)b * Hkv + h) * T * d;
                    const double *Vh = V + ((size_t)b * Hkv + h) * T * d;
                    for (int i = 0; i < g; ++i) a[i] = 0.0;
                    for (int hq = h * r; hq < h * r + r; ++hq) {
                        const double *q =
                            Q + (((size_t)b * Hq + hq) * T + last) * d;
                        for (int i = 0; i < g; ++i)
                            s[i] = dot(q, Kh + (size_t)(first + i) * d, d) *
                                   scale;
                        softmax_inplace(s, g);
                        for (int i = 0; i < g; ++i) a[i] += s[i] / r;
                    }
                    double *kc = Kc + (((size_t)b * Hkv + h) * m + j) * d;
                    double *vc = Vc + (((size_t)b * Hkv + h) * m + j) * d;
                    for (int c = 0; c < d; ++c) {
                        double ks = 0.0, vs = 0.0;
                        for (int i = 0; i < g; ++i) {
                            ks += a[i] * Kh[(size_t)(first + i) * d + c];
                            vs += a[i] * Vh[(size_t)(first + i) * d + c];
                        }
                        kc[c] = ks;
                        vc[c] = vs;
                    }
                    if (A)
                        for (int i = 0; i < g; ++i)
                            A[(((size_t)b * Hkv + h) * m + j) * g + i] = a[i];
                }
        free(s);
        free(a);
    }
    return CCA_ORACLE_OK;
}

/*
 * Latent-condensed pooling, the LCA variant (page "Latent-Condensed
 * Transformer for Efficient Long Context Modeling", section 2 方法论,
 * 核心设计思想: 语义凝聚 and 位置锚定).  A later method by the same group:
 * history is split into groups; inside a group every token gets an
 * importance score from the dot product of the group's average query with
 * its key; the content part of the group is condensed by weighted pooling
 * with these scores, while the positional part of the key (the rotary key
 * K_R of multi-head latent attention) is not mixed: the group keeps the
 * positional key of its highest-scoring token, the anchor.
 *
 * Readings taken (the summary gives no formulas):
 *   - the average query of group j is the mean of the group's own g query
 *     rows, q_bar = (1/g) sum_i q_{jg+i}, per query head;
 *   - scores q_bar . k_i / sqrt(d) over the full key, normalised with a
 *     softmax over the group (the pooling of the earlier CCA method);
 *     with grouped-query attention the weights are the mean of the r query
 *     heads' softmax vectors, as for CCA;
 *   - the key row's last d_rope entries are its positional part and the
 *     rest its content part (in the latent form the content key and the
 *     value are linear in the latent vector C_KV, so pooling C_KV equals
 *     pooling them with the same weights); values are content only;
 *   - the anchor is the token of largest weight, the first one on a tie;
 *   - a trailing partial group gets no core token (as for CCA).
 * Writes Kc, Vc [B, Hkv, m, d]; if A is not NULL the weights [B, Hkv, m, g];
 * if anchor is not NULL the anchor index within each group [B, Hkv, m].
 */
int cca_oracle_lca_pool(const double *Q, const double *K, const double *V,
                        double *Kc, double *Vc, double *A, long *anchor, int B,
                        int Hq, int Hkv, long T, int d, int g, int d_rope)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T < 0 || d <= 0 ||
        g <= 0 || d_rope < 0 || d_rope > d)
        return CCA_ORACLE_EINVAL;
    const int r = Hq / Hkv;
    const long m = T / g;
    const int d_content = d - d_rope;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);

#pragma omp parallel num_threads(cca_oracle_threads())
    {
        double *qbar = (double *)malloc(sizeof(double) * (size_t)d);
        double *p = (double *)malloc(sizeof(double) * (size_t)g);
        double *wgt = (double *)malloc(sizeof(double) * (size_t)g);
#pragma omp for collapse(3) schedule(static)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hkv; ++h)
                for (long j = 0; j < m; ++j) {
                    const long first = j * g;
                    const double *Kg = K + (((size_t)b * Hkv + h) * T + first) * d;
                    const double *Vg = V + (((size_t)b * Hkv + h) * T + first) * d;
                    for (int i = 0; i < g; ++i) wgt[i] = 0.0;
                    for (int k = 0; k < r; ++k) {
                        const double *Qg =
                            Q + (((size_t)b * Hq + h * r + k) * T + first) * d;
                        /* the group's average query for this head */
                        for (int c = 0; c < d; ++c) {
                            double acc = 0.0;
                            for (int i = 0; i < g; ++i) acc += Qg[(size_t)i * d + c];
                            qbar[c] = acc / g;
                        }
                        for (int i = 0; i < g; ++i)
                            p[i] = dot(qbar, Kg + (size_t)i * d, d) * inv_sqrt_d;
                        softmax_inplace(p, g);
                        for (int i = 0; i < g; ++i) wgt[i] += p[i] / (double)r;
                    }
                    int best = 0;
                    for (int i = 1; i < g; ++i)
                        if (wgt[i] > wgt[best]) best = i;
                    const size_t out = ((size_t)b * Hkv + h) * m + j;
                    double *kc = Kc + out * d;
                    double *vc = Vc + out * d;
                    for (int c = 0; c < d; ++c) {
                        double kacc = 0.0, vacc = 0.0;
                        for (int i = 0; i < g; ++i) {
                            kacc += wgt[i] * Kg[(size_t)i * d + c];
                            vacc += wgt[i] * Vg[(size_t)i * d + c];
                        }
                        kc[c] = c < d_content ? kacc : Kg[(size_t)best * d + c];
                        vc[c] = vacc;
                    }
                    if (A)
                        for (int i = 0; i < g; ++i) A[out * g + i] = wgt[i];
                    if (anchor) anchor[out] = best;
                }
        free(qbar);
        free(p);
        free(wgt);
    }
    return CCA_ORACLE_OK;
}

/*
 * One query row of the fused attention (write-up, section 全局-局部模块可微融合
 * "differentiable global-local fusion"): the keys and values of the two
 * modules are concatenated into one key matrix and one value matrix, and the
 * output is a single attention over them.
 *
 * Readings taken: query t sees the core tokens of exactly the groups that
 * end before its window, j < ws(t)/g (all complete, all in the past), then
 * the raw tokens ws(t) .. t; one softmax of the 1/sqrt(d)-scaled logits over
 * that concatenation (no extra weights or gate: the fusion adds no
 * parameters).  With this split every token 0..t is reached exactly once,
 * either inside a core token or raw (the "reachability" the write-up asks
 * for in its introduction).
 *
 * keys_core[j], vals_core[j] for j < nc and keys_raw[i], vals_raw[i] for
 * i < nl are given as pointer arrays; logit is scratch of nc + nl doubles.
 */
static void attend_one(const double *q, const double *const *kcore,
                       const double *const *vcore, long nc,
                       const double *const *kraw, const double *const *vraw,
                       long nl, int d, double *logit, double *out)
{
    const double scale = 1.0 / sqrt((double)d);
    for (long j = 0; j < nc; ++j) logit[j] = dot(q, kcore[j], d) * scale;
    for (long i = 0; i < nl; ++i) logit[nc + i] = dot(q, kraw[i], d) * scale;
    softmax_inplace(logit, nc + nl);
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (long j = 0; j < nc; ++j)
        for (int c = 0; c < d; ++c) out[c] += logit[j] * vcore[j][c];
    for (long i = 0; i < nl; ++i)
        for (int c = 0; c < d; ++c) out[c] += logit[nc + i] * vraw[i][c];
}

int cca_oracle_attend_rows(const double *Q, const double *K, const double *V,
                           const double *Kc, const double *Vc, int B, int Hq,
                           int Hkv, long T, int d, int g, int w,
                           const long *rows, long nrows, double *O)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T < 0 || d <= 0 ||
        g <= 0 || w < 0 || nrows < 0)
        return CCA_ORACLE_EINVAL;
    for (long n = 0; n < nrows; ++n)
        if (rows[n] < 0 || rows[n] >= T) return CCA_ORACLE_EINVAL;
    const int r = Hq / Hkv;
    const long m = T / g;
    const long maxkeys = m + w + g + 1;

#pragma omp parallel num_threads(cca_oracle_threads())
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)maxkeys);
        const double **kp =
            (const double **)malloc(sizeof(double *) * (size_t)maxkeys);
        const double **vp =
            (const double **)malloc(sizeof(double *) * (size_t)maxkeys);
#pragma omp for collapse(3) schedule(dynamic, 4)
        for (int b = 0; b < B; ++b)
            for (int hq = 0; hq < Hq; ++hq)
                for (long n = 0; n < nrows; ++n) {
                    const int h = hq / r;
                    const long t = rows[n];
                    const long ws = cca_oracle_window_start(t, g, w);
                    const long nc = ws / g, nl = t - ws + 1;
                    const size_t kv = (size_t)b * Hkv + h;
                    for (long j = 0; j < nc; ++j) {
                        kp[j] = Kc + (kv * m + j) * d;
                        vp[j] = Vc + (kv * m + j) * d;
                    }
                    for (long i = 0; i < nl; ++i) {
                        kp[nc + i] = K + (kv * T + ws + i) * d;
                        vp[nc + i] = V + (kv * T + ws + i) * d;
                    }
                    const double *q = Q + (((size_t)b * Hq + hq) * T + t) * d;
                    double *o = O + (((size_t)b * Hq + hq) * nrows + n) * d;
                    attend_one(q, kp, vp, nc, kp + nc, vp + nc, nl, d, logit,
                               o);
                }
        free(logit);
        free(kp);
        free(vp);
    }
    return CCA_ORACLE_OK;
}

/*
 * Decode cache.  The write-up (section 基于 Triton 的底层加速) says the
 * method supports a KV cache for decoding, and (section 计算和存储效率对比)
 * that it shrinks the KV cache; the layout is not given.  Reading taken, in
 * line with the decode description of the same group's later Latent-
 * Condensed Transformer summary (section 推理流程, Decoding): keep the core
 * key/value of every completed group (slot j = group j) and the most recent
 * raw tokens in a ring (token p in slot p mod tail_cap, tail_cap >= w + g so
 * the whole local window of the newest token is present).  When a token
 * completes a group, that group is pooled from the ring; the group's last
 * token is the new token itself, so its queries do the scoring.
 */
static int cache_ok(const cca_oracle_cache *c)
{
    return c && c->B >= 0 && c->Hq > 0 && c->Hkv > 0 && c->Hq % c->Hkv == 0 &&
           c->d > 0 && c->g > 0 && c->w >= 0 && c->core_cap >= 0 &&
           c->tail_cap >= (long)c->w + c->g && c->len >= 0;
}

int cca_oracle_cache_append(cca_oracle_cache *c, const double *q,
                            const double *k, const double *v)
{
    if (!cache_ok(c)) return CCA_ORACLE_EINVAL;
    const long t = c->len;
    const int B = c->B, Hq = c->Hq, Hkv = c->Hkv, d = c->d, g = c->g;
    const int r = Hq / Hkv;
    if (t / g >= c->core_cap) return CCA_ORACLE_ECAPACITY;
    const long slot = t % c->tail_cap;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const size_t kv = (size_t)b * Hkv + h;
            memcpy(c->k_tail + (kv * c->tail_cap + slot) * d,
                   k + kv * d, sizeof(double) * d);
            memcpy(c->v_tail + (kv * c->tail_cap + slot) * d,
                   v + kv * d, sizeof(double) * d);
        }
    if ((t + 1) % g == 0) {
        const long j = t / g, first = t - g + 1;
        const double scale = 1.0 / sqrt((double)d);
        double *s = (double *)malloc(sizeof(double) * g);
        double *a = (double *)malloc(sizeof(double) * g);
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hkv; ++h) {
                const size_t kv = (size_t)b * Hkv + h;
                for (int i = 0; i < g; ++i) a[i] = 0.0;
                for (int hq = h * r; hq < h * r + r; ++hq) {
                    const double *qq = q + ((size_t)b * Hq + hq) * d;
                    for (int i = 0; i < g; ++i) {
                        const long p = first + i;
                        s[i] = dot(qq, c->k_tail + (kv * c->tail_cap +
                                                    p % c->tail_cap) * d,
                                   d) * scale;
                    }
                    softmax_inplace(s, g);
                    for (int i = 0; i < g; ++i) a[i] += s[i] / r;
                }
                double *kc = c->k_core + (kv * c->core_cap + j) * d;
                double *vc = c->v_core + (kv * c->core_cap + j) * d;
                for (int e = 0; e < d; ++e) {
                    double ks = 0.0, vs = 0.0;
                    for (int i = 0; i < g; ++i) {
                        const long p = first + i;
                        const size_t row = kv * c->tail_cap + p % c->tail_cap;
                        ks += a[i] * c->k_tail[row * d + e];
                        vs += a[i] * c->v_tail[row * d + e];
                    }
                    kc[e] = ks;
                    vc[e] = vs;
                }
            }
        free(s);
        free(a);
    }
    c->len = t + 1;
    return CCA_ORACLE_OK;
}

/*
 * Decode cache of the LCA variant (page "Latent-Condensed Transformer for
 * Efficient Long Context Modeling", section 2 方法论, 推理流程: the cache
 * keeps the condensed vectors, their anchors and the newest w tokens, and
 * condenses old groups as new tokens arrive).
 *
 * Reading taken: a group is condensed when its last token arrives, with the
 * weights and anchor of cca_oracle_lca_pool; its average query needs every
 * query row of the group, which the cache does not keep, so q_sum
 * [B, Hq, d] holds the sum of the query rows of the open group per head.
 * Token t = len: k, v go to ring slot t % tail_cap; if t completes group
 * j = t / g the group is condensed from the ring with average queries
 * (q_sum + q) / g into core slot j and q_sum restarts at zero, otherwise q
 * is added to q_sum.  Then len = t + 1.
 */
int cca_oracle_lca_cache_append(cca_oracle_cache *c, double *q_sum, const double *q,
                                const double *k, const double *v, int d_rope)
{
    if (!cache_ok(c) || !q_sum || d_rope < 0 || d_rope > c->d) return CCA_ORACLE_EINVAL;
    const long t = c->len;
    const int B = c->B, Hq = c->Hq, Hkv = c->Hkv, d = c->d, g = c->g;
    const int r = Hq / Hkv;
    if (t / g >= c->core_cap) return CCA_ORACLE_ECAPACITY;
    const long slot = t % c->tail_cap;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const size_t kv = (size_t)b * Hkv + h;
            memcpy(c->k_tail + (kv * c->tail_cap + slot) * d, k + kv * d, sizeof(double) * d);
            memcpy(c->v_tail + (kv * c->tail_cap + slot) * d, v + kv * d, sizeof(double) * d);
        }
    const size_t nq = (size_t)B * Hq * d;
    if ((t + 1) % g != 0) {
        for (size_t e = 0; e < nq; ++e) q_sum[e] += q[e];
        c->len = t + 1;
        return CCA_ORACLE_OK;
    }
    const long j = t / g, first = t - g + 1;
    const int d_content = d - d_rope;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    double *qbar = (double *)malloc(sizeof(double) * (size_t)d);
    double *p = (double *)malloc(sizeof(double) * (size_t)g);
    double *wgt = (double *)malloc(sizeof(double) * (size_t)g);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const size_t kv = (size_t)b * Hkv + h;
            for (int i = 0; i < g; ++i) wgt[i] = 0.0;
            for (int k2 = 0; k2 < r; ++k2) {
                const size_t qh = ((size_t)b * Hq + h * r + k2) * d;
                for (int e = 0; e < d; ++e) qbar[e] = (q_sum[qh + e] + q[qh + e]) / g;
                for (int i = 0; i < g; ++i) {
                    const long pos = first + i;
                    p[i] = dot(qbar, c->k_tail + (kv * c->tail_cap + pos % c->tail_cap) * d, d) *
                           inv_sqrt_d;
                }
                softmax_inplace(p, g);
                for (int i = 0; i < g; ++i) wgt[i] += p[i] / (double)r;
            }
            int best = 0;
            for (int i = 1; i < g; ++i)
                if (wgt[i] > wgt[best]) best = i;
            const size_t best_row = kv * c->tail_cap + (first + best) % c->tail_cap;
            double *kc = c->k_core + (kv * c->core_cap + j) * d;
            double *vc = c->v_core + (kv * c->core_cap + j) * d;
            for (int e = 0; e < d; ++e) {
                double kacc = 0.0, vacc = 0.0;
                for (int i = 0; i < g; ++i) {
                    const size_t row = kv * c->tail_cap + (first + i) % c->tail_cap;
                    kacc += wgt[i] * c->k_tail[row * d + e];
                    vacc += wgt[i] * c->v_tail[row * d + e];
                }
                kc[e] = e < d_content ? kacc : c->k_tail[best_row * d + e];
                vc[e] = vacc;
            }
        }
    free(qbar);
    free(p);
    free(wgt);
    for (size_t e = 0; e < nq; ++e) q_sum[e] = 0.0;
    c->len = t + 1;
    return CCA_ORACLE_OK;
}

int cca_oracle_decode(const cca_oracle_cache *c, const double *q, double *o)
{
    if (!cache_ok(c) || c->len <= 0) return CCA_ORACLE_EINVAL;
    const long t = c->len - 1;
    const int B = c->B, Hq = c->Hq, Hkv = c->Hkv, d = c->d, g = c->g;
    const int r = Hq / Hkv;
    const long ws = cca_oracle_window_start(t, g, c->w);
    const long nc = ws / g, nl = t - ws + 1;
    if (nc > c->core_cap || nl > c->tail_cap) return CCA_ORACLE_ECAPACITY;
    const long n = nc + nl;

#pragma omp parallel num_threads(cca_oracle_threads())
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)n);
        const double **kp =
            (const double **)malloc(sizeof(double *) * (size_t)n);
        const double **vp =
            (const double **)malloc(sizeof(double *) * (size_t)n);
#pragma omp for collapse(2) schedule(static)
        for (int b = 0; b < B; ++b)
            for (int hq = 0; hq < Hq; ++hq) {
                const size_t kv = (size_t)b * Hkv + hq / r;
                for (long j = 0; j < nc; ++j) {
                    kp[j] = c->k_core + (kv * c->core_cap + j) * d;
                    vp[j] = c->v_core + (kv * c->core_cap + j) * d;
                }
                for (long i = 0; i < nl; ++i) {
                    const long p = ws + i;
                    kp[nc + i] = c->k_tail + (kv * c->tail_cap +
                                              p % c->tail_cap) * d;
                    vp[nc + i] = c->v_tail + (kv * c->tail_cap +
                                              p % c->tail_cap) * d;
                }
                attend_one(q + ((size_t)b * Hq + hq) * d, kp, vp, nc,
                           kp + nc, vp + nc, nl, d, logit,
                           o + ((size_t)b * Hq + hq) * d);
            }
        free(logit);
        free(kp);
        free(vp);
    }
    return CCA_ORACLE_OK;
}
