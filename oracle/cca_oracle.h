/*
 * CCA-Attention CPU oracle: test infrastructure only.
 *
 * A plain, slow, fp64 restatement of what CCA-Attention computes, written to
 * be checked by eye against the method's description in the write-up
 * "ICML 2025 | 全局池化+局部保留，CCA-Attention为LLM长文本建模带来突破性进展"
 * (a summary of "Core Context Aware Transformers for Long Context Language
 * Modeling").  Only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, helper or constant
 * with the CUDA library, and the CUDA library never calls it.
 *
 * Notation (all tensors row-major, contiguous, float64):
 *   Q [B, Hq, T, d], K and V [B, Hkv, T, d], r = Hq / Hkv, query head hq
 *   reads key/value head hq / r.  g = group size, w = local window.
 *   m = floor(T / g) complete groups; group j holds tokens jg .. jg+g-1.
 *   ws(t) = g * floor(max(t - w, 0) / g) is the start of the local window
 *   of query t; query t attends to the core tokens of groups j < ws(t)/g and
 *   to the raw tokens ws(t) .. t, under one softmax.
 *
 * Every function returns 0 on success or a nonzero code (see below) after
 * writing nothing.
 */
#ifndef CCA_ORACLE_H
#define CCA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

#define CCA_ORACLE_OK 0
#define CCA_ORACLE_EINVAL 1
#define CCA_ORACLE_ECAPACITY 3

/* Number of OpenMP threads the oracle uses (set to n > 0; returns the
 * current setting). */
int cca_oracle_set_threads(int n);
int cca_oracle_threads(void);

/* Start of the group-aligned local window of query t. */
long cca_oracle_window_start(long t, long g, long w);

/* Globally-aware pooling.  Writes Kc, Vc [B, Hkv, m, d] and, if A is not
 * NULL, the pooling weights A [B, Hkv, m, g]. */
int cca_oracle_pool(const double *Q, const double *K, const double *V,
                    double *Kc, double *Vc, double *A, int B, int Hq, int Hkv,
                    long T, int d, int g);

/* Latent-condensed pooling (the LCA variant): weights from the group's
 * average query, content dims [0, d - d_rope) pooled, positional dims
 * [d - d_rope, d) copied from the group's highest-weight token.  Writes Kc,
 * Vc [B, Hkv, m, d]; A [B, Hkv, m, g] and anchor [B, Hkv, m] when not NULL. */
int cca_oracle_lca_pool(const double *Q, const double *K, const double *V,
                        double *Kc, double *Vc, double *A, long *anchor, int B,
                        int Hq, int Hkv, long T, int d, int g, int d_rope);

/* Fused core + local attention for the query rows listed in rows[0..nrows)
 * (every batch entry and query head).  Kc, Vc are [B, Hkv, m, d] with
 * m = floor(T / g).  Writes O [B, Hq, nrows, d]. */
int cca_oracle_attend_rows(const double *Q, const double *K, const double *V,
                           const double *Kc, const double *Vc, int B, int Hq,
                           int Hkv, long T, int d, int g, int w,
                           const long *rows, long nrows, double *O);

/* Decode-time cache: core slots (slot j = group j) and a ring of raw tokens
 * (token p in slot p mod tail_cap).  Buffers are owned by the caller. */
typedef struct {
    double *k_core, *v_core; /* [B, Hkv, core_cap, d] */
    double *k_tail, *v_tail; /* [B, Hkv, tail_cap, d] */
    int B, Hq, Hkv, d, g, w;
    long core_cap, tail_cap, len;
} cca_oracle_cache;

/* Append token t = len: store k, v [B, Hkv, d] in the tail; when the token
 * completes group j = t / g, pool that group with the token's own queries
 * q [B, Hq, d] into core slot j.  Then len = t + 1. */
int cca_oracle_cache_append(cca_oracle_cache *c, const double *q,
                            const double *k, const double *v);

/* LCA variant: append token t = len (ring slot t % tail_cap); q_sum
 * [B, Hq, d] holds the open group's query sums, to which q is added, or, if
 * t completes group j = t / g, the group is condensed as cca_oracle_lca_pool
 * does, with average queries (q_sum + q) / g, into core slot j and q_sum is
 * zeroed.  Then len = t + 1. */
int cca_oracle_lca_cache_append(cca_oracle_cache *c, double *q_sum, const double *q,
                                const double *k, const double *v, int d_rope);

/* Attention of the newest token t = len - 1 with queries q [B, Hq, d] over
 * the cache; writes o [B, Hq, d]. */
int cca_oracle_decode(const cca_oracle_cache *c, const double *q, double *o);

#ifdef __cplusplus
}
#endif
#endif
