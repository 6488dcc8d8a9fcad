/*
 * libcca: CCA-Attention (Core Context Aware attention) on NVIDIA B200
 * (sm_100a), as a C ABI.
 *
 * The method is the one described in the write-up "ICML 2025 | 全局池化+局部
 * 保留，CCA-Attention为LLM长文本建模带来突破性进展" of the paper "Core Context
 * Aware Transformers for Long Context Language Modeling":
 *
 *  - globally-aware pooling (section 全局感知池化): the sequence is cut into
 *    non-overlapping groups of g tokens; the query of each group's last
 *    token scores the group's keys, softmax(q . k / sqrt(d)), and those
 *    weights average the group's keys and values into one core key/value;
 *  - locality-preserving module (section 局部保留模块): every token also sees
 *    the raw keys/values of a window of at least w preceding tokens, aligned
 *    to the group size;
 *  - global-local fusion (section 全局-局部模块可微融合): one softmax over the
 *    concatenation of the core and the raw keys;
 *  - KV-cache support for decoding (section 基于 Triton 的底层加速).
 *
 * Definitions used by every call (r = Hq / Hkv; query head hq reads
 * key/value head hq / r):
 *   m          = floor(T / g) complete groups; group j = tokens jg..jg+g-1
 *   ws(t)      = g * floor(max(t - w, 0) / g), start of t's local window
 *   query t attends to core keys/values of groups j < ws(t) / g and to raw
 *   keys/values ws(t)..t, all scaled by 1/sqrt(d), under one softmax.
 *   Grouped-query attention (r > 1): each key/value head gets one core
 *   key/value per group, weighted by the mean of its r query heads' softmax
 *   vectors.
 *
 * Data: Q, K, V and raw cache rows are bf16; core keys/values (Kc, Vc and
 * the cache's core slots) are fp16, whose 11 significant bits keep the
 * error of the pooled rows of large keys well inside the attention's error
 * budget.  All tensors are row-major and contiguous, layout [B, H, T, d]
 * ("head-major"); d is 64 or 128.  Arithmetic is fp32 (scores, softmax,
 * accumulation) with bf16 (raw keys) or fp16 (core keys) tensor-core
 * operands.  Because core rows and the query copy used against them are
 * fp16, input magnitudes must stay below 65504; larger values are clamped
 * and reported as CCA_ERR_RANGE by cca_device_status().
 *
 * Memory: every pointer is a device pointer owned by the caller and
 * borrowed for the call; the library allocates nothing.  Calls are
 * asynchronous on the given stream (the CUDA runtime's cudaStream_t; 0 is
 * the legacy default stream).  Outputs must not alias inputs.  Pointers
 * must be 16-byte aligned (the per-row length arrays: 8-byte).
 *
 * Errors: argument checks run on the host before any launch; a call that
 * fails them returns a nonzero status and writes nothing.  CCA_ERR_CUDA
 * reports a launch error.  Device-side waits are bounded: a wait that runs
 * out records a timeout in a device status word and the kernel returns
 * early; cca_device_status() reads and clears it (and the fp16 range and
 * per-row capacity flags).
 */
#ifndef CCA_H
#define CCA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CCA_OK = 0,
    CCA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or shape */
    CCA_ERR_UNSUPPORTED = 2, /* d not 64/128, g or w beyond the limits     */
    CCA_ERR_CAPACITY = 3,    /* cache has no room for the request          */
    CCA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed          */
    CCA_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out         */
    CCA_ERR_RANGE = 6,       /* a value beyond the fp16 range was clamped  */
    CCA_ERR_SCRATCH = 7      /* request exceeds the library's fixed scratch */
} cca_status;

/* Element type of an output that may be written in either precision. */
typedef enum { CCA_BF16 = 0, CCA_F32 = 1 } cca_dtype;

/* Largest group size the kernels accept. */
#define CCA_MAX_G 256

/*
 * Decode cache (section 基于 Triton 的底层加速 says the kernel supports a KV
 * cache; section 计算和存储效率对比 that it shrinks it).  It holds the core
 * key/value of every completed group and the newest raw tokens in a ring:
 *   k_core, v_core: fp16 [B, Hkv, core_cap, d]; slot j = group j
 *   k_tail, v_tail: bf16 [B, Hkv, tail_cap, d]; token p in slot p % tail_cap
 * tail_cap >= w + g keeps the whole local window of the newest token.
 * All batch rows share one length `len` (tokens appended so far), which the
 * host keeps in this struct.  The buffers belong to the caller.
 */
typedef struct {
    void *k_core, *v_core;
    void *k_tail, *v_tail;
    int B, Hq, Hkv, d, g, w;
    int64_t core_cap, tail_cap;
    int64_t len;
} cca_cache;

/*
 * Globally-aware pooling (section 全局感知池化).
 *   Q [B, Hq, T, d], K and V [B, Hkv, T, d]  (bf16, read)
 *   Kc, Vc [B, Hkv, m, d], m = floor(T / g)  (fp16, written)
 * For each (b, kv head h, group j) the scores of the group's last query
 * against the group's keys are soft-maxed (per query head, averaged over
 * the r query heads of h) and pool that group's keys and values.  A trailing
 * partial group is not pooled.  1 <= g <= CCA_MAX_G.
 */
cca_status cca_pool(const void *Q, const void *K, const void *V, void *Kc,
                    void *Vc, int B, int Hq, int Hkv, int64_t T, int d, int g,
                    cudaStream_t stream);

/*
 * Fused core + local attention for a whole sequence (sections 局部保留模块
 * and 全局-局部模块可微融合).
 *   Q [B, Hq, T, d], K, V [B, Hkv, T, d] (bf16), Kc, Vc [B, Hkv, m, d]
 *   (fp16, from cca_pool), O [B, Hq, T, d] written in o_dtype (bf16 or
 *   fp32), 32-byte aligned (CCA_ERR_INVALID_ARG otherwise).
 * O[t] = softmax over { q_t . Kc[j] / sqrt(d) : j < ws(t)/g } and
 * { q_t . K[i] / sqrt(d) : ws(t) <= i <= t } applied to [Vc ; V].
 * Runs on tcgen05 tensor cores with TMA-staged tiles.
 */
cca_status cca_attn_prefill(const void *Q, const void *K, const void *V,
                            const void *Kc, const void *Vc, void *O,
                            cca_dtype o_dtype, int B, int Hq, int Hkv,
                            int64_t T, int d, int g, int w,
                            cudaStream_t stream);

/*
 * Training: the forward attention of cca_attn_prefill that also writes
 * each row's log-sum-exp, lse [B, Hq, T] (fp32, device memory, log2 units:
 * lse[t] = log2 of the sum over t's keys of 2^(q_t . key * log2(e) /
 * sqrt(d))), which cca_attn_backward reads.  Other arguments, results and
 * errors as cca_attn_prefill.
 */
cca_status cca_attn_prefill_lse(const void *Q, const void *K, const void *V, const void *Kc,
                                const void *Vc, void *O, cca_dtype o_dtype, float *lse, int B,
                                int Hq, int Hkv, int64_t T, int d, int g, int w,
                                cudaStream_t stream);

/* Bytes of device workspace cca_attn_backward needs for these shapes
 * (0 for an invalid shape). */
size_t cca_attn_backward_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int d, int g);

/*
 * Backward pass for training (the write-up's section 全局-局部模块可微融合
 * calls the global-local fusion differentiable, and its section 基于 Triton
 * 的底层加速 says the fused operator serves training): for an upstream
 * gradient dO of the attention output, the gradients of
 * L = sum(dO * O) with respect to Q, K and V, through the fused attention
 * (queries, raw window keys/values, pooled core keys/values) and through
 * the pooling (section 全局感知池化: each group's weights come from its last
 * query and its keys).
 *   Q, K, V, Kc, Vc as for cca_attn_prefill; O and lse from
 *   cca_attn_prefill_lse on the same inputs (O in o_dtype); dO [B, Hq, T, d]
 *   bf16.  dQ [B, Hq, T, d], dK, dV [B, Hkv, T, d]: fp32, written, each
 *   32-byte aligned (CCA_ERR_INVALID_ARG otherwise).
 *   workspace: cca_attn_backward_workspace_bytes bytes of device memory,
 *   256-byte aligned (fp16 copies of Q and dO, per-row sums, fp32 core
 *   gradients; the call clears what it accumulates).  r = Hq / Hkv <= 32.
 * Runs as four launches on `stream` (per-row sums; dQ on tcgen05 tensor
 * cores, persistent CTAs taking one 128-row query tile at a time; dK, dV on
 * tcgen05, persistent CTAs taking one 128-key tile at a time; the pooling's
 * chain rule, one warp per group).  Errors as
 * cca_attn_prefill; values beyond the fp16 range in Q or dO are clamped in
 * the core stream's copies and reported as CCA_ERR_RANGE.
 */
cca_status cca_attn_backward(const void *Q, const void *K, const void *V, const void *Kc,
                             const void *Vc, const void *O, cca_dtype o_dtype,
                             const float *lse, const void *dO, float *dQ, float *dK,
                             float *dV, int B, int Hq, int Hkv, int64_t T, int d, int g,
                             int w, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/*
 * Fill a cache from a prefix of T tokens (Q, K, V as for cca_pool).  The
 * write-up's section 基于 Triton 的底层加速 gives the operator KV-cache
 * support for prefill and decode; section 计算和存储效率对比 measures the
 * cache's size against full attention.  This call pools every complete
 * group into its core slot (section 全局感知池化) and copies the last
 * min(T, tail_cap) raw tokens into their ring slots (the window of
 * section 局部保留模块); it sets c->len = T.
 * CCA_ERR_CAPACITY if floor((T - 1) / g) >= core_cap.  The cache's shape
 * fields (B, Hq, Hkv, d, g, w, core_cap, tail_cap) must be set.
 */
cca_status cca_cache_prefill(cca_cache *c, const void *Q, const void *K,
                             const void *V, int64_t T, cudaStream_t stream);

/*
 * Append one token t = c->len per batch row (KV-cache support, section
 * 基于 Triton 的底层加速; pooling of a completed group, section
 * 全局感知池化): q_t [B, Hq, d], k_t, v_t [B, Hkv, d] (bf16).  k_t, v_t
 * go to ring slot t % tail_cap; if the token completes group j = t / g
 * ((t + 1) % g == 0), that group is pooled from the ring with the token's
 * own queries (it is the group's last token) into core slot j.  On success c->len becomes t + 1.  CCA_ERR_CAPACITY (nothing
 * written) if t / g >= core_cap.
 */
cca_status cca_cache_append(cca_cache *c, const void *q_t, const void *k_t,
                            const void *v_t, cudaStream_t stream);

/* Bytes of device workspace cca_attn_decode needs for this cache (for its
 * current and any smaller length). */
size_t cca_decode_workspace_bytes(const cca_cache *c);

/*
 * Attention of the newest token t = c->len - 1 over the cache: core slots
 * j < ws(t)/g and ring slots of tokens ws(t)..t, one softmax (the fused
 * core + local attention of sections 局部保留模块 and 全局-局部模块可微融合,
 * for one query, from the cache of section 基于 Triton 的底层加速).
 *   q_t [B, Hq, d] (bf16), o_t [B, Hq, d] written in o_dtype.
 * Split over key ranges; partial results go to `workspace` (device memory
 * of at least cca_decode_workspace_bytes(c) bytes, 256-byte aligned, its
 * contents need no initialisation: the call clears the few counters it
 * uses with cudaMemsetAsync on `stream`).  The last block of each (batch,
 * kv head) to finish combines the partials, in the same kernel.
 */
cca_status cca_attn_decode(const cca_cache *c, const void *q_t, void *o_t,
                           cca_dtype o_dtype, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/*
 * One decode step in one launch: cca_cache_append of token t = c->len
 * followed by cca_attn_decode of that token, fused into a single kernel
 * (the write-up's section 基于 Triton 的底层加速 describes one
 * cache-friendly operator with native KV-cache support; sections
 * 全局感知池化, 局部保留模块 and 全局-局部模块可微融合 define what it
 * computes).  Arguments as for the two calls: q_t [B, Hq, d], k_t, v_t
 * [B, Hkv, d] (bf16), o_t [B, Hq, d] in o_dtype.  The results, and the
 * cache contents afterwards, equal those of the two separate calls.  On
 * success c->len becomes t + 1; CCA_ERR_CAPACITY (nothing launched) if
 * t / g >= core_cap.
 * Workspace: as for cca_attn_decode (cca_decode_workspace_bytes(c) bytes,
 * 256-byte aligned), but this call does not clear the completion counters
 * it keeps there: zero-fill a workspace once before its first use with a
 * cache (e.g. cudaMemsetAsync(ws, 0, bytes, stream)).  Every decode call of
 * this library (this one, cca_attn_decode, cca_attn_decode_rows) leaves the
 * counters at zero when it completes, so the workspace stays ready for the
 * next call on the same cache.  Calls sharing a workspace must not overlap
 * on the GPU.
 */
cca_status cca_decode_step(cca_cache *c, const void *q_t, const void *k_t, const void *v_t,
                           void *o_t, cca_dtype o_dtype, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/*
 * Per-row lengths in device memory (the same cache append and decode
 * attention as above, sections 基于 Triton 的底层加速, 全局感知池化,
 * 局部保留模块 and 全局-局部模块可微融合).  These two calls read each batch
 * row's length from `lens` (device memory, B entries of long long, 8-byte
 * aligned) instead of c->len, so rows may have different lengths and a
 * sequence of decode steps can be captured once in a CUDA graph and
 * replayed (nothing the host must know changes from step to step).
 * c->len is neither read nor written.  lens[b] must be the number of tokens
 * row b holds: as set when the row was filled (cca_cache_prefill of that
 * row) and advanced by cca_cache_append_rows.  The library cannot tell a
 * larger value from a real length: a row whose lens[b] runs ahead of what
 * was appended is decoded from stale ring and core slots, and only a length
 * beyond the cache's capacity is reported.
 *
 * cca_cache_append_rows: row b appends its token t = lens[b] exactly as
 * cca_cache_append does (ring slot t % tail_cap, pooling of group t / g when
 * the token completes it), then sets lens[b] = t + 1, all on the device.  A
 * row whose token would not fit (t / g >= core_cap) is left unchanged and
 * cca_device_status() reports CCA_ERR_CAPACITY.  Requires Hkv <= 32 (one
 * warp per key/value head in one block per row): CCA_ERR_UNSUPPORTED
 * otherwise.
 */
cca_status cca_cache_append_rows(const cca_cache *c, long long *lens, const void *q_t,
                                 const void *k_t, const void *v_t, cudaStream_t stream);

/*
 * cca_attn_decode_rows (sections 局部保留模块 and 全局-局部模块可微融合 for
 * one query per row): cca_attn_decode for token t_b = lens[b] - 1 of every
 * row b, each over its own core slots and ring window.  The workspace
 * is the same as cca_attn_decode's.  A row with lens[b] == 0 gets a zero
 * output; a row longer than the cache gets a zero output and
 * cca_device_status() reports CCA_ERR_CAPACITY.
 */
cca_status cca_attn_decode_rows(const cca_cache *c, const long long *lens, const void *q_t,
                                void *o_t, cca_dtype o_dtype, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/* Size of the library's fixed decode scratch (bytes): the largest
 * cca_decode_workspace_bytes() that cca_attn_decode_noalloc can serve. */
#define CCA_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * cca_attn_decode without a caller-provided workspace.  The paper has no
 * counterpart: this is a service for callers that cannot allocate device
 * memory, such as runtimes that plan all device memory up front and forbid
 * other allocations, plug-in hosts that only pass input and output pointers,
 * or latency-critical loops that cannot afford cudaMalloc (which may
 * synchronise the device).  It computes exactly what cca_attn_decode
 * computes, with the split-K partials in a fixed array of
 * CCA_NOALLOC_SCRATCH_BYTES that the library holds on every GPU it is loaded
 * on until the process exits; it allocates nothing.
 *   Returns CCA_ERR_SCRATCH (nothing launched) if the cache needs more
 *   workspace than that array; other errors as cca_attn_decode.
 *   The first call in each CUDA context (once per device for the runtime's
 *   primary contexts, and again after a context is re-created, e.g. after
 *   cudaDeviceReset) looks up the array's device address with that context
 *   current, so make it before any stream capture begins.
 *   All calls share the array: calls whose kernels may overlap on the GPU
 *   (e.g. on unordered streams) race.  Nothing in it needs clearing.
 */
cca_status cca_attn_decode_noalloc(const cca_cache *c, const void *q_t, void *o_t,
                                   cca_dtype o_dtype, cudaStream_t stream);

/*
 * The LCA variant (page "Latent-Condensed Transformer for Efficient Long
 * Context Modeling", section 2 方法论, 核心设计思想): a later method by the
 * authors of CCA that condenses each group differently and keeps the same
 * core + local attention.  Per group of g tokens and key/value head:
 *   - semantic condensation (语义凝聚): every query head's average query
 *     over the group's own g query rows scores the group's keys,
 *     q_bar . k / sqrt(d); softmax per query head, mean over the r query
 *     heads of the key/value head; the weights pool the value and the
 *     content part of the key (entries [0, d - d_rope));
 *   - positional anchoring (位置锚定): the positional part of the key (the
 *     last d_rope entries: the rotary key of latent attention) is not mixed
 *     but copied from the group's highest-weight token (the first one on a
 *     tie).
 * d_rope: 0 <= d_rope <= d, a multiple of 8 (CCA_ERR_INVALID_ARG
 * otherwise).  The condensed rows (fp16, range clamp as for cca_pool) feed
 * cca_attn_prefill and cca_attn_decode unchanged: the local window and the
 * single softmax over [core ; raw] (section 局部上下文保留 and 推理流程 of
 * that page) are CCA's.
 */

/* Condensation of every complete group: arguments, layout and errors as
 * cca_pool, plus d_rope.  Reads every query row (the group averages), not
 * only each group's last. */
cca_status cca_lca_pool(const void *Q, const void *K, const void *V, void *Kc, void *Vc, int B,
                        int Hq, int Hkv, int64_t T, int d, int g, int d_rope,
                        cudaStream_t stream);

/*
 * Decode cache for the LCA variant (推理流程 of that page: the cache keeps
 * the condensed rows and the newest w tokens, and condenses each group as
 * it completes).  q_sum [B, Hq, d] (fp32, device memory, 16-byte aligned,
 * caller-owned) holds per query head the sum of the query rows of the open
 * (incomplete) group: a completed group needs its average query, and a
 * query row is not kept once its token is appended.
 *
 * cca_lca_cache_prefill: as cca_cache_prefill, with cca_lca_pool's
 * condensation; sets q_sum to the sums of the trailing partial group's
 * query rows (zero if T is a multiple of g) and c->len = T.
 *
 * cca_lca_cache_append: as cca_cache_append for token t = c->len (ring slot
 * t % tail_cap); adds q_t to q_sum, or, if t completes group j = t / g,
 * condenses group j from the ring with average queries (q_sum + q_t) / g
 * into core slot j and zeroes q_sum.  c->len becomes t + 1.
 * CCA_ERR_CAPACITY (nothing written) if t / g >= core_cap.
 *
 * The same q_sum and d_rope must serve every call on one cache.  Decode
 * attention is cca_attn_decode on the same cache.
 */
cca_status cca_lca_cache_prefill(cca_cache *c, float *q_sum, const void *Q, const void *K,
                                 const void *V, int64_t T, int d_rope, cudaStream_t stream);
cca_status cca_lca_cache_append(cca_cache *c, float *q_sum, const void *q_t, const void *k_t,
                                const void *v_t, int d_rope, cudaStream_t stream);

/*
 * Synchronise `stream`, then report CCA_ERR_CUDA if a CUDA error is
 * pending, CCA_ERR_TIMEOUT if any kernel of this library recorded a
 * timed-out wait since the last call, CCA_ERR_CAPACITY if a per-row call
 * met a row longer than its cache, CCA_ERR_RANGE if one clamped a value to
 * the fp16 range, else CCA_OK.  The records are cleared.
 */
cca_status cca_device_status(cudaStream_t stream);

/*
 * Failure-path self-test: launch on `stream` one small kernel that waits,
 * with the library's bounded wait and a limit of `limit_us` microseconds
 * (1 .. 2000000), on a barrier that nothing completes.  The wait runs out
 * and the kernel records a timeout, so a later cca_device_status(stream)
 * returns CCA_ERR_TIMEOUT, and the context stays usable (no fault, trap or
 * hang).  The pages define no such step; it lets callers and tests check
 * how the library reports a stuck kernel.  CCA_ERR_INVALID_ARG for a limit
 * outside the range (nothing launched), CCA_ERR_CUDA on a launch error.
 */
cca_status cca_selftest_wait_timeout(unsigned int limit_us, cudaStream_t stream);

/* Human-readable name of a status. */
const char *cca_status_string(cca_status s);

/* Library version, "major.minor.patch". */
const char *cca_version(void);

/* Text of the CUDA error behind the calling thread's last CCA_ERR_CUDA
 * ("no error" if there was none).  The string is static. */
const char *cca_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* CCA_H */
