// The C ABI of libcca (include/cca.h): argument checks on the host, then
// the kernel launches.  A call that fails a check returns its status before
// touching the GPU.
#include "../../include/cca.h"
#include "common.cuh"
#include "internal.h"

#include <cstdint>

namespace {

constexpr int64_t kMaxT = (int64_t(1) << 31) - 256;  // 32-bit row indices

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool ptr_ok(const void *p, bool needed)
{
    return !needed || (p != nullptr && aligned16(p));
}

bool overlap(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

cca_status shape_status(int B, int Hq, int Hkv, int64_t T, int d, int g, int w)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || T < 0 || g < 1 || w < 0)
        return CCA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return CCA_ERR_UNSUPPORTED;
    if (g > CCA_MAX_G || T > kMaxT || w > (1 << 30)) return CCA_ERR_UNSUPPORTED;
    // pooling scratch: 8 warps x (r*g + g) floats of shared memory
    const int64_t r = Hq / Hkv;
    if ((r + 1) * g > 7000) return CCA_ERR_UNSUPPORTED;
    return CCA_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

cca_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return CCA_OK;
    g_last_cuda_error = e;
    return CCA_ERR_CUDA;
}

cca_status cache_status(const cca_cache *c)
{
    if (!c) return CCA_ERR_INVALID_ARG;
    const cca_status s = shape_status(c->B, c->Hq, c->Hkv, 0, c->d, c->g, c->w);
    if (s != CCA_OK) return s;
    if (c->core_cap < 0 || c->tail_cap < static_cast<int64_t>(c->w) + c->g ||
        c->len < 0)
        return CCA_ERR_INVALID_ARG;
    if (c->Hq / c->Hkv > 16) return CCA_ERR_UNSUPPORTED;
    if (!ptr_ok(c->k_tail, true) || !ptr_ok(c->v_tail, true) ||
        !ptr_ok(c->k_core, c->core_cap > 0) || !ptr_ok(c->v_core, c->core_cap > 0))
        return CCA_ERR_INVALID_ARG;
    return CCA_OK;
}

}  // namespace

extern "C" {

cca_status cca_pool(const void *Q, const void *K, const void *V, void *Kc, void *Vc,
                    int B, int Hq, int Hkv, int64_t T, int d, int g, cudaStream_t stream)
{
    const cca_status s = shape_status(B, Hq, Hkv, T, d, g, 0);
    if (s != CCA_OK) return s;
    const int64_t m = T / g;
    const bool any = m > 0;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(Kc, any) ||
        !ptr_ok(Vc, any))
        return CCA_ERR_INVALID_ARG;
    if (!any) return CCA_OK;
    const size_t in_q = size_t(B) * Hq * T * d * 2, in_kv = size_t(B) * Hkv * T * d * 2;
    const size_t out = size_t(B) * Hkv * m * d * 2;
    if (overlap(Kc, out, Q, in_q) || overlap(Kc, out, K, in_kv) ||
        overlap(Kc, out, V, in_kv) || overlap(Vc, out, Q, in_q) ||
        overlap(Vc, out, K, in_kv) || overlap(Vc, out, V, in_kv) ||
        overlap(Kc, out, Vc, out))
        return CCA_ERR_INVALID_ARG;
    return from_cuda(cca::launch_pool(Q, K, V, Kc, Vc, B, Hq, Hkv, T, d, g, m, stream));
}

cca_status cca_attn_prefill(const void *Q, const void *K, const void *V, const void *Kc,
                            const void *Vc, void *O, cca_dtype o_dtype, int B, int Hq,
                            int Hkv, int64_t T, int d, int g, int w, cudaStream_t stream)
{
    const cca_status s = shape_status(B, Hq, Hkv, T, d, g, w);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    const bool any = T > 0;
    const int64_t m = T / g;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(O, any) ||
        !ptr_ok(Kc, m > 0) || !ptr_ok(Vc, m > 0))
        return CCA_ERR_INVALID_ARG;
    if (any && (reinterpret_cast<uintptr_t>(O) & 31u) != 0)
        return CCA_ERR_INVALID_ARG;  // output rows are written with 32-byte stores
    if (!any) return CCA_OK;
    const int64_t n_items = ((T + 255) / 256) * int64_t(B) * Hq;
    if (n_items > INT32_MAX) return CCA_ERR_UNSUPPORTED;
    const size_t esz = o_dtype == CCA_F32 ? 4 : 2;
    const size_t out = size_t(B) * Hq * T * d * esz;
    const size_t in_q = size_t(B) * Hq * T * d * 2, in_kv = size_t(B) * Hkv * T * d * 2;
    const size_t in_c = size_t(B) * Hkv * m * d * 2;
    if (overlap(O, out, Q, in_q) || overlap(O, out, K, in_kv) || overlap(O, out, V, in_kv) ||
        overlap(O, out, Kc, in_c) || overlap(O, out, Vc, in_c))
        return CCA_ERR_INVALID_ARG;
    return from_cuda(cca::launch_prefill(Q, K, V, Kc, Vc, O, o_dtype == CCA_F32, B, Hq,
                                         Hkv, T, d, g, w, stream));
}

cca_status cca_attn_prefill_lse(const void *Q, const void *K, const void *V, const void *Kc,
                                const void *Vc, void *O, cca_dtype o_dtype, float *lse, int B,
                                int Hq, int Hkv, int64_t T, int d, int g, int w,
                                cudaStream_t stream)
{
    const cca_status s = shape_status(B, Hq, Hkv, T, d, g, w);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    const bool any = T > 0;
    const int64_t m = T / g;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(O, any) ||
        !ptr_ok(lse, any) || !ptr_ok(Kc, m > 0) || !ptr_ok(Vc, m > 0))
        return CCA_ERR_INVALID_ARG;
    if (any && (reinterpret_cast<uintptr_t>(O) & 31u) != 0)
        return CCA_ERR_INVALID_ARG;  // output rows are written with 32-byte stores
    if (!any) return CCA_OK;
    const int64_t n_items = ((T + 255) / 256) * int64_t(B) * Hq;
    if (n_items > INT32_MAX) return CCA_ERR_UNSUPPORTED;
    const size_t esz = o_dtype == CCA_F32 ? 4 : 2;
    const size_t out = size_t(B) * Hq * T * d * esz, lse_b = size_t(B) * Hq * T * 4;
    const size_t in_q = size_t(B) * Hq * T * d * 2, in_kv = size_t(B) * Hkv * T * d * 2;
    const size_t in_c = size_t(B) * Hkv * m * d * 2;
    if (overlap(O, out, Q, in_q) || overlap(O, out, K, in_kv) || overlap(O, out, V, in_kv) ||
        overlap(O, out, Kc, in_c) || overlap(O, out, Vc, in_c) || overlap(lse, lse_b, O, out) ||
        overlap(lse, lse_b, Q, in_q) || overlap(lse, lse_b, K, in_kv) ||
        overlap(lse, lse_b, V, in_kv) || overlap(lse, lse_b, Kc, in_c) ||
        overlap(lse, lse_b, Vc, in_c))
        return CCA_ERR_INVALID_ARG;
    return from_cuda(cca::launch_prefill(Q, K, V, Kc, Vc, O, o_dtype == CCA_F32, B, Hq, Hkv, T,
                                         d, g, w, stream, lse));
}

size_t cca_attn_backward_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int d, int g)
{
    if (shape_status(B, Hq, Hkv, T, d, g, 0) != CCA_OK) return 0;
    return cca::bw_layout(B, Hq, Hkv, T, d, g).total;
}

cca_status cca_attn_backward(const void *Q, const void *K, const void *V, const void *Kc,
                             const void *Vc, const void *O, cca_dtype o_dtype,
                             const float *lse, const void *dO, float *dQ, float *dK,
                             float *dV, int B, int Hq, int Hkv, int64_t T, int d, int g,
                             int w, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream)
{
    const cca_status s = shape_status(B, Hq, Hkv, T, d, g, w);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    if (Hq / Hkv > 32) return CCA_ERR_UNSUPPORTED;
    const bool any = T > 0;
    const int64_t m = T / g;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(O, any) ||
        !ptr_ok(lse, any) || !ptr_ok(dO, any) || !ptr_ok(dQ, any) || !ptr_ok(dK, any) ||
        !ptr_ok(dV, any) || !ptr_ok(Kc, m > 0) || !ptr_ok(Vc, m > 0))
        return CCA_ERR_INVALID_ARG;
    // the gradient rows are written with 32-byte stores
    if (any && ((reinterpret_cast<uintptr_t>(dQ) | reinterpret_cast<uintptr_t>(dK) |
                 reinterpret_cast<uintptr_t>(dV)) & 31u) != 0)
        return CCA_ERR_INVALID_ARG;
    if (!any) return CCA_OK;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < cca::bw_layout(B, Hq, Hkv, T, d, g).total)
        return CCA_ERR_INVALID_ARG;
    if (((T + 127) / 128) * int64_t(B) * Hq > INT32_MAX) return CCA_ERR_UNSUPPORTED;
    // the outputs alias nothing the call reads, nor each other, nor the workspace
    const size_t nq = size_t(B) * Hq * T * d, nk = size_t(B) * Hkv * T * d;
    const size_t nc = size_t(B) * Hkv * m * d;
    const void *ins[9] = {Q, K, V, Kc, Vc, O, lse, dO, workspace};
    const size_t in_n[9] = {nq * 2, nk * 2, nk * 2, nc * 2, nc * 2,
                            nq * (o_dtype == CCA_F32 ? 4 : 2), size_t(B) * Hq * T * 4, nq * 2,
                            workspace_bytes};
    void *outs[3] = {dQ, dK, dV};
    const size_t out_n[3] = {nq * 4, nk * 4, nk * 4};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 9; ++j)
            if (overlap(outs[i], out_n[i], ins[j], in_n[j])) return CCA_ERR_INVALID_ARG;
        for (int j = i + 1; j < 3; ++j)
            if (overlap(outs[i], out_n[i], outs[j], out_n[j])) return CCA_ERR_INVALID_ARG;
    }
    return from_cuda(cca::launch_backward(Q, K, V, Kc, Vc, O, o_dtype == CCA_F32, lse, dO, dQ, dK,
                                          dV, B, Hq, Hkv, T, d, g, w, workspace, stream));
}

cca_status cca_cache_prefill(cca_cache *c, const void *Q, const void *K, const void *V,
                             int64_t T, cudaStream_t stream)
{
    cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (T < 0 || T > kMaxT) return CCA_ERR_INVALID_ARG;
    const bool any = T > 0;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any))
        return CCA_ERR_INVALID_ARG;
    if (any && (T - 1) / c->g >= c->core_cap) return CCA_ERR_CAPACITY;
    if (any) {
        cudaError_t e = cca::launch_pool(Q, K, V, c->k_core, c->v_core, c->B, c->Hq,
                                         c->Hkv, T, c->d, c->g, c->core_cap, stream);
        if (e != cudaSuccess) return from_cuda(e);
        const int64_t p0 = T > c->tail_cap ? T - c->tail_cap : 0;
        e = cca::launch_tail_fill(K, V, c->k_tail, c->v_tail, c->B, c->Hkv, T, c->d, p0,
                                  c->tail_cap, stream);
        if (e != cudaSuccess) return from_cuda(e);
    }
    c->len = T;
    return CCA_OK;
}

cca_status cca_cache_append(cca_cache *c, const void *q_t, const void *k_t,
                            const void *v_t, cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (!ptr_ok(q_t, true) || !ptr_ok(k_t, true) || !ptr_ok(v_t, true))
        return CCA_ERR_INVALID_ARG;
    const int64_t t = c->len;
    if (t >= kMaxT || t / c->g >= c->core_cap) return CCA_ERR_CAPACITY;
    const cudaError_t e = cca::launch_append(q_t, k_t, v_t, c->k_core, c->v_core,
                                             c->k_tail, c->v_tail, c->B, c->Hq, c->Hkv,
                                             c->d, c->g, c->core_cap, c->tail_cap, t,
                                             stream);
    if (e != cudaSuccess) return from_cuda(e);
    c->len = t + 1;
    return CCA_OK;
}

// ---- the LCA variant -------------------------------------------------------

cca_status cca_lca_pool(const void *Q, const void *K, const void *V, void *Kc, void *Vc, int B,
                        int Hq, int Hkv, int64_t T, int d, int g, int d_rope,
                        cudaStream_t stream)
{
    const cca_status s = shape_status(B, Hq, Hkv, T, d, g, 0);
    if (s != CCA_OK) return s;
    if (d_rope < 0 || d_rope > d || d_rope % 8 != 0) return CCA_ERR_INVALID_ARG;
    const int64_t m = T / g;
    const bool any = m > 0;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(Kc, any) ||
        !ptr_ok(Vc, any))
        return CCA_ERR_INVALID_ARG;
    if (!any) return CCA_OK;
    const size_t in_q = size_t(B) * Hq * T * d * 2, in_kv = size_t(B) * Hkv * T * d * 2;
    const size_t out = size_t(B) * Hkv * m * d * 2;
    if (overlap(Kc, out, Q, in_q) || overlap(Kc, out, K, in_kv) ||
        overlap(Kc, out, V, in_kv) || overlap(Vc, out, Q, in_q) ||
        overlap(Vc, out, K, in_kv) || overlap(Vc, out, V, in_kv) ||
        overlap(Kc, out, Vc, out))
        return CCA_ERR_INVALID_ARG;
    return from_cuda(
        cca::launch_lca_pool(Q, K, V, Kc, Vc, B, Hq, Hkv, T, d, g, d_rope, m, stream));
}

cca_status cca_lca_cache_prefill(cca_cache *c, float *q_sum, const void *Q, const void *K,
                                 const void *V, int64_t T, int d_rope, cudaStream_t stream)
{
    cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (T < 0 || T > kMaxT) return CCA_ERR_INVALID_ARG;
    if (d_rope < 0 || d_rope > c->d || d_rope % 8 != 0) return CCA_ERR_INVALID_ARG;
    const bool any = T > 0;
    if (!ptr_ok(Q, any) || !ptr_ok(K, any) || !ptr_ok(V, any) || !ptr_ok(q_sum, true))
        return CCA_ERR_INVALID_ARG;
    if (any && (T - 1) / c->g >= c->core_cap) return CCA_ERR_CAPACITY;
    const int64_t m = T / c->g;
    cudaError_t e = cudaSuccess;
    if (m > 0)
        e = cca::launch_lca_pool(Q, K, V, c->k_core, c->v_core, c->B, c->Hq, c->Hkv, T, c->d,
                                 c->g, d_rope, c->core_cap, stream);
    if (e == cudaSuccess && any) {
        const int64_t p0 = T > c->tail_cap ? T - c->tail_cap : 0;
        e = cca::launch_tail_fill(K, V, c->k_tail, c->v_tail, c->B, c->Hkv, T, c->d, p0,
                                  c->tail_cap, stream);
    }
    if (e == cudaSuccess)
        e = cca::launch_lca_qsum_fill(Q, q_sum, c->B, c->Hq, c->d, T, m * c->g, stream);
    if (e != cudaSuccess) return from_cuda(e);
    c->len = T;
    return CCA_OK;
}

cca_status cca_lca_cache_append(cca_cache *c, float *q_sum, const void *q_t, const void *k_t,
                                const void *v_t, int d_rope, cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (d_rope < 0 || d_rope > c->d || d_rope % 8 != 0) return CCA_ERR_INVALID_ARG;
    if (!ptr_ok(q_t, true) || !ptr_ok(k_t, true) || !ptr_ok(v_t, true) ||
        !ptr_ok(q_sum, true))
        return CCA_ERR_INVALID_ARG;
    const int64_t t = c->len;
    if (t >= kMaxT || t / c->g >= c->core_cap) return CCA_ERR_CAPACITY;
    const cudaError_t e = cca::launch_lca_append(q_t, k_t, v_t, q_sum, c->k_core, c->v_core,
                                                 c->k_tail, c->v_tail, c->B, c->Hq, c->Hkv,
                                                 c->d, c->g, d_rope, c->core_cap, c->tail_cap,
                                                 t, stream);
    if (e != cudaSuccess) return from_cuda(e);
    c->len = t + 1;
    return CCA_OK;
}

size_t cca_decode_workspace_bytes(const cca_cache *c)
{
    if (cache_status(c) != CCA_OK) return 0;
    return cca::decode_workspace_bytes(c->B, c->Hq, c->Hkv, c->d, c->core_cap, c->tail_cap);
}

cca_status cca_attn_decode(const cca_cache *c, const void *q_t, void *o_t,
                           cca_dtype o_dtype, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    if (c->len < 1) return CCA_ERR_INVALID_ARG;
    if (!ptr_ok(q_t, true) || !ptr_ok(o_t, true) || workspace == nullptr ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CCA_ERR_INVALID_ARG;
    if (workspace_bytes < cca::decode_workspace_bytes(c->B, c->Hq, c->Hkv, c->d, c->core_cap,
                                                      c->tail_cap))
        return CCA_ERR_INVALID_ARG;
    const int64_t t = c->len - 1;
    const int64_t ws = cca::window_start(t, c->g, c->w);
    if (ws / c->g > c->core_cap) return CCA_ERR_CAPACITY;
    return from_cuda(cca::launch_decode(c->k_core, c->v_core, c->k_tail, c->v_tail, q_t,
                                        o_t, o_dtype == CCA_F32, workspace, c->B, c->Hq,
                                        c->Hkv, c->d, c->g, c->w, c->core_cap,
                                        c->tail_cap, t, stream));
}

cca_status cca_decode_step(cca_cache *c, const void *q_t, const void *k_t, const void *v_t,
                           void *o_t, cca_dtype o_dtype, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    if (!ptr_ok(q_t, true) || !ptr_ok(k_t, true) || !ptr_ok(v_t, true) || !ptr_ok(o_t, true) ||
        workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return CCA_ERR_INVALID_ARG;
    if (workspace_bytes < cca::decode_workspace_bytes(c->B, c->Hq, c->Hkv, c->d, c->core_cap,
                                                      c->tail_cap))
        return CCA_ERR_INVALID_ARG;
    const int64_t t = c->len;
    if (t >= kMaxT || t / c->g >= c->core_cap) return CCA_ERR_CAPACITY;
    const size_t out = size_t(c->B) * c->Hq * c->d * (o_dtype == CCA_F32 ? 4 : 2);
    const size_t in_q = size_t(c->B) * c->Hq * c->d * 2, in_kv = size_t(c->B) * c->Hkv * c->d * 2;
    if (overlap(o_t, out, q_t, in_q) || overlap(o_t, out, k_t, in_kv) ||
        overlap(o_t, out, v_t, in_kv) || overlap(o_t, out, workspace, workspace_bytes))
        return CCA_ERR_INVALID_ARG;
    const cudaError_t e = cca::launch_decode_step(
        c->k_core, c->v_core, c->k_tail, c->v_tail, q_t, k_t, v_t, o_t, o_dtype == CCA_F32,
        workspace, c->B, c->Hq, c->Hkv, c->d, c->g, c->w, c->core_cap, c->tail_cap, t, stream);
    if (e != cudaSuccess) return from_cuda(e);
    c->len = t + 1;
    return CCA_OK;
}

cca_status cca_cache_append_rows(const cca_cache *c, long long *lens, const void *q_t,
                                 const void *k_t, const void *v_t, cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (!ptr_ok(q_t, true) || !ptr_ok(k_t, true) || !ptr_ok(v_t, true) ||
        lens == nullptr || (reinterpret_cast<uintptr_t>(lens) & 7u) != 0)
        return CCA_ERR_INVALID_ARG;
    // one CTA per row, one warp per key/value head
    if (c->Hkv > 32 || cca::append_rows_smem_bytes(c->Hq, c->Hkv, c->g) > 200u * 1024u)
        return CCA_ERR_UNSUPPORTED;
    return from_cuda(cca::launch_append_rows(q_t, k_t, v_t, c->k_core, c->v_core, c->k_tail,
                                             c->v_tail, lens, c->B, c->Hq, c->Hkv, c->d,
                                             c->g, c->core_cap, c->tail_cap, stream));
}

cca_status cca_attn_decode_rows(const cca_cache *c, const long long *lens, const void *q_t,
                                void *o_t, cca_dtype o_dtype, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream)
{
    const cca_status s = cache_status(c);
    if (s != CCA_OK) return s;
    if (o_dtype != CCA_BF16 && o_dtype != CCA_F32) return CCA_ERR_INVALID_ARG;
    if (!ptr_ok(q_t, true) || !ptr_ok(o_t, true) || workspace == nullptr ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || lens == nullptr ||
        (reinterpret_cast<uintptr_t>(lens) & 7u) != 0)
        return CCA_ERR_INVALID_ARG;
    if (workspace_bytes < cca::decode_workspace_bytes(c->B, c->Hq, c->Hkv, c->d, c->core_cap,
                                                      c->tail_cap))
        return CCA_ERR_INVALID_ARG;
    return from_cuda(cca::launch_decode_rows(c->k_core, c->v_core, c->k_tail, c->v_tail, q_t,
                                             o_t, o_dtype == CCA_F32, workspace, lens, c->B,
                                             c->Hq, c->Hkv, c->d, c->g, c->w, c->core_cap,
                                             c->tail_cap, stream));
}

cca_status cca_device_status(cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return from_cuda(e);
    unsigned int a = 0, b = 0, c = 0, d = 0, f = 0, h = 0, l = 0;
    if ((e = cca::prefill_status_read_clear(&a)) != cudaSuccess ||
        (e = cca::pool_status_read_clear(&b)) != cudaSuccess ||
        (e = cca::append_status_read_clear(&c)) != cudaSuccess ||
        (e = cca::selftest_status_read_clear(&d)) != cudaSuccess ||
        (e = cca::decode_status_read_clear(&f)) != cudaSuccess ||
        (e = cca::backward_status_read_clear(&h)) != cudaSuccess ||
        (e = cca::lca_status_read_clear(&l)) != cudaSuccess)
        return from_cuda(e);
    const unsigned int st = a | b | c | d | f | h | l;
    if (st & cca::kStatusTimeout) return CCA_ERR_TIMEOUT;
    if (st & cca::kStatusCapacity) return CCA_ERR_CAPACITY;
    if (st & cca::kStatusRange) return CCA_ERR_RANGE;
    return CCA_OK;
}

const char *cca_status_string(cca_status s)
{
    switch (s) {
    case CCA_OK: return "CCA_OK";
    case CCA_ERR_INVALID_ARG: return "CCA_ERR_INVALID_ARG";
    case CCA_ERR_UNSUPPORTED: return "CCA_ERR_UNSUPPORTED";
    case CCA_ERR_CAPACITY: return "CCA_ERR_CAPACITY";
    case CCA_ERR_CUDA: return "CCA_ERR_CUDA";
    case CCA_ERR_TIMEOUT: return "CCA_ERR_TIMEOUT";
    case CCA_ERR_RANGE: return "CCA_ERR_RANGE";
    case CCA_ERR_SCRATCH: return "CCA_ERR_SCRATCH";
    }
    return "CCA_ERR_UNKNOWN";
}

const char *cca_version(void) { return "0.1.0"; }

const char *cca_last_error(void)
{
    return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

}  // extern "C"
