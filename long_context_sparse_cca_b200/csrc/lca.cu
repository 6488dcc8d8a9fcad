// The LCA variant: latent-condensed pooling (page "Latent-Condensed
// Transformer for Efficient Long Context Modeling", section 2 方法论,
// 核心设计思想: 语义凝聚 and 位置锚定), a later method by the authors of CCA.
//
// Per group of g tokens and key/value head: every query head's average query
// over the group's own g query rows scores the group's keys
// (q_bar . k / sqrt(d)); softmax per query head, mean over the r query heads
// of the key/value head (as for CCA's pooling); the content part of the key
// (entries [0, d - d_rope)) and the whole value are pooled with these
// weights, while the positional part (the last d_rope entries, the rotary
// key of latent attention) is copied from the group's highest-weight token,
// the anchor (the first one on a tie).  The condensed rows then serve the
// same fused core + local attention as CCA's (prefill and decode kernels
// are shared).
//
// Kernels: lca_pool_kernel (one warp per group; register-resident path for
// g = 16 and 32), lca_append_kernel (decode: ring write, running sum of the
// open group's queries, condensation of the group the token completes),
// qsum_fill_kernel (the running sums after a prefix).  All HBM- or
// latency-bound; fp32 arithmetic, fp16 core rows with the fp16 range clamp.
#include "internal.h"
#include "pool_warp.cuh"

namespace cca {

__device__ unsigned int g_lca_status;  // kStatusRange: a core value was clamped

namespace {

constexpr int kLcaWarps = 8;  // warps per block (pooling)

// Index of the largest weight[i], i < g, the smallest index on a tie (the
// weights are softmax means, so >= 0).  Every lane gets the result.
__device__ __forceinline__ int warp_argmax_first(const float *weight, int g)
{
    const int lane = threadIdx.x & 31;
    float bw = -1.f;
    int bi = 0x7fffffff;
    for (int i = lane; i < g; i += 32) {
        const float v = weight[i];
        if (v > bw) {
            bw = v;
            bi = i;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ow = __shfl_xor_sync(0xffffffffu, bw, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ow > bw || (ow == bw && oi < bi)) {
            bw = ow;
            bi = oi;
        }
    }
    return bi < g ? bi : 0;  // no valid weight (non-finite inputs): token 0
}

// Softmax of each query head's logits (log2 units, logit[k * g + i]), mean
// over the r heads into weight[0..g).  Warp-cooperative.
__device__ __forceinline__ void head_mean_softmax(float *logit, float *weight, int r, int g)
{
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < g; i += 32) weight[i] = 0.f;
    __syncwarp();
    const float inv_r = 1.0f / static_cast<float>(r);
    for (int k = 0; k < r; ++k) {
        float mx = -INFINITY;
        for (int i = lane; i < g; i += 32) mx = fmaxf(mx, logit[k * g + i]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < g; i += 32) {
            const float e = exp2f(logit[k * g + i] - mx);
            logit[k * g + i] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        const float c = inv_r / sum;
        for (int i = lane; i < g; i += 32) weight[i] += logit[k * g + i] * c;
        __syncwarp();
    }
}

// Condense one group, any g.  Lane l owns entries [l*DPL, (l+1)*DPL) of
// every row (DPL = D / 32).
//   key_row(i), val_row(i): row i < g of the group's keys / values (bf16).
//   qbar(k, q): fills q[0..DPL) with this lane's entries of query head k's
//     average query (fp32).
//   scratch: r*g + g floats of this warp's shared memory.
// d_rope is a multiple of 8, so a lane's entries are all content or all
// positional.  Returns true on every lane if a value was clamped.
template <int D, class KeyRow, class ValRow, class QBar>
__device__ __forceinline__ bool lca_group_warp(KeyRow key_row, ValRow val_row, QBar qbar,
                                               int r, int g, int d_rope, float scale_log2,
                                               float *scratch, uint16_t *kc_out,
                                               uint16_t *vc_out)
{
    constexpr int DPL = D / 32;
    using RV = RowVec<D>;
    using VT = typename RV::T;
    const int lane = threadIdx.x & 31;
    float *logit = scratch;           // [r][g]
    float *weight = scratch + r * g;  // [g]
    for (int k = 0; k < r; ++k) {
        float q[DPL];
        qbar(k, q);
        for (int i0 = 0; i0 < g; i0 += 8) {
            VT kv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u < g) kv[u] = reinterpret_cast<const VT *>(key_row(i0 + u))[lane];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (i0 + u < g) {
                    float kf[DPL];
                    RV::to_f32(kv[u], kf);
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) s = fmaf(q[e], kf[e], s);
                    s = warp_sum(s);
                    if (lane == 0) logit[k * g + i0 + u] = s * scale_log2;
                }
            }
        }
    }
    __syncwarp();
    head_mean_softmax(logit, weight, r, g);
    const int anchor = warp_argmax_first(weight, g);

    float ak[DPL], av[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) ak[e] = av[e] = 0.f;
    for (int i0 = 0; i0 < g; i0 += 8) {
        VT kv[8], vv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (i0 + u < g) {
                kv[u] = reinterpret_cast<const VT *>(key_row(i0 + u))[lane];
                vv[u] = reinterpret_cast<const VT *>(val_row(i0 + u))[lane];
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (i0 + u < g) {
                const float a = weight[i0 + u];
                float kf[DPL], vf[DPL];
                RV::to_f32(kv[u], kf);
                RV::to_f32(vv[u], vf);
#pragma unroll
                for (int e = 0; e < DPL; ++e) {
                    ak[e] = fmaf(a, kf[e], ak[e]);
                    av[e] = fmaf(a, vf[e], av[e]);
                }
            }
        }
    }
    if (lane * DPL >= D - d_rope)  // positional entries: the anchor's own
        RV::to_f32(reinterpret_cast<const VT *>(key_row(anchor))[lane], ak);
    bool over = false;
    reinterpret_cast<VT *>(kc_out)[lane] = RV::to_f16(ak, over);
    reinterpret_cast<VT *>(vc_out)[lane] = RV::to_f16(av, over);
    return __any_sync(0xffffffffu, over);
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float (&f)[8])
{
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 f32x8_to_f16(const float (&f)[8], bool &over)
{
    uint4 h;
    h.x = pack_f16x2(clamp_f16(f[0], over), clamp_f16(f[1], over));
    h.y = pack_f16x2(clamp_f16(f[2], over), clamp_f16(f[3], over));
    h.z = pack_f16x2(clamp_f16(f[4], over), clamp_f16(f[5], over));
    h.w = pack_f16x2(clamp_f16(f[6], over), clamp_f16(f[7], over));
    return h;
}

// Condense one group of compile-time size G (16 or 32) with the group's
// rows in registers.  The warp is cut into RPW = 32 / (D/8) row slots of
// D/8 lanes; lane l owns entries [8*(l % (D/8)), +8) of rows i with
// i % RPW == l / (D/8), as 16-byte loads.  The average query of a head is
// summed over the lane's rows, then over the row slots.  Same arithmetic
// as lca_group_warp, in another summation order.
//   q_row(k, i): row i of the group's queries of query head k.
template <int D, int G, class KeyRow, class ValRow, class QRow>
__device__ __forceinline__ bool lca_group_warp_fast(KeyRow key_row, ValRow val_row, QRow q_row,
                                                    int r, int d_rope, float scale_log2,
                                                    float *scratch, uint16_t *kc_out,
                                                    uint16_t *vc_out)
{
    constexpr int LPR = D / 8;     // lanes per row
    constexpr int RPW = 32 / LPR;  // rows per warp step
    constexpr int NR = G / RPW;    // rows per lane
    const int lane = threadIdx.x & 31;
    const int kl = lane % LPR, slot = lane / LPR;
    float *logit = scratch;           // [r][G]
    float *weight = scratch + r * G;  // [G]
    constexpr float inv_g = 1.0f / static_cast<float>(G);

    uint4 kv[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n)
        kv[n] = *reinterpret_cast<const uint4 *>(key_row(n * RPW + slot) + kl * 8);
    for (int k = 0; k < r; ++k) {
        uint4 qv[NR];
#pragma unroll
        for (int n = 0; n < NR; ++n)
            qv[n] = *reinterpret_cast<const uint4 *>(q_row(k, n * RPW + slot) + kl * 8);
        float q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = 0.f;
#pragma unroll
        for (int n = 0; n < NR; ++n) {
            float f[8];
            bf16x8_to_f32(qv[n], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] += f[e];
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] += __shfl_xor_sync(0xffffffffu, q[e], o);
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] *= inv_g;
#pragma unroll
        for (int n = 0; n < NR; ++n) {
            float kf[8];
            bf16x8_to_f32(kv[n], kf);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(q[e], kf[e], s);
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (kl == 0) logit[k * G + n * RPW + slot] = s * scale_log2;
        }
    }
    __syncwarp();
    head_mean_softmax(logit, weight, r, G);
    const int anchor = warp_argmax_first(weight, G);

    float ak[8], av[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ak[e] = av[e] = 0.f;
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float a = weight[n * RPW + slot];
        float kf[8];
        bf16x8_to_f32(kv[n], kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) ak[e] = fmaf(a, kf[e], ak[e]);
    }
    uint4 vv[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n)
        vv[n] = *reinterpret_cast<const uint4 *>(val_row(n * RPW + slot) + kl * 8);
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float a = weight[n * RPW + slot];
        float vf[8];
        bf16x8_to_f32(vv[n], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) av[e] = fmaf(a, vf[e], av[e]);
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], o);
            av[e] += __shfl_xor_sync(0xffffffffu, av[e], o);
        }
    bool over = false;
    if (slot == 0) {
        if (kl * 8 >= D - d_rope)  // positional entries: the anchor's own
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(key_row(anchor) + kl * 8), ak);
        *reinterpret_cast<uint4 *>(kc_out + kl * 8) = f32x8_to_f16(ak, over);
    } else if (slot == 1) {
        *reinterpret_cast<uint4 *>(vc_out + kl * 8) = f32x8_to_f16(av, over);
    }
    return __any_sync(0xffffffffu, over);
}

// G > 0: register-resident path for that group size; G == 0: any g.
template <int D, int G>
__global__ void __launch_bounds__(kLcaWarps * 32, 2)
    lca_pool_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                    const uint16_t *__restrict__ V, uint16_t *__restrict__ Kc,
                    uint16_t *__restrict__ Vc, int Hq, int Hkv, int64_t T, int g, int d_rope,
                    int64_t m, int64_t out_rows, int64_t n_groups, float scale_log2)
{
    extern __shared__ float lca_smem[];
    const int warp = threadIdx.x >> 5;
    const int r = Hq / Hkv;
    float *scratch = lca_smem + warp * (r * g + g);
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * kLcaWarps + warp; gid < n_groups;
         gid += static_cast<int64_t>(gridDim.x) * kLcaWarps) {
        const int64_t bh = gid / m, j = gid - bh * m;
        const int64_t b = bh / Hkv, h = bh - b * Hkv;
        const int64_t first = j * g;
        const uint16_t *Kg = K + (bh * T + first) * D;
        const uint16_t *Vg = V + (bh * T + first) * D;
        const uint16_t *Qg = Q + ((b * Hq + h * r) * T + first) * D;
        auto krow = [&](int i) { return Kg + static_cast<int64_t>(i) * D; };
        auto vrow = [&](int i) { return Vg + static_cast<int64_t>(i) * D; };
        uint16_t *kc = Kc + (bh * out_rows + j) * D;
        uint16_t *vc = Vc + (bh * out_rows + j) * D;
        bool over;
        if constexpr (G > 0) {
            auto qrow = [&](int k, int i) {
                return Qg + (static_cast<int64_t>(k) * T + i) * D;
            };
            over = lca_group_warp_fast<D, G>(krow, vrow, qrow, r, d_rope, scale_log2, scratch,
                                             kc, vc);
        } else {
            constexpr int DPL = D / 32;
            const int lane = threadIdx.x & 31;
            const float inv_g = 1.0f / static_cast<float>(g);
            auto qbar = [&](int k, float (&q)[DPL]) {
                using VT = typename RowVec<D>::T;
                const uint16_t *qh = Qg + static_cast<int64_t>(k) * T * D;
#pragma unroll
                for (int e = 0; e < DPL; ++e) q[e] = 0.f;
                for (int i = 0; i < g; ++i) {
                    float f[DPL];
                    RowVec<D>::to_f32(reinterpret_cast<const VT *>(qh + static_cast<int64_t>(i) * D)[lane], f);
#pragma unroll
                    for (int e = 0; e < DPL; ++e) q[e] += f[e];
                }
#pragma unroll
                for (int e = 0; e < DPL; ++e) q[e] *= inv_g;
            };
            over = lca_group_warp<D>(krow, vrow, qbar, r, g, d_rope, scale_log2, scratch, kc,
                                     vc);
        }
        if (over && (threadIdx.x & 31) == 0) atomicOr(&g_lca_status, kStatusRange);
    }
}

constexpr int kLcaAppendWarps = 4;

// Decode: append token t to pair bh = b * Hkv + h.  Ring slot t % tail_cap
// takes k_t, v_t.  q_sum [B, Hq, D] (fp32) holds, per query head, the sum
// of the queries of the group's tokens appended so far; if t completes
// group j = t / g, the group is condensed with average queries
// (q_sum + q_t) / g into core slot j and the sums restart at zero,
// otherwise q_t is added to them.  One warp per pair; the warp owns its r
// query heads' sums.
template <int D>
__global__ void __launch_bounds__(kLcaAppendWarps * 32)
    lca_append_kernel(const uint16_t *__restrict__ q_t, const uint16_t *__restrict__ k_t,
                      const uint16_t *__restrict__ v_t, float *__restrict__ q_sum,
                      uint16_t *__restrict__ k_core, uint16_t *__restrict__ v_core,
                      uint16_t *__restrict__ k_tail, uint16_t *__restrict__ v_tail, int B,
                      int Hq, int Hkv, int g, int d_rope, int64_t core_cap, int64_t tail_cap,
                      int64_t t, float scale_log2)
{
    extern __shared__ float lca_append_smem[];
    constexpr int DPL = D / 32;
    using RV = RowVec<D>;
    using VT = typename RV::T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = static_cast<int64_t>(blockIdx.x) * kLcaAppendWarps + warp;
    if (bh >= static_cast<int64_t>(B) * Hkv) return;
    const int r = Hq / Hkv;
    const int64_t b = bh / Hkv, h = bh - b * Hkv;
    const int64_t slot = t % tail_cap;
    reinterpret_cast<VT *>(k_tail + (bh * tail_cap + slot) * D)[lane] =
        reinterpret_cast<const VT *>(k_t + bh * D)[lane];
    reinterpret_cast<VT *>(v_tail + (bh * tail_cap + slot) * D)[lane] =
        reinterpret_cast<const VT *>(v_t + bh * D)[lane];
    auto qs = [&](int k) { return q_sum + ((b * Hq + h * r + k) * D + lane * DPL); };
    auto qin = [&](int k) {
        return reinterpret_cast<const VT *>(q_t + (b * Hq + h * r + k) * D)[lane];
    };
    if ((t + 1) % g != 0) {
        for (int k = 0; k < r; ++k) {
            float f[DPL];
            RV::to_f32(qin(k), f);
            float *s = qs(k);
#pragma unroll
            for (int e = 0; e < DPL; ++e) s[e] += f[e];
        }
        return;
    }
    const int64_t first = t - g + 1, j = t / g;
    const uint16_t *kt_base = k_tail + bh * tail_cap * D;
    const uint16_t *vt_base = v_tail + bh * tail_cap * D;
    const float inv_g = 1.0f / static_cast<float>(g);
    const bool over = lca_group_warp<D>(
        [&](int i) {
            return i == g - 1 ? k_t + bh * D : kt_base + ((first + i) % tail_cap) * D;
        },
        [&](int i) {
            return i == g - 1 ? v_t + bh * D : vt_base + ((first + i) % tail_cap) * D;
        },
        [&](int k, float (&q)[DPL]) {
            float f[DPL];
            RV::to_f32(qin(k), f);
            const float *s = qs(k);
#pragma unroll
            for (int e = 0; e < DPL; ++e) q[e] = (s[e] + f[e]) * inv_g;
        },
        r, g, d_rope, scale_log2, lca_append_smem + warp * (r * g + g),
        k_core + (bh * core_cap + j) * D, v_core + (bh * core_cap + j) * D);
    for (int k = 0; k < r; ++k) {
        float *s = qs(k);
#pragma unroll
        for (int e = 0; e < DPL; ++e) s[e] = 0.f;
    }
    if (over && lane == 0) atomicOr(&g_lca_status, kStatusRange);
}

// q_sum[b, hq, :] = sum of Q[b, hq, p, :] over p in [p0, T) (the open
// group after a prefix of T tokens; zero when p0 == T).  One thread per
// (b, hq, entry).
__global__ void qsum_fill_kernel(const uint16_t *__restrict__ Q, float *__restrict__ q_sum,
                                 int64_t BH, int d, int64_t T, int64_t p0)
{
    const int64_t n = BH * d;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t bh = i / d, c = i - bh * d;
        float s = 0.f;
        for (int64_t p = p0; p < T; ++p) {
            const uint32_t bits = static_cast<uint32_t>(Q[(bh * T + p) * d + c]) << 16;
            s += __uint_as_float(bits);
        }
        q_sum[i] = s;
    }
}

int grid_for(int64_t want, int per_sm)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = static_cast<int64_t>(per_sm) * sms;
    return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_lca_pool(const void *Q, const void *K, const void *V, void *Kc, void *Vc,
                            int B, int Hq, int Hkv, int64_t T, int d, int g, int d_rope,
                            int64_t out_rows, cudaStream_t s)
{
    const int64_t m = T / g;
    const int64_t n_groups = static_cast<int64_t>(B) * Hkv * m;
    if (n_groups == 0) return cudaSuccess;
    const int r = Hq / Hkv;
    const size_t smem = sizeof(float) * kLcaWarps * (r * g + g);
    const int blocks = grid_for((n_groups + kLcaWarps - 1) / kLcaWarps, 64);
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    const auto *q = static_cast<const uint16_t *>(Q);
    const auto *k = static_cast<const uint16_t *>(K);
    const auto *v = static_cast<const uint16_t *>(V);
    auto *kc = static_cast<uint16_t *>(Kc);
    auto *vc = static_cast<uint16_t *>(Vc);
    auto go = [&](auto kern) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        kern<<<blocks, kLcaWarps * 32, smem, s>>>(q, k, v, kc, vc, Hq, Hkv, T, g, d_rope, m,
                                                   out_rows, n_groups, scale_log2);
    };
    if (d == 128) {
        if (g == 16)
            go(lca_pool_kernel<128, 16>);
        else if (g == 32)
            go(lca_pool_kernel<128, 32>);
        else
            go(lca_pool_kernel<128, 0>);
    } else {
        if (g == 16)
            go(lca_pool_kernel<64, 16>);
        else if (g == 32)
            go(lca_pool_kernel<64, 32>);
        else
            go(lca_pool_kernel<64, 0>);
    }
    return cudaGetLastError();
}

cudaError_t launch_lca_append(const void *q_t, const void *k_t, const void *v_t, float *q_sum,
                              void *k_core, void *v_core, void *k_tail, void *v_tail, int B,
                              int Hq, int Hkv, int d, int g, int d_rope, int64_t core_cap,
                              int64_t tail_cap, int64_t t, cudaStream_t s)
{
    const int64_t pairs = static_cast<int64_t>(B) * Hkv;
    const int blocks = static_cast<int>((pairs + kLcaAppendWarps - 1) / kLcaAppendWarps);
    const int r = Hq / Hkv;
    const size_t smem = sizeof(float) * kLcaAppendWarps * (r * g + g);
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    auto go = [&](auto kern) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        kern<<<blocks, kLcaAppendWarps * 32, smem, s>>>(
            static_cast<const uint16_t *>(q_t), static_cast<const uint16_t *>(k_t),
            static_cast<const uint16_t *>(v_t), q_sum, static_cast<uint16_t *>(k_core),
            static_cast<uint16_t *>(v_core), static_cast<uint16_t *>(k_tail),
            static_cast<uint16_t *>(v_tail), B, Hq, Hkv, g, d_rope, core_cap, tail_cap, t,
            scale_log2);
    };
    if (d == 128)
        go(lca_append_kernel<128>);
    else
        go(lca_append_kernel<64>);
    return cudaGetLastError();
}

cudaError_t launch_lca_qsum_fill(const void *Q, float *q_sum, int B, int Hq, int d, int64_t T,
                                 int64_t p0, cudaStream_t s)
{
    const int64_t n = static_cast<int64_t>(B) * Hq * d;
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = grid_for((n + threads - 1) / threads, 8);
    qsum_fill_kernel<<<blocks, threads, 0, s>>>(static_cast<const uint16_t *>(Q), q_sum,
                                                 static_cast<int64_t>(B) * Hq, d, T, p0);
    return cudaGetLastError();
}

cudaError_t lca_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_lca_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_lca_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
