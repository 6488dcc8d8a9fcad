// Warp-level globally-aware pooling of one group (section 全局感知池化 of the
// CCA write-up): the query of the group's last token scores the group's g
// keys, softmax(q . k / sqrt(d)); with grouped-query attention the weights
// are the mean of the r query heads' softmax vectors; the weights pool the
// group's keys and values into one core key and one core value.
//
// One warp handles one group.  Lane l owns dims [l*DPL, (l+1)*DPL) of every
// row (DPL = D / 32), so each row is read by one coalesced warp load.
// Scores are reduced across the warp, kept in the warp's shared-memory
// scratch, soft-maxed in fp32, and the pooled sums accumulate in fp32.  The
// core key and value are stored in fp16 (11 significant bits: the pooled
// rows of heavy keys are large, and bf16 storage would cost the following
// attention up to 2e-2 of absolute error); values beyond the fp16 range are
// clamped and the function returns true.
#pragma once

#include "common.cuh"

namespace cca {

template <int D>
struct RowVec;
template <>
struct RowVec<128> {  // 4 bf16 per lane
    using T = uint2;
    static __device__ __forceinline__ void to_f32(T v, float (&f)[4])
    {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
        f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    }
    static __device__ __forceinline__ T to_f16(const float (&f)[4], bool &over)
    {
        return make_uint2(pack_f16x2(clamp_f16(f[0], over), clamp_f16(f[1], over)),
                          pack_f16x2(clamp_f16(f[2], over), clamp_f16(f[3], over)));
    }
};
template <>
struct RowVec<64> {  // 2 bf16 per lane
    using T = uint32_t;
    static __device__ __forceinline__ void to_f32(T v, float (&f)[2])
    {
        f[0] = bf16_lo(v); f[1] = bf16_hi(v);
    }
    static __device__ __forceinline__ T to_f16(const float (&f)[2], bool &over)
    {
        return pack_f16x2(clamp_f16(f[0], over), clamp_f16(f[1], over));
    }
};

// Pool one group.
//   key_row(i), val_row(i): pointers to row i (0 <= i < g) of the group's
//     keys / values (bf16, D elements each).
//   q_row(k): pointer to the scoring query of the k-th query head (k < r).
//   scratch: r*g + g floats of this warp's shared memory.
//   kc_out, vc_out: destination rows (fp16, D elements).
//   scale_log2 = log2(e) / sqrt(D).
// Returns true (on every lane) if a pooled value was clamped.
template <int D, class KeyRow, class ValRow, class QRow>
__device__ __forceinline__ bool pool_group_warp(KeyRow key_row, ValRow val_row,
                                                QRow q_row, int r, int g,
                                                float scale_log2, float *scratch,
                                                uint16_t *kc_out,
                                                uint16_t *vc_out)
{
    constexpr int DPL = D / 32;
    using V = RowVec<D>;
    using VT = typename V::T;
    const int lane = threadIdx.x & 31;
    float *logit = scratch;           // [r][g] scaled scores (log2 units)
    float *weight = scratch + r * g;  // [g] pooling weights

    // Scores: each key row is loaded once and scored by all r queries.
    for (int i0 = 0; i0 < g; i0 += 8) {
        VT kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + u < g)
                kv[u] = reinterpret_cast<const VT *>(key_row(i0 + u))[lane];
        for (int k = 0; k < r; ++k) {
            float q[DPL];
            V::to_f32(reinterpret_cast<const VT *>(q_row(k))[lane], q);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (i0 + u < g) {
                    float kf[DPL];
                    V::to_f32(kv[u], kf);
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

    // Weights: mean over the r query heads of softmax over the g scores.
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
    }
    __syncwarp();

    // Pooled key and value: weighted sums of the group's rows.
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
                V::to_f32(kv[u], kf);
                V::to_f32(vv[u], vf);
#pragma unroll
                for (int e = 0; e < DPL; ++e) {
                    ak[e] = fmaf(a, kf[e], ak[e]);
                    av[e] = fmaf(a, vf[e], av[e]);
                }
            }
        }
    }
    bool over = false;
    reinterpret_cast<VT *>(kc_out)[lane] = V::to_f16(ak, over);
    reinterpret_cast<VT *>(vc_out)[lane] = V::to_f16(av, over);
    return __any_sync(0xffffffffu, over);
}

// ---------------------------------------------------------------------------
// Register-resident pooling for a compile-time group size G (16 or 32).
//
// The warp is cut into RPW = 32 / (D/8) row slots of D/8 lanes; lane l owns
// dims [8*(l % (D/8)), +8) of rows i with i % RPW == l / (D/8), loaded as
// 16-byte vectors.  All of the group's key rows are requested before any
// arithmetic (then all its value rows, for G = 32 only once the keys are
// pooled), so each warp keeps G * 2 * D bytes in flight.  Scores are reduced
// over the lanes of a row; the pooled sums are reduced over the row slots.
// Same arithmetic as pool_group_warp: fp32 scores, fp32 softmax per query
// head, mean over heads, fp32 weighted sums, fp16 stores.
template <int D, int G, class KeyRow, class ValRow, class QRow>
__device__ __forceinline__ bool pool_group_warp_fast(KeyRow key_row, ValRow val_row,
                                                     QRow q_row, int r,
                                                     float scale_log2, float *scratch,
                                                     uint16_t *kc_out, uint16_t *vc_out)
{
    constexpr int LPR = D / 8;          // lanes per row
    constexpr int RPW = 32 / LPR;       // rows per warp step
    constexpr int NR = G / RPW;         // rows per lane
    const int lane = threadIdx.x & 31;
    const int kl = lane % LPR, slot = lane / LPR;
    float *logit = scratch;             // [r][G]
    float *weight = scratch + r * G;    // [G]

    auto to8 = [](uint4 v, float (&f)[8]) {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    };
    uint4 kv[NR], vv[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n)
        kv[n] = *reinterpret_cast<const uint4 *>(key_row(n * RPW + slot) + kl * 8);
    if (G <= 16) {
#pragma unroll
        for (int n = 0; n < NR; ++n)
            vv[n] = *reinterpret_cast<const uint4 *>(val_row(n * RPW + slot) + kl * 8);
    }
    // scores, all r query heads per key row
    for (int k = 0; k < r; ++k) {
        float q[8];
        to8(*reinterpret_cast<const uint4 *>(q_row(k) + kl * 8), q);
#pragma unroll
        for (int n = 0; n < NR; ++n) {
            float kf[8];
            to8(kv[n], kf);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(q[e], kf[e], s);
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (kl == 0) logit[k * G + n * RPW + slot] = s * scale_log2;
        }
    }
    __syncwarp();
    // weights: mean over the r query heads of softmax over the G scores
    if (lane < G) weight[lane] = 0.f;
    if (G > 32) for (int i = lane + 32; i < G; i += 32) weight[i] = 0.f;
    __syncwarp();
    const float inv_r = 1.0f / static_cast<float>(r);
    for (int k = 0; k < r; ++k) {
        float mx = -INFINITY;
        for (int i = lane; i < G; i += 32) mx = fmaxf(mx, logit[k * G + i]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < G; i += 32) {
            const float e = exp2f(logit[k * G + i] - mx);
            logit[k * G + i] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        const float c = inv_r / sum;
        for (int i = lane; i < G; i += 32) weight[i] += logit[k * G + i] * c;
    }
    __syncwarp();
    // pooled key, then pooled value
    float ak[8], av[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ak[e] = av[e] = 0.f;
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float a = weight[n * RPW + slot];
        float kf[8];
        to8(kv[n], kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) ak[e] = fmaf(a, kf[e], ak[e]);
    }
    if (G > 16) {
#pragma unroll
        for (int n = 0; n < NR; ++n)
            vv[n] = *reinterpret_cast<const uint4 *>(val_row(n * RPW + slot) + kl * 8);
    }
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const float a = weight[n * RPW + slot];
        float vf[8];
        to8(vv[n], vf);
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
        uint4 h;
        h.x = pack_f16x2(clamp_f16(ak[0], over), clamp_f16(ak[1], over));
        h.y = pack_f16x2(clamp_f16(ak[2], over), clamp_f16(ak[3], over));
        h.z = pack_f16x2(clamp_f16(ak[4], over), clamp_f16(ak[5], over));
        h.w = pack_f16x2(clamp_f16(ak[6], over), clamp_f16(ak[7], over));
        *reinterpret_cast<uint4 *>(kc_out + kl * 8) = h;
    } else if (slot == 1) {
        uint4 h;
        h.x = pack_f16x2(clamp_f16(av[0], over), clamp_f16(av[1], over));
        h.y = pack_f16x2(clamp_f16(av[2], over), clamp_f16(av[3], over));
        h.z = pack_f16x2(clamp_f16(av[4], over), clamp_f16(av[5], over));
        h.w = pack_f16x2(clamp_f16(av[6], over), clamp_f16(av[7], over));
        *reinterpret_cast<uint4 *>(vc_out + kl * 8) = h;
    }
    return __any_sync(0xffffffffu, over);
}

}  // namespace cca
