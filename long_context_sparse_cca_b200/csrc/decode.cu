// cca_attn_decode: attention of the newest token over the decode cache
// (core keys/values of the groups before its window, raw ring tokens of the
// window; one softmax, sections 局部保留模块 and 全局-局部模块可微融合 of the
// CCA write-up).
//
// Core rows are fp16, ring rows bf16; scores and sums are fp32.
//
// HBM-bound split-K GEMV: the keys of one (batch, key/value head) are cut
// into chunks; one CTA streams one chunk's K and V rows once for all r query
// heads of that key/value head, producing a partial (max, sum, unnormalised
// output) per query head.  The last CTA of a (batch, key/value head) to
// finish, found by an atomic ticket, rescales and adds the partials and
// writes the output: one launch, no separate merge kernel.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace cca {

__device__ unsigned int g_decode_status;  // kStatusCapacity

namespace {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeChunk = 256;  // keys per split

template <int D>
struct DecodeShape {
    static constexpr int KL = D / 8;              // lanes per key row (16 B each)
    static constexpr int KPW = 32 / KL;           // keys per warp step
    static constexpr int NG = (kDecodeThreads / 32) * KPW;  // key groups per CTA
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8])
{
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ void f16x8_to_f32(const uint4 v, float (&f)[8])
{
    f[0] = f16_lo(v.x); f[1] = f16_hi(v.x);
    f[2] = f16_lo(v.y); f[3] = f16_hi(v.y);
    f[4] = f16_lo(v.z); f[5] = f16_hi(v.z);
    f[6] = f16_lo(v.w); f[7] = f16_hi(v.w);
}

// Eight elements of a cache row: core rows are fp16, ring rows bf16.
__device__ __forceinline__ void row8_to_f32(const uint4 v, bool core, float (&f)[8])
{
    if (core)
        f16x8_to_f32(v, f);
    else
        bf16x8_to_f32(v, f);
}

struct CacheView {
    const uint16_t *k_core, *v_core, *k_tail, *v_tail;
    int64_t core_cap, tail_cap, ws, n_core;
    int64_t ws_slot;  // ws % tail_cap: ring slot of the window's first token
    // Row of key k (0 <= k < n_keys) of pair bh: core slot k, or the ring
    // slot of raw token ws + (k - n_core).  The window holds at most
    // tail_cap tokens, so one wrap-around step replaces a modulo.
    __device__ __forceinline__ int64_t row(int64_t bh, int64_t k, bool &core) const
    {
        core = k < n_core;
        if (core) return bh * core_cap + k;
        int64_t slot = ws_slot + (k - n_core);
        if (slot >= tail_cap) slot -= tail_cap;
        return bh * tail_cap + slot;
    }
};

// The token a fused decode step appends (cca_decode_step).  Its key/value
// rows are read from these inputs, not from the ring slot this launch
// writes; the CTA with a pair's last split writes that ring slot and, when
// the token completes a group, pools the group into its core slot.  No key
// any CTA of the launch reads is written by it: the ring slot of token t
// held token t - tail_cap, before the window, and core slot t / g is not in
// token t's core set.
struct StepArgs {
    const uint16_t *k_t, *v_t;                    // [B, Hkv, D] rows of token t
    uint16_t *k_core, *v_core, *k_tail, *v_tail;  // the cache, written
    int g;
    int64_t t;
};

// The append of a fused step for pair bh, by the whole CTA with the
// decode kernel's own lane layout (lane kl of a row slot kg holds 16 bytes
// of a row), so that the kernel's register budget does not grow: the ring
// slot of token t, and when t completes group j = t / g, the pooling of
// that group (section 全局感知池化: the scores of the group's keys against
// the queries of its last token, token t, soft-maxed per query head and
// averaged over the r heads, weight the group's keys and values; the same
// arithmetic as the separate append: fp32 scores, exp2f, fp32 sums, fp16
// rows).  Scratch: lg (r g + g floats) and red (NG D floats).
template <int D, int R>
__device__ __forceinline__ void step_append(const StepArgs &st, const uint16_t *q_t,
                                            int64_t b, int64_t h, int Hq,
                                            int64_t bh, int r, int64_t tail_cap,
                                            int64_t core_cap, float scale_log2, float *lg,
                                            float *red)
{
    using S = DecodeShape<D>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kl = lane % S::KL, kg = warp * S::KPW + lane / S::KL;
    const int64_t slot = bh * tail_cap + st.t % tail_cap;
    for (int c = tid; c < D / 8; c += kDecodeThreads) {
        reinterpret_cast<uint4 *>(st.k_tail + slot * D)[c] =
            reinterpret_cast<const uint4 *>(st.k_t + bh * D)[c];
        reinterpret_cast<uint4 *>(st.v_tail + slot * D)[c] =
            reinterpret_cast<const uint4 *>(st.v_t + bh * D)[c];
    }
    const int g = st.g;
    if ((st.t + 1) % g != 0) return;
    const int64_t j = st.t / g;
    const int first_slot = static_cast<int>((st.t - g + 1) % tail_cap);
    const int cap = static_cast<int>(tail_cap);
    // row i of the group: the ring slot of token t - g + 1 + i (g <= tail_cap:
    // one wrap-around step), or for the last one (token t) the input row
    auto grow = [&](const uint16_t *ring, const uint16_t *in, int i) {
        int slot = first_slot + i;
        if (slot >= cap) slot -= cap;
        return i == g - 1 ? in + bh * D : ring + (bh * tail_cap + slot) * D;
    };
    float *logit = lg, *weight = lg + r * g;
    // the scoring queries: token t's own (it is the group's last token)
    float q[R][8];
#pragma unroll
    for (int k = 0; k < R; ++k)
        if (k < r)
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(q_t + (b * Hq + h * r + k) * D + kl * 8),
                          q[k]);
    // scores (loop bound uniform per warp: the shuffles need every lane)
    for (int base = 0; base < g; base += S::NG) {
        const int i = base + kg;
        float kf[8];
        if (i < g)
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(grow(st.k_tail, st.k_t, i) + kl * 8), kf);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) kf[e] = 0.f;
#pragma unroll
        for (int k = 0; k < R; ++k) {
            if (k < r) {
                float sc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) sc = fmaf(q[k][e], kf[e], sc);
#pragma unroll
                for (int o = 1; o < S::KL; o <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
                if (kl == 0 && i < g) logit[k * g + i] = sc * scale_log2;
            }
        }
    }
    __syncthreads();
    // per query head: softmax over the g scores (numerators left in logit)
    for (int k = warp; k < r; k += kDecodeThreads / 32) {
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
        if (lane == 0) red[k] = (1.0f / static_cast<float>(r)) / sum;
    }
    __syncthreads();
    for (int i = tid; i < g; i += kDecodeThreads) {
        float wi = 0.f;
        for (int k = 0; k < r; ++k) wi += logit[k * g + i] * red[k];
        weight[i] = wi;
    }
    __syncthreads();
    // pooled key, then pooled value: per-slot partial sums, then a sum over
    // the row slots through shared memory
    bool over = false;
    for (int which = 0; which < 2; ++which) {
        const uint16_t *ring = which ? st.v_tail : st.k_tail;
        const uint16_t *in = which ? st.v_t : st.k_t;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int i = kg; i < g; i += S::NG) {
            float f[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(grow(ring, in, i) + kl * 8), f);
            const float wi = weight[i];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wi, f[e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[kg * D + kl * 8 + e] = acc[e];
        __syncthreads();
        uint16_t *out = (which ? st.v_core : st.k_core) + (bh * core_cap + j) * D;
        for (int c = tid; c < D; c += kDecodeThreads) {
            float sum = 0.f;
            for (int s = 0; s < S::NG; ++s) sum += red[s * D + c];
            out[c] = __half_as_ushort(__float2half_rn(clamp_f16(sum, over)));
        }
        __syncthreads();
    }
    if (__syncthreads_or(over) && tid == 0) atomicOr(&g_decode_status, kStatusRange);
}

template <int D, int R, bool STEP>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(CacheView cv, StepArgs st, const uint16_t *__restrict__ q_t,
                        float *__restrict__ part_o, float2 *__restrict__ part_ml,
                        unsigned int *__restrict__ tickets, void *__restrict__ o_t,
                        int out_f32, int Hq, int Hkv, int64_t n_keys, int chunk,
                        int nsplit, float scale_log2, const long long *__restrict__ lens,
                        int g, int w, int64_t core_cap, int stride)
{
    using S = DecodeShape<D>;
    extern __shared__ float dsm[];
    const int r = Hq / Hkv;
    // [R][chunk] scores (a fused step's pooling also uses it: (r + 1) g)
    const int lg_floats = STEP ? max(R * chunk, (r + 1) * st.g) : R * chunk;
    float *lg = dsm;
    float *red = dsm + lg_floats;                  // [NG][R][D]
    float *stat = red + S::NG * R * D;             // [R][2]
    const int split = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / Hkv, h = bh - b * Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kl = lane % S::KL, kg = warp * S::KPW + lane / S::KL;
    // Uniform lengths: the host planned the split.  Per-row lengths (lens
    // in device memory): this CTA plans its own row; the grid covers the
    // cache's capacity and CTAs past the row's keys leave at once.
    CacheView cvb = cv;
    if (lens != nullptr) {
        const int64_t tb = lens[b] - 1;
        const int64_t wsb = tb >= 0 ? window_start(tb, g, w) : 0;
        if (tb < 0 || wsb / g > core_cap) {
            // an empty row has zero output; a row past the cache is reported
            if (split == 0) {
                if (tb >= 0 && tid == 0) atomicOr(&g_decode_status, kStatusCapacity);
                for (int idx = tid; idx < r * D; idx += kDecodeThreads) {
                    const int64_t orow = b * Hq + h * r + idx / D;
                    if (out_f32)
                        static_cast<float *>(o_t)[orow * D + idx % D] = 0.f;
                    else
                        static_cast<uint16_t *>(o_t)[orow * D + idx % D] = 0;
                }
            }
            return;
        }
        cvb.ws = wsb;
        cvb.ws_slot = wsb % cv.tail_cap;
        cvb.n_core = wsb / g;
        n_keys = cvb.n_core + (tb - wsb + 1);
        nsplit = static_cast<int>((n_keys + chunk - 1) / chunk);
        if (split >= nsplit) return;
    } else {
        stride = nsplit;
    }
    const int64_t c0 = static_cast<int64_t>(split) * chunk;
    const int64_t c1 = c0 + chunk < n_keys ? c0 + chunk : n_keys;
    const int nk = static_cast<int>(c1 - c0);

    float q[R][8];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        if (k < r) {
            const uint4 v = *reinterpret_cast<const uint4 *>(
                q_t + (b * Hq + h * r + k) * D + kl * 8);
            bf16x8_to_f32(v, q[k]);
        }
    }

    // The keys streamed from the cache: all of the chunk, except (fused
    // step, last split) the appended token, whose rows come from the inputs
    // and are added after each loop, outside the hot path.
    const bool new_key = STEP && split == nsplit - 1;
    const int nkc = new_key ? nk - 1 : nk;

    // Scores of this chunk's keys, all query heads at once.  The loop bound
    // is the same for every lane (the shuffles below need the whole warp);
    // each lane's key i = base + kg + u * NG is guarded instead.
    for (int base = 0; base < nkc; base += 4 * S::NG) {
        const int i0 = base + kg;
        uint4 kv[4];
        bool kcore[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            kv[u] = make_uint4(0u, 0u, 0u, 0u);
            kcore[u] = false;
            if (i < nkc) {
                const int64_t row = cvb.row(bh, c0 + i, kcore[u]);
                const uint16_t *src = kcore[u] ? cv.k_core : cv.k_tail;
                kv[u] = ldg_stream(src + row * D + kl * 8);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            float kf[8];
            row8_to_f32(kv[u], kcore[u], kf);
#pragma unroll
            for (int k = 0; k < R; ++k) {
                if (k < r) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) s = fmaf(q[k][e], kf[e], s);
#pragma unroll
                    for (int o = 1; o < S::KL; o <<= 1)
                        s += __shfl_xor_sync(0xffffffffu, s, o);
                    if (kl == 0 && i < nkc) lg[k * chunk + i] = s * scale_log2;
                }
            }
        }
    }
    if (new_key && warp == 0) {
        // the appended token's scores (the upper half-warp repeats them)
        float kf[8];
        bf16x8_to_f32(ldg_stream(st.k_t + bh * D + kl * 8), kf);
#pragma unroll
        for (int k = 0; k < R; ++k) {
            if (k < r) {
                float sc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) sc = fmaf(q[k][e], kf[e], sc);
#pragma unroll
                for (int o = 1; o < S::KL; o <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
                if (lane == 0) lg[k * chunk + nk - 1] = sc * scale_log2;
            }
        }
    }
    __syncthreads();

    // Per query head: chunk maximum, exponentials, sum.
    for (int k = warp; k < r; k += kDecodeThreads / 32) {
        float mx = -INFINITY;
        for (int i = lane; i < nk; i += 32) mx = fmaxf(mx, lg[k * chunk + i]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < nk; i += 32) {
            const float e = fast_exp2(lg[k * chunk + i] - mx);
            lg[k * chunk + i] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        if (lane == 0) {
            stat[2 * k] = mx;
            stat[2 * k + 1] = sum;
        }
    }
    __syncthreads();

    // Weighted sum of the chunk's value rows.
    float acc[R][8];
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
    for (int base = 0; base < nkc; base += 4 * S::NG) {
        const int i0 = base + kg;
        uint4 vv[4];
        bool vcore[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            vv[u] = make_uint4(0u, 0u, 0u, 0u);
            vcore[u] = false;
            if (i < nkc) {
                const int64_t row = cvb.row(bh, c0 + i, vcore[u]);
                const uint16_t *src = vcore[u] ? cv.v_core : cv.v_tail;
                vv[u] = ldg_stream(src + row * D + kl * 8);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            if (i < nkc) {
                float vf[8];
                row8_to_f32(vv[u], vcore[u], vf);
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    if (k < r) {
                        const float p = lg[k * chunk + i];
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(p, vf[e], acc[k][e]);
                    }
                }
            }
        }
    }
    if (new_key && kg == 0) {
        // the appended token's value row, into row slot 0's sums
        float vf[8];
        bf16x8_to_f32(ldg_stream(st.v_t + bh * D + kl * 8), vf);
#pragma unroll
        for (int k = 0; k < R; ++k) {
            if (k < r) {
                const float p = lg[k * chunk + nk - 1];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(p, vf[e], acc[k][e]);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < R; ++k)
        if (k < r)
#pragma unroll
            for (int e = 0; e < 8; ++e) red[(kg * R + k) * D + kl * 8 + e] = acc[k][e];
    __syncthreads();
    for (int idx = tid; idx < r * D; idx += kDecodeThreads) {
        const int k = idx / D, c = idx - k * D;
        float s = 0.f;
#pragma unroll 4
        for (int gi = 0; gi < S::NG; ++gi) s += red[(gi * R + k) * D + c];
        const int64_t qrow = (b * Hq + h * r + k) * stride + split;
        part_o[qrow * D + c] = s;
        if (c == 0) part_ml[qrow] = make_float2(stat[2 * k], stat[2 * k + 1]);
    }

    if (STEP && split == nsplit - 1) {
        // the append (ring slot of token t, pooling of the group it
        // completes), after this CTA's own keys, so that none of its state
        // is live in the loops above; nothing this launch reads is written
        // here.  Scratch: the score and partial-sum buffers, free now (the
        // merge below uses them again only after the barrier).
        __syncthreads();
        step_append<D, R>(st, q_t, b, h, Hq, bh, r, cv.tail_cap, cv.core_cap, scale_log2, lg,
                          red);
    }
    // Ticket: the CTA that takes the last one merges.  The fence makes this
    // CTA's partials visible device-wide before its ticket is counted.
    __threadfence();
    __syncthreads();
    __shared__ unsigned int last;
    if (tid == 0) last = atomicAdd(&tickets[bh], 1u) == static_cast<unsigned int>(nsplit - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();

    // Merge, per query head k: M = max_s m_s, L = sum_s 2^(m_s - M) l_s,
    // o = sum_s 2^(m_s - M) o_s / L.  Partials are read from L2 (__ldcg):
    // other CTAs wrote them.  The weights 2^(m_s - M) go to shared memory
    // (the score buffer, free now) when they fit; every thread then keeps
    // several independent 16-byte loads of partial outputs in flight.
    const bool wfit = nsplit <= chunk;
    for (int k = warp; k < r; k += kDecodeThreads / 32) {
        const float2 *ml = part_ml + (b * Hq + h * r + k) * stride;
        float mx = -INFINITY;
        for (int sp = lane; sp < nsplit; sp += 32) mx = fmaxf(mx, __ldcg(&ml[sp].x));
        mx = warp_max(mx);
        float l = 0.f;
        for (int sp = lane; sp < nsplit; sp += 32) {
            const float2 v = __ldcg(&ml[sp]);
            const float wgt = fast_exp2(v.x - mx);
            if (wfit) lg[k * chunk + sp] = wgt;
            l = fmaf(wgt, v.y, l);
        }
        l = warp_sum(l);
        if (lane == 0) {
            stat[2 * k] = mx;
            stat[2 * k + 1] = 1.0f / l;
        }
    }
    __syncthreads();
    constexpr int C4 = D / 4;                    // float4 columns of a row
    constexpr int SG = kDecodeThreads / C4;      // splits taken at once
    float4 *red4 = reinterpret_cast<float4 *>(red);  // [SG][C4]
    const int c4 = tid % C4, g0 = tid / C4;
    for (int k = 0; k < r; ++k) {
        const int64_t orow = b * Hq + h * r + k;
        const float2 *ml = part_ml + orow * stride;
        const float4 *po4 = reinterpret_cast<const float4 *>(part_o + orow * stride * D) + c4;
        const float mx = stat[2 * k];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int sp = g0; sp < nsplit; sp += SG) {
            const float wgt = wfit ? lg[k * chunk + sp] : fast_exp2(__ldcg(&ml[sp].x) - mx);
            const float4 v = __ldcg(po4 + static_cast<int64_t>(sp) * C4);
            acc.x = fmaf(wgt, v.x, acc.x);
            acc.y = fmaf(wgt, v.y, acc.y);
            acc.z = fmaf(wgt, v.z, acc.z);
            acc.w = fmaf(wgt, v.w, acc.w);
        }
        red4[g0 * C4 + c4] = acc;
        __syncthreads();
        if (tid < C4) {
            float4 o = red4[tid];
#pragma unroll
            for (int gi = 1; gi < SG; ++gi) {
                const float4 v = red4[gi * C4 + tid];
                o.x += v.x;
                o.y += v.y;
                o.z += v.z;
                o.w += v.w;
            }
            const float inv = stat[2 * k + 1];
            if (out_f32) {
                reinterpret_cast<float4 *>(static_cast<float *>(o_t) + orow * D)[tid] =
                    make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
            } else {
                reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o_t) + orow * D)[tid] =
                    make_uint2(pack_bf16x2(o.x * inv, o.y * inv),
                               pack_bf16x2(o.z * inv, o.w * inv));
            }
        }
        __syncthreads();
    }
    // Every CTA of this pair has taken its ticket: leave the counter at zero
    // for the next call (a fused step relies on it; the other calls also
    // clear it first).
    if (tid == 0) tickets[bh] = 0u;
}

template <int D, int R, bool STEP = false>
cudaError_t launch_split(const CacheView &cv, const void *q_t, float *part_o,
                         float2 *part_ml, unsigned int *tickets, void *o_t, bool o_f32,
                         int B, int Hq, int Hkv, int64_t n_keys, int nsplit,
                         float scale_log2, cudaStream_t s, const long long *lens = nullptr,
                         int g = 0, int w = 0, int64_t core_cap = 0, int stride = 0,
                         const StepArgs &st = StepArgs{})
{
    using S = DecodeShape<D>;
    // score buffer (a fused step pools a group in it: (r + 1) g floats),
    // partial sums, statistics; the same layout as the kernel's
    const int r = Hq / Hkv;
    const int lg_floats = STEP ? std::max(R * kDecodeChunk, (r + 1) * st.g) : R * kDecodeChunk;
    const size_t smem = sizeof(float) * (lg_floats + S::NG * R * D + 2 * R);
    auto kern = decode_split_kernel<D, R, STEP>;
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    dim3 grid(nsplit, B * Hkv);
    kern<<<grid, kDecodeThreads, smem, s>>>(cv, st, static_cast<const uint16_t *>(q_t),
                                            part_o, part_ml, tickets, o_t, o_f32 ? 1 : 0,
                                            Hq, Hkv, n_keys, kDecodeChunk, nsplit,
                                            scale_log2, lens, g, w, core_cap, stride);
    return cudaGetLastError();
}

}  // namespace

DecodePlan decode_plan(int64_t t, int g, int w, int B, int Hkv)
{
    (void)B;
    (void)Hkv;
    DecodePlan p;
    p.ws = window_start(t, g, w);
    p.n_core = p.ws / g;
    p.n_keys = p.n_core + (t - p.ws + 1);
    p.chunk = kDecodeChunk;
    p.nsplit = static_cast<int>((p.n_keys + kDecodeChunk - 1) / kDecodeChunk);
    return p;
}

int decode_max_splits(int64_t core_cap, int64_t tail_cap)
{
    return static_cast<int>((core_cap + tail_cap + kDecodeChunk - 1) / kDecodeChunk);
}

// Workspace: part_o [B, Hq, splits, d] fp32 | part_ml [B, Hq, splits] (max,
// sum) | tickets [B * Hkv] u32, each part 256-byte aligned.
namespace {
struct WorkspaceLayout {
    size_t o_bytes, ml_bytes, ticket_bytes;
};
WorkspaceLayout workspace_layout(int B, int Hq, int Hkv, int d, int64_t core_cap,
                                 int64_t tail_cap)
{
    const size_t rows = static_cast<size_t>(B) * Hq *
                        static_cast<size_t>(decode_max_splits(core_cap, tail_cap));
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return {up(rows * d * sizeof(float)), up(rows * sizeof(float2)),
            up(static_cast<size_t>(B) * Hkv * sizeof(unsigned int))};
}
}  // namespace

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t core_cap,
                              int64_t tail_cap)
{
    const WorkspaceLayout L = workspace_layout(B, Hq, Hkv, d, core_cap, tail_cap);
    return L.o_bytes + L.ml_bytes + L.ticket_bytes;
}

cudaError_t launch_decode(const void *k_core, const void *v_core,
                          const void *k_tail, const void *v_tail,
                          const void *q_t, void *o_t, bool o_f32,
                          void *workspace, int B, int Hq, int Hkv, int d,
                          int g, int w, int64_t core_cap, int64_t tail_cap,
                          int64_t t, cudaStream_t s)
{
    const DecodePlan p = decode_plan(t, g, w, B, Hkv);
    const WorkspaceLayout L = workspace_layout(B, Hq, Hkv, d, core_cap, tail_cap);
    char *ws = static_cast<char *>(workspace);
    float *part_o = reinterpret_cast<float *>(ws);
    float2 *part_ml = reinterpret_cast<float2 *>(ws + L.o_bytes);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(ws + L.o_bytes + L.ml_bytes);
    CacheView cv{static_cast<const uint16_t *>(k_core),
                 static_cast<const uint16_t *>(v_core),
                 static_cast<const uint16_t *>(k_tail),
                 static_cast<const uint16_t *>(v_tail),
                 core_cap,
                 tail_cap,
                 p.ws,
                 p.n_core,
                 p.ws % tail_cap};
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    const int r = Hq / Hkv;
    // the tickets start at zero on every call (the workspace is not
    // assumed to hold anything)
    cudaError_t e = cudaMemsetAsync(tickets, 0, sizeof(unsigned int) * B * Hkv, s);
    if (e != cudaSuccess) return e;
#define CCA_SPLIT(DD, RR)                                                          \
    e = launch_split<DD, RR>(cv, q_t, part_o, part_ml, tickets, o_t, o_f32, B, Hq, \
                             Hkv, p.n_keys, p.nsplit, scale_log2, s)
    if (d == 128) {
        if (r == 1) CCA_SPLIT(128, 1);
        else if (r == 2) CCA_SPLIT(128, 2);
        else if (r <= 4) CCA_SPLIT(128, 4);
        else if (r <= 8) CCA_SPLIT(128, 8);
        else CCA_SPLIT(128, 16);
    } else {
        if (r == 1) CCA_SPLIT(64, 1);
        else if (r == 2) CCA_SPLIT(64, 2);
        else if (r <= 4) CCA_SPLIT(64, 4);
        else if (r <= 8) CCA_SPLIT(64, 8);
        else CCA_SPLIT(64, 16);
    }
#undef CCA_SPLIT
    return e;
}

cudaError_t launch_decode_step(void *k_core, void *v_core, void *k_tail, void *v_tail,
                               const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               bool o_f32, void *workspace, int B, int Hq, int Hkv, int d,
                               int g, int w, int64_t core_cap, int64_t tail_cap, int64_t t,
                               cudaStream_t s)
{
    const DecodePlan p = decode_plan(t, g, w, B, Hkv);
    const WorkspaceLayout L = workspace_layout(B, Hq, Hkv, d, core_cap, tail_cap);
    char *ws = static_cast<char *>(workspace);
    float *part_o = reinterpret_cast<float *>(ws);
    float2 *part_ml = reinterpret_cast<float2 *>(ws + L.o_bytes);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(ws + L.o_bytes + L.ml_bytes);
    CacheView cv{static_cast<const uint16_t *>(k_core),
                 static_cast<const uint16_t *>(v_core),
                 static_cast<const uint16_t *>(k_tail),
                 static_cast<const uint16_t *>(v_tail),
                 core_cap,
                 tail_cap,
                 p.ws,
                 p.n_core,
                 p.ws % tail_cap};
    StepArgs st{static_cast<const uint16_t *>(k_t),
                static_cast<const uint16_t *>(v_t),
                static_cast<uint16_t *>(k_core),
                static_cast<uint16_t *>(v_core),
                static_cast<uint16_t *>(k_tail),
                static_cast<uint16_t *>(v_tail),
                g,
                t};
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    const int r = Hq / Hkv;
    // no ticket clearing here: every call leaves the tickets at zero, and a
    // new workspace is zero-filled by its owner (see cca_decode_step)
    cudaError_t e = cudaSuccess;
#define CCA_SPLIT(DD, RR)                                                                \
    e = launch_split<DD, RR, true>(cv, q_t, part_o, part_ml, tickets, o_t, o_f32, B, Hq,  \
                                   Hkv, p.n_keys, p.nsplit, scale_log2, s, nullptr, 0, 0, \
                                   0, 0, st)
    if (d == 128) {
        if (r == 1) CCA_SPLIT(128, 1);
        else if (r == 2) CCA_SPLIT(128, 2);
        else if (r <= 4) CCA_SPLIT(128, 4);
        else if (r <= 8) CCA_SPLIT(128, 8);
        else CCA_SPLIT(128, 16);
    } else {
        if (r == 1) CCA_SPLIT(64, 1);
        else if (r == 2) CCA_SPLIT(64, 2);
        else if (r <= 4) CCA_SPLIT(64, 4);
        else if (r <= 8) CCA_SPLIT(64, 8);
        else CCA_SPLIT(64, 16);
    }
#undef CCA_SPLIT
    return e;
}

cudaError_t launch_decode_rows(const void *k_core, const void *v_core,
                               const void *k_tail, const void *v_tail,
                               const void *q_t, void *o_t, bool o_f32,
                               void *workspace, const long long *lens, int B, int Hq,
                               int Hkv, int d, int g, int w, int64_t core_cap,
                               int64_t tail_cap, cudaStream_t s)
{
    const WorkspaceLayout L = workspace_layout(B, Hq, Hkv, d, core_cap, tail_cap);
    const int maxs = decode_max_splits(core_cap, tail_cap);
    char *ws = static_cast<char *>(workspace);
    float *part_o = reinterpret_cast<float *>(ws);
    float2 *part_ml = reinterpret_cast<float2 *>(ws + L.o_bytes);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(ws + L.o_bytes + L.ml_bytes);
    // ws and n_core are planned per row inside the kernel
    CacheView cv{static_cast<const uint16_t *>(k_core),
                 static_cast<const uint16_t *>(v_core),
                 static_cast<const uint16_t *>(k_tail),
                 static_cast<const uint16_t *>(v_tail),
                 core_cap,
                 tail_cap,
                 0,
                 0,
                 0};
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    const int r = Hq / Hkv;
    cudaError_t e = cudaMemsetAsync(tickets, 0, sizeof(unsigned int) * B * Hkv, s);
    if (e != cudaSuccess) return e;
#define CCA_SPLIT(DD, RR)                                                            \
    e = launch_split<DD, RR>(cv, q_t, part_o, part_ml, tickets, o_t, o_f32, B, Hq,   \
                             Hkv, 0, maxs, scale_log2, s, lens, g, w, core_cap, maxs)
    if (d == 128) {
        if (r == 1) CCA_SPLIT(128, 1);
        else if (r == 2) CCA_SPLIT(128, 2);
        else if (r <= 4) CCA_SPLIT(128, 4);
        else if (r <= 8) CCA_SPLIT(128, 8);
        else CCA_SPLIT(128, 16);
    } else {
        if (r == 1) CCA_SPLIT(64, 1);
        else if (r == 2) CCA_SPLIT(64, 2);
        else if (r <= 4) CCA_SPLIT(64, 4);
        else if (r <= 8) CCA_SPLIT(64, 8);
        else CCA_SPLIT(64, 16);
    }
#undef CCA_SPLIT
    return e;
}

cudaError_t decode_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_decode_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_decode_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
