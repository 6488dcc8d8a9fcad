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
// output) per query head; a merge kernel rescales and adds the partials.
#include "common.cuh"
#include "internal.h"

namespace cca {

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
    // Row of key k (0 <= k < n_keys) of pair bh: core slot k, or the ring
    // slot of raw token ws + (k - n_core).
    __device__ __forceinline__ int64_t row(int64_t bh, int64_t k, bool &core) const
    {
        core = k < n_core;
        return core ? bh * core_cap + k
                    : bh * tail_cap + (ws + (k - n_core)) % tail_cap;
    }
};

template <int D, int R>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(CacheView cv, const uint16_t *__restrict__ q_t,
                        float *__restrict__ part_o, float2 *__restrict__ part_ml,
                        int Hq, int Hkv, int64_t n_keys, int chunk, int nsplit,
                        float scale_log2)
{
    using S = DecodeShape<D>;
    extern __shared__ float dsm[];
    const int r = Hq / Hkv;
    float *lg = dsm;                               // [R][chunk]
    float *red = dsm + R * chunk;                  // [NG][R][D]
    float *stat = red + S::NG * R * D;             // [R][2]
    const int split = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / Hkv, h = bh - b * Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kl = lane % S::KL, kg = warp * S::KPW + lane / S::KL;
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

    // Scores of this chunk's keys, all query heads at once.  The loop bound
    // is the same for every lane (the shuffles below need the whole warp);
    // each lane's key i = base + kg + u * NG is guarded instead.
    for (int base = 0; base < nk; base += 4 * S::NG) {
        const int i0 = base + kg;
        uint4 kv[4];
        bool kcore[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            kv[u] = make_uint4(0u, 0u, 0u, 0u);
            kcore[u] = false;
            if (i < nk) {
                const int64_t row = cv.row(bh, c0 + i, kcore[u]);
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
                    if (kl == 0 && i < nk) lg[k * chunk + i] = s * scale_log2;
                }
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
    for (int base = 0; base < nk; base += 4 * S::NG) {
        const int i0 = base + kg;
        uint4 vv[4];
        bool vcore[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            vv[u] = make_uint4(0u, 0u, 0u, 0u);
            vcore[u] = false;
            if (i < nk) {
                const int64_t row = cv.row(bh, c0 + i, vcore[u]);
                const uint16_t *src = vcore[u] ? cv.v_core : cv.v_tail;
                vv[u] = ldg_stream(src + row * D + kl * 8);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * S::NG;
            if (i < nk) {
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
        const int64_t qrow = (b * Hq + h * r + k) * nsplit + split;
        part_o[qrow * D + c] = s;
        if (c == 0) part_ml[qrow] = make_float2(stat[2 * k], stat[2 * k + 1]);
    }
}

// One warp per (batch, query head): combine the splits' partials.  Lanes
// take the splits in parallel for the maximum and the weights
// 2^(m_s - max), which go to shared memory; then each lane adds its D/32
// output dims over the splits with independent loads.
constexpr int kMergeWarps = 4;

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
    decode_merge_kernel(const float *__restrict__ part_o,
                        const float2 *__restrict__ part_ml, void *__restrict__ o_t,
                        int out_f32, int64_t rows, int nsplit)
{
    constexpr int DPL = D / 32;
    extern __shared__ float merge_w[];  // [kMergeWarps][nsplit]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeWarps + warp;
    if (row >= rows) return;
    float *w = merge_w + warp * nsplit;
    const float2 *ml = part_ml + row * nsplit;
    float mx = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) mx = fmaxf(mx, ml[s].x);
    mx = warp_max(mx);
    float l = 0.f;
    for (int s = lane; s < nsplit; s += 32) {
        const float2 v = ml[s];
        const float c = fast_exp2(v.x - mx);
        w[s] = c;
        l = fmaf(c, v.y, l);
    }
    l = warp_sum(l);
    __syncwarp();
    float acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    const float *po = part_o + row * nsplit * D + lane * DPL;
#pragma unroll 4
    for (int s = 0; s < nsplit; ++s) {
        const float c = w[s];
        const float *src = po + static_cast<int64_t>(s) * D;
        if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(src);
            acc[0] = fmaf(c, v.x, acc[0]);
            acc[1] = fmaf(c, v.y, acc[1]);
            acc[2] = fmaf(c, v.z, acc[2]);
            acc[3] = fmaf(c, v.w, acc[3]);
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(src);
            acc[0] = fmaf(c, v.x, acc[0]);
            acc[1] = fmaf(c, v.y, acc[1]);
        }
    }
    const float inv = 1.0f / l;
    if (out_f32) {
        float *o = static_cast<float *>(o_t) + row * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[e] = acc[e] * inv;
    } else {
        uint16_t *o = static_cast<uint16_t *>(o_t) + row * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; e += 2)
            *reinterpret_cast<uint32_t *>(o + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    }
}

template <int D, int R>
cudaError_t launch_split(const CacheView &cv, const void *q_t, float *part_o,
                         float2 *part_ml, int B, int Hq, int Hkv, int64_t n_keys,
                         int nsplit, float scale_log2, cudaStream_t s)
{
    using S = DecodeShape<D>;
    const size_t smem =
        sizeof(float) * (R * kDecodeChunk + S::NG * R * D + 2 * R);
    auto kern = decode_split_kernel<D, R>;
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    dim3 grid(nsplit, B * Hkv);
    kern<<<grid, kDecodeThreads, smem, s>>>(cv, static_cast<const uint16_t *>(q_t),
                                            part_o, part_ml, Hq, Hkv, n_keys,
                                            kDecodeChunk, nsplit, scale_log2);
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

size_t decode_workspace_bytes(int B, int Hq, int d, int64_t core_cap,
                              int64_t tail_cap)
{
    const size_t rows = static_cast<size_t>(B) * Hq *
                        static_cast<size_t>(decode_max_splits(core_cap, tail_cap));
    size_t o_bytes = rows * d * sizeof(float);
    o_bytes = (o_bytes + 255) / 256 * 256;
    return o_bytes + rows * sizeof(float2);
}

cudaError_t launch_decode(const void *k_core, const void *v_core,
                          const void *k_tail, const void *v_tail,
                          const void *q_t, void *o_t, bool o_f32,
                          void *workspace, int B, int Hq, int Hkv, int d,
                          int g, int w, int64_t core_cap, int64_t tail_cap,
                          int64_t t, cudaStream_t s)
{
    const DecodePlan p = decode_plan(t, g, w, B, Hkv);
    const int maxs = decode_max_splits(core_cap, tail_cap);
    const size_t rows_max = static_cast<size_t>(B) * Hq * maxs;
    size_t o_bytes = rows_max * d * sizeof(float);
    o_bytes = (o_bytes + 255) / 256 * 256;
    float *part_o = static_cast<float *>(workspace);
    float2 *part_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) + o_bytes);
    CacheView cv{static_cast<const uint16_t *>(k_core),
                 static_cast<const uint16_t *>(v_core),
                 static_cast<const uint16_t *>(k_tail),
                 static_cast<const uint16_t *>(v_tail),
                 core_cap,
                 tail_cap,
                 p.ws,
                 p.n_core};
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    const int r = Hq / Hkv;
    cudaError_t e;
#define CCA_SPLIT(DD, RR)                                                          \
    e = launch_split<DD, RR>(cv, q_t, part_o, part_ml, B, Hq, Hkv, p.n_keys,     \
                             p.nsplit, scale_log2, s)
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
    if (e != cudaSuccess) return e;
    const int64_t rows = static_cast<int64_t>(B) * Hq;
    const int blocks = static_cast<int>((rows + kMergeWarps - 1) / kMergeWarps);
    const size_t msmem = sizeof(float) * kMergeWarps * p.nsplit;
    if (d == 128)
        decode_merge_kernel<128><<<blocks, kMergeWarps * 32, msmem, s>>>(
            part_o, part_ml, o_t, o_f32 ? 1 : 0, rows, p.nsplit);
    else
        decode_merge_kernel<64><<<blocks, kMergeWarps * 32, msmem, s>>>(
            part_o, part_ml, o_t, o_f32 ? 1 : 0, rows, p.nsplit);
    return cudaGetLastError();
}

}  // namespace cca
