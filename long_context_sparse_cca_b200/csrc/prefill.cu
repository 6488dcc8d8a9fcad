// cca_attn_prefill: fused core + local attention over a whole sequence
// (sections 局部保留模块 and 全局-局部模块可微融合 of the CCA write-up; its
// section 基于 Triton 的底层加速 describes the authors' FlashAttention-style
// fused operator, which this kernel re-designs for sm_100a).
//
// Query t attends to two key streams under one online softmax:
//   local stream K/V rows ws(t) .. t             (raw window, bf16)
//   core stream  Kc/Vc rows j < ws(t)/g          (pooled groups, fp16)
// with ws(t) = g * floor(max(t - w, 0) / g).  Local tiles run as bf16 x bf16
// MMAs with bf16 P; core tiles as fp16 x fp16 MMAs against an fp16 copy of
// the Q tile, with fp16 P.
//
// Design (one persistent CTA per SM, 192 threads):
//   warps 0-3  softmax: thread i owns query row i of the 128-row tile; makes
//              the fp16 copy of Q; reads S from tensor memory, masks, online
//              softmax (fp32, exp2, lazy rescale), writes P back into tensor
//              memory over S, rescales O when its max moved, and runs the
//              epilogue O / l.
//   warp 4     TMA producer: Q tile, then per key tile a K tile and a V tile
//              into multi-stage shared-memory rings (128-byte swizzle).
//   warp 5     tcgen05 issuer: S = Q K^T (A, B from shared memory) into one of
//              two S buffers in tensor memory; O += P V (A = P from tensor
//              memory, B = V from shared memory).
// Tensor memory: S0 [0,128), S1 [128,256), O [256, 256 + D) columns.
// Work items are (query tile, batch, query head), heaviest (latest) query
// tiles first, dealt round-robin to the CTAs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cca {

__device__ unsigned int g_prefill_status;  // kStatusTimeout | kStatusRange

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;         // log2 units

template <int D>
struct Pf {
    // 128 query rows per tile, 128 keys per tile
    static constexpr int NBOX = D / 64;          // 64-column swizzled boxes
    static constexpr int BOX_BYTES = 128 * 128;  // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;
    static constexpr int KST = D == 128 ? 3 : 4;  // K ring stages
    static constexpr int VST = D == 128 ? 2 : 3;  // V ring stages
    static constexpr int OFF_Q = 0;                     // Q tile, bf16
    static constexpr int OFF_QH = TILE_BYTES;           // Q tile, fp16 copy
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    static constexpr int SMEM = OFF_BAR + 512 + 1024;  // + barriers + align slack
    static constexpr uint32_t S_STRIDE = 128;  // S buffer b at column b * 128
    static constexpr uint32_t O_COL = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

struct Params {
    int B, Hq, Hkv, r;
    int T, g, w, m;
    int n_qtiles, n_items;
    float scale_log2;
    void *O;
    int o_f32;
};

// Geometry of one work item (query tile t0 .. tlast of one batch entry and
// query head).  Its key tiles are the local stream first (raw keys
// ws(t0) .. tlast, bf16), then the core stream (pooled keys 0 ..
// ws(tlast)/g - 1, fp16).
struct Geom {
    int b, hq, h, t0, tlast;
    int ws_lo, ws_hi;     // ws(t0), ws(tlast)
    int nc_lo, nc_hi;     // core counts of the first / last row
    int n_local, n_core_tiles, n_tiles;
};

__device__ __forceinline__ int ws_of(int t, int g, int w)
{
    const int lo = t > w ? t - w : 0;
    return (lo / g) * g;
}

__device__ __forceinline__ Geom geom(int item, const Params &p)
{
    Geom G;
    const int bhq_count = p.B * p.Hq;
    const int qt = p.n_qtiles - 1 - item / bhq_count;
    const int bhq = item - (item / bhq_count) * bhq_count;
    G.b = bhq / p.Hq;
    G.hq = bhq - G.b * p.Hq;
    G.h = G.hq / p.r;
    G.t0 = qt * 128;
    G.tlast = min(G.t0 + 127, p.T - 1);
    G.ws_lo = ws_of(G.t0, p.g, p.w);
    G.ws_hi = ws_of(G.tlast, p.g, p.w);
    G.nc_lo = G.ws_lo / p.g;
    G.nc_hi = G.ws_hi / p.g;
    G.n_core_tiles = (G.nc_hi + 127) / 128;
    G.n_local = (G.tlast - G.ws_lo + 1 + 127) / 128;
    G.n_tiles = G.n_local + G.n_core_tiles;
    return G;
}

// Key tile j of an item: stream and first key index.
__device__ __forceinline__ bool tile_is_core(const Geom &G, int j) { return j >= G.n_local; }
__device__ __forceinline__ int tile_key0(const Geom &G, int j)
{
    return j >= G.n_local ? (j - G.n_local) * 128 : G.ws_lo + j * 128;
}

struct Bars {
    uint64_t q_full, q_empty, qh_full;
    uint64_t k_full[4], k_empty[4];
    uint64_t v_full[4], v_empty[4];
    uint64_t s_full[2], p_full[2];
    uint64_t o_bar, o_empty, mma_done;
    uint32_t tmem_base;
    int abort;  // set when any role gives up
    int never;  // stays 0: drain waits are bounded by time only
};

__device__ __forceinline__ void record_timeout(Bars *bars)
{
    atomicOr(&g_prefill_status, kStatusTimeout);
    *reinterpret_cast<volatile int *>(&bars->abort) = 1;
}

// All lanes wait; the warp proceeds only if every lane saw completion.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Bars *bars)
{
    bool ok = wait_bounded(bar, parity, &bars->abort, kWaitLimitNs);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) record_timeout(bars);
    return ok;
}

__device__ __forceinline__ bool lane_wait(uint64_t *bar, uint32_t parity, Bars *bars)
{
    const bool ok = wait_bounded(bar, parity, &bars->abort, kWaitLimitNs);
    if (!ok) record_timeout(bars);
    return ok;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const Params p)
{
    using C = Pf<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sQh = smem + C::OFF_QH;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->qh_full, 4);
        for (int s = 0; s < C::KST; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < C::VST; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], 4);
        }
        mbar_init(&bars->o_bar, 1);
        mbar_init(&bars->o_empty, 4);
        mbar_init(&bars->mma_done, 1);
        bars->abort = 0;
        bars->never = 0;
        mbar_fence_init();
    }
    if (warp == 4) {
        tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc = 0, vc = 0, qc = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                const Geom G = geom(item, p);
                if (qc > 0 && !(ok = lane_wait(&bars->q_empty, (qc - 1) & 1, bars))) break;
                mbar_arrive_expect_tx(&bars->q_full, C::TILE_BYTES);
                for (int bx = 0; bx < C::NBOX; ++bx)
                    tma_load_3d(sQ + bx * C::BOX_BYTES, &tmQ, &bars->q_full, bx * 64,
                                G.t0, G.b * p.Hq + G.hq);
                ++qc;
                const int z = G.b * p.Hkv + G.h;
                for (int j = 0; j < G.n_tiles; ++j) {
                    const bool core = tile_is_core(G, j);
                    const int key0 = tile_key0(G, j);
                    const CUtensorMap *mk = core ? &tmKc : &tmK;
                    const CUtensorMap *mv = core ? &tmVc : &tmV;
                    {
                        const int s = kc % C::KST;
                        if (!(ok = lane_wait(&bars->k_empty[s], ((kc / C::KST) & 1) ^ 1, bars)))
                            break;
                        mbar_arrive_expect_tx(&bars->k_full[s], C::TILE_BYTES);
                        for (int bx = 0; bx < C::NBOX; ++bx)
                            tma_load_3d(sK + s * C::TILE_BYTES + bx * C::BOX_BYTES, mk,
                                        &bars->k_full[s], bx * 64, key0, z);
                        ++kc;
                    }
                    {
                        const int s = vc % C::VST;
                        if (!(ok = lane_wait(&bars->v_empty[s], ((vc / C::VST) & 1) ^ 1, bars)))
                            break;
                        mbar_arrive_expect_tx(&bars->v_full[s], C::TILE_BYTES);
                        for (int bx = 0; bx < C::NBOX; ++bx)
                            tma_load_3d(sV + s * C::TILE_BYTES + bx * C::BOX_BYTES, mv,
                                        &bars->v_full[s], bx * 64, key0, z);
                        ++vc;
                    }
                }
            }
            // Drain: every issued copy must have landed before the CTA exits
            // (the last fill of each ring stage, and the last Q tile).
            const volatile int *never = &bars->never;
            for (uint32_t s = 0; s < C::KST && s < kc; ++s) {
                const uint32_t last = kc - 1 - ((kc - 1 - s) % C::KST);
                wait_bounded(&bars->k_full[last % C::KST], (last / C::KST) & 1, never,
                             kWaitLimitNs);
            }
            for (uint32_t s = 0; s < C::VST && s < vc; ++s) {
                const uint32_t last = vc - 1 - ((vc - 1 - s) % C::VST);
                wait_bounded(&bars->v_full[last % C::VST], (last / C::VST) & 1, never,
                             kWaitLimitNs);
            }
            if (qc > 0) wait_bounded(&bars->q_full, (qc - 1) & 1, never, kWaitLimitNs);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk_bf = idesc_f32acc(128, 128, true, false, false);
            constexpr uint32_t idesc_qk_h = idesc_f32acc(128, 128, false, false, false);
            constexpr uint32_t idesc_pv_bf = idesc_f32acc(128, D, true, false, true);
            constexpr uint32_t idesc_pv_h = idesc_f32acc(128, D, false, false, true);
            const uint32_t q_base = smem_addr(sQ), qh_base = smem_addr(sQh),
                           k_base = smem_addr(sK), v_base = smem_addr(sV);
            uint32_t kc = 0, vc = 0, it = 0, qhc = 0;
            int k = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.n_items;
                 item += gridDim.x, ++k) {
                const Geom G = geom(item, p);
                if (!(ok = lane_wait(&bars->q_full, k & 1, bars))) break;
                const uint32_t it0 = it;
                auto issue_pv = [&](int jj) -> bool {
                    const uint32_t itp = it0 + jj;
                    const uint32_t bp = itp & 1;
                    if (!lane_wait(&bars->p_full[bp], (itp >> 1) & 1, bars)) return false;
                    const uint32_t sv = vc % C::VST;
                    if (!lane_wait(&bars->v_full[sv], (vc / C::VST) & 1, bars)) return false;
                    if (jj == 0 && k > 0 && !lane_wait(&bars->o_empty, (k - 1) & 1, bars))
                        return false;
                    tc_fence_after_sync();
                    const uint32_t idesc = tile_is_core(G, jj) ? idesc_pv_h : idesc_pv_bf;
                    const uint32_t vs = v_base + sv * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t bdesc =
                            smem_desc_sw128(vs + kk * 16 * 128, C::BOX_BYTES, 1024);
                        mma_ts(tmem + C::O_COL, tmem + bp * C::S_STRIDE + kk * 8, bdesc,
                               idesc, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars->o_bar);
                    mma_commit(&bars->v_empty[sv]);
                    ++vc;
                    return true;
                };
                for (int j = 0; j < G.n_tiles; ++j) {
                    const uint32_t b = it & 1;
                    const bool core = tile_is_core(G, j);
                    if (core && j == G.n_local) {
                        // the fp16 copy of Q is written by the softmax warps
                        if (!(ok = lane_wait(&bars->qh_full, qhc & 1, bars))) break;
                        ++qhc;
                    }
                    const uint32_t s = kc % C::KST;
                    if (!(ok = lane_wait(&bars->k_full[s], (kc / C::KST) & 1, bars))) break;
                    tc_fence_after_sync();
                    const uint32_t ks = k_base + s * C::TILE_BYTES;
                    const uint32_t qs = core ? qh_base : q_base;
                    const uint32_t idesc = core ? idesc_qk_h : idesc_qk_bf;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                        const uint64_t adesc = smem_desc_sw128(qs + off, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(ks + off, 16, 1024);
                        mma_ss(tmem + b * C::S_STRIDE, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->s_full[b]);
                    mma_commit(&bars->k_empty[s]);
                    ++kc;
                    if (j == G.n_tiles - 1) mma_commit(&bars->q_empty);
                    ++it;
                    if (j > 0 && !(ok = issue_pv(j - 1))) break;
                }
                if (ok) ok = issue_pv(G.n_tiles - 1);
            }
            // Wait for every issued tensor-core operation to finish.
            mma_commit(&bars->mma_done);
            wait_bounded(&bars->mma_done, 0, &bars->never, kWaitLimitNs);
        }
    } else {
        // ------------------------------------------------ softmax warps
        const int row = threadIdx.x;  // 0..127 = tensor-memory lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t it = 0, pv_waits = 0, k = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++k) {
            const Geom G = geom(item, p);
            const int t = G.t0 + row;
            const int ws_t = ws_of(t, p.g, p.w);
            const int nc_t = ws_t / p.g;
            if (!(ok = warp_wait(&bars->q_full, k & 1, bars))) break;
            if (G.n_core_tiles > 0) {
                // fp16 copy of the Q tile for the core stream (same swizzled
                // layout: 16-byte chunks of 8 elements keep their places)
                bool over = false;
                const uint4 *src = reinterpret_cast<const uint4 *>(sQ);
                uint4 *dst = reinterpret_cast<uint4 *>(sQh);
#pragma unroll 4
                for (int c = threadIdx.x; c < C::TILE_BYTES / 16; c += 128) {
                    const uint4 v = src[c];
                    uint4 h;
                    h.x = pack_f16x2(clamp_f16(bf16_lo(v.x), over), clamp_f16(bf16_hi(v.x), over));
                    h.y = pack_f16x2(clamp_f16(bf16_lo(v.y), over), clamp_f16(bf16_hi(v.y), over));
                    h.z = pack_f16x2(clamp_f16(bf16_lo(v.z), over), clamp_f16(bf16_hi(v.z), over));
                    h.w = pack_f16x2(clamp_f16(bf16_lo(v.w), over), clamp_f16(bf16_hi(v.w), over));
                    dst[c] = h;
                }
                if (over) atomicOr(&g_prefill_status, kStatusRange);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->qh_full);
            }
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < G.n_tiles; ++j, ++it) {
                const uint32_t b = it & 1;
                if (!(ok = warp_wait(&bars->s_full[b], (it >> 1) & 1, bars))) break;
                tc_fence_after_sync();
                float x[128];
                {
                    uint32_t u[128];
                    tmem_ld128_wait(tmem + lane_off + b * C::S_STRIDE, u);
#pragma unroll
                    for (int e = 0; e < 128; ++e) x[e] = __uint_as_float(u[e]);
                }
                // Mask keys this row does not see.
                const bool core = tile_is_core(G, j);
                const int key0 = tile_key0(G, j);
                const bool need_mask = core ? (key0 + 128 > G.nc_lo)
                                            : (key0 < G.ws_hi || key0 + 127 > G.t0);
                if (need_mask) {
                    const int lo = core ? 0 : ws_t;
                    const int hi = core ? nc_t - 1 : t;
#pragma unroll
                    for (int e = 0; e < 128; ++e) {
                        const int key = key0 + e;
                        if (key < lo || key > hi) x[e] = -INFINITY;
                    }
                }
                float mx = x[0];
#pragma unroll
                for (int e = 1; e < 128; ++e) mx = fmaxf(mx, x[e]);
                const float m_tile = mx * p.scale_log2;
                float alpha = 1.f;
                if (m_tile > m_run + kRescaleThreshold) {
                    alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_tile);
                    m_run = m_tile;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                // P in the element type of this tile's values (fp16 core,
                // bf16 raw); the row sum uses the rounded weights P V sees.
                uint32_t pk[64];
                float rs = 0.f;
                if (core) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const float p0 = fast_exp2(fmaf(x[2 * e], p.scale_log2, -m_use));
                        const float p1 = fast_exp2(fmaf(x[2 * e + 1], p.scale_log2, -m_use));
                        pk[e] = pack_f16x2(p0, p1);
                        rs += f16_lo(pk[e]) + f16_hi(pk[e]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const float p0 = fast_exp2(fmaf(x[2 * e], p.scale_log2, -m_use));
                        const float p1 = fast_exp2(fmaf(x[2 * e + 1], p.scale_log2, -m_use));
                        pk[e] = pack_bf16x2(p0, p1);
                        rs += bf16_lo(pk[e]) + bf16_hi(pk[e]);
                    }
                }
                l_run = fmaf(l_run, alpha, rs);
                if (j > 0) {
                    // O must hold P V of the previous tile before it is rescaled
                    if (!(ok = warp_wait(&bars->o_bar, pv_waits & 1, bars))) break;
                    ++pv_waits;
                    tc_fence_after_sync();
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t u[32];
                            tmem_ld32_wait(tmem + lane_off + C::O_COL + c * 32, u);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                            tmem_st32(tmem + lane_off + C::O_COL + c * 32, u);
                        }
                    }
                }
                {
                    uint32_t u[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = pk[e];
                    tmem_st32(tmem + lane_off + b * C::S_STRIDE, u);
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = pk[32 + e];
                    tmem_st32(tmem + lane_off + b * C::S_STRIDE + 32, u);
                }
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[b]);
            }
            if (!ok) break;
            // Epilogue: O / l for this row.
            if (!(ok = warp_wait(&bars->o_bar, pv_waits & 1, bars))) break;
            ++pv_waits;
            tc_fence_after_sync();
            float o[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t u[32];
                tmem_ld32_wait(tmem + lane_off + C::O_COL + c * 32, u);
#pragma unroll
                for (int e = 0; e < 32; ++e) o[c * 32 + e] = __uint_as_float(u[e]);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_empty);
            if (t < p.T) {
                const float inv = 1.0f / l_run;
                const int64_t orow =
                    (static_cast<int64_t>(G.b) * p.Hq + G.hq) * p.T + t;
                if (p.o_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.O) +
                                                             orow * D);
#pragma unroll
                    for (int c = 0; c < D / 4; ++c)
                        dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv,
                                             o[4 * c + 2] * inv, o[4 * c + 3] * inv);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.O) +
                                                           orow * D);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c)
                        dst[c] = make_uint4(pack_bf16x2(o[8 * c] * inv, o[8 * c + 1] * inv),
                                            pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv),
                                            pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv),
                                            pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv));
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 3-D map over a [planes, rows, d] tensor of 16-bit elements (bf16 or
// fp16), 64 x 128 x 1 boxes, 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap *m, const void *ptr, int d, int64_t rows, int64_t planes,
              bool f16 = false)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(planes)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(rows) * d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          3, const_cast<void *>(ptr),
                          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const void *Q, const void *K, const void *V, const void *Kc,
                     const void *Vc, void *O, bool o_f32, int B, int Hq, int Hkv,
                     int64_t T, int g, int w, cudaStream_t s)
{
    using C = Pf<D>;
    CUtensorMap mQ, mK, mV, mKc, mVc;
    const int64_t m = T / g;
    bool ok = make_map(&mQ, Q, D, T, static_cast<int64_t>(B) * Hq) &&
              make_map(&mK, K, D, T, static_cast<int64_t>(B) * Hkv) &&
              make_map(&mV, V, D, T, static_cast<int64_t>(B) * Hkv);
    if (m > 0)
        ok = ok && make_map(&mKc, Kc, D, m, static_cast<int64_t>(B) * Hkv, true) &&
             make_map(&mVc, Vc, D, m, static_cast<int64_t>(B) * Hkv, true);
    else {  // no core rows: the core maps are never read
        mKc = mK;
        mVc = mV;
    }
    if (!ok) return cudaErrorInvalidValue;
    Params p;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.r = Hq / Hkv;
    p.T = static_cast<int>(T);
    p.g = g;
    p.w = w;
    p.m = static_cast<int>(m);
    p.n_qtiles = static_cast<int>((T + 127) / 128);
    p.n_items = p.n_qtiles * B * Hq;
    p.scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
    p.O = O;
    p.o_f32 = o_f32 ? 1 : 0;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = p.n_items < sms ? p.n_items : sms;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    prefill_kernel<D><<<grid, 192, C::SMEM, s>>>(mQ, mK, mV, mKc, mVc, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const void *Q, const void *K, const void *V,
                           const void *Kc, const void *Vc, void *O, bool o_f32,
                           int B, int Hq, int Hkv, int64_t T, int d, int g,
                           int w, cudaStream_t s)
{
    if (T == 0) return cudaSuccess;
    if (d == 128) return launch_d<128>(Q, K, V, Kc, Vc, O, o_f32, B, Hq, Hkv, T, g, w, s);
    return launch_d<64>(Q, K, V, Kc, Vc, O, o_f32, B, Hq, Hkv, T, g, w, s);
}

cudaError_t prefill_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_prefill_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_prefill_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
