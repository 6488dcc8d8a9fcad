// cca_attn_backward: gradients of CCA attention for training.
//
// The write-up calls the global-local fusion differentiable (section
// 全局-局部模块可微融合) and its fused operator serves training (section 基于
// Triton 的底层加速).  For upstream gradients dO of the fused attention output
// O, this computes dQ, dK, dV of L = sum(dO * O), where O depends on Q, K, V
// directly (queries; raw keys/values of the local window) and through the
// pooled core keys/values (section 全局感知池化).  With logits
// x = (q . key) / sqrt(d), P = softmax(x) per row (from the forward's
// log-sum-exp), dP = dO . value and D = rowsum(dO * O):
//   dS = P (dP - D),  dQ = sum dS key / sqrt(d),
//   dKey = sum dS q / sqrt(d),  dValue = sum P dO,
// for raw keys (dK, dV) and core keys (dKc, dVc); then the pooling's chain
// rule moves dKc, dVc onto the group's keys, values and scoring queries.
//
// Launches, in order on the caller's stream:
//   1. bw_prep_kernel: D = rowsum(dO * O); fp16 copies of Q and dO for the
//      core stream (core keys/values are fp16, and an MMA takes one type);
//   2. bw_dq_kernel (tcgen05): per 128-row query tile, over its key tiles
//      (local then core): S = Q K^T, dP = dO V^T, dS, dQ += dS K;
//   3. bw_dkv_kernel (tcgen05): per 128-key tile, over the query tiles and
//      query heads that see it: S^T = K Q^T, dP^T = V dO^T, dV += P^T dO,
//      dK += dS^T Q; raw tiles store dK, dV; core tiles (whose query range
//      is long, so it is cut into chunks) add into fp32 dKc, dVc;
//   4. bw_pool_kernel: one warp per group, the pooling's chain rule.
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_map.h"

namespace cca {

__device__ unsigned int g_backward_status;  // kStatusTimeout | kStatusRange

namespace {

constexpr uint64_t kBwWaitNs = 2000000000ull;  // 2 s per wait
constexpr int kCoreChunk = 16;                 // query tiles per core work item

template <int D>
struct Bt {
    static constexpr int NBOX = D / 64;
    static constexpr int BOX_BYTES = 128 * 128;
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;  // 128 rows x D, 16-bit
};

struct BwParams {
    int B, Hq, Hkv, r, T, g, w, m;
    float scale;       // 1 / sqrt(d)
    float scale_log2;  // log2(e) / sqrt(d)
    const float *lse;  // [B, Hq, T], log2 units
    const float *Dv;   // [B, Hq, T]
    float *dQ;         // [B, Hq, T, d]
    float *dK, *dV;    // [B, Hkv, T, d]
    float *dKc, *dVc;  // [B, Hkv, m, d], accumulated (zero on entry)
    int n_qt, n_kt, n_ct;
    int n_items, n_core_items;
};

__device__ __forceinline__ int ws_of(int t, int g, int w)
{
    const int lo = t > w ? t - w : 0;
    return (lo / g) * g;
}

// Shared helpers of the two tcgen05 kernels ---------------------------------

struct BwBars {
    uint64_t q_full[2], q_empty[2];  // query-side tiles (Q, dO)
    uint64_t k_full[4], k_empty[4];  // key-side ring (dQ kernel)
    uint64_t v_full[4], v_empty[4];
    uint64_t kv_full, kv_empty;      // key-side tiles (dK/dV kernel)
    uint64_t s_full, s_free, p_full, mm_done, acc_empty, drain;
    uint64_t hs_full[2], hp_full[2], hmm_done[2];  // per 64-query half (dK/dV kernel)
    uint32_t tmem_base;
    int abort, never;
};

__device__ __forceinline__ void bw_timeout(BwBars *bars)
{
    atomicOr(&g_backward_status, kStatusTimeout);
    *reinterpret_cast<volatile int *>(&bars->abort) = 1;
}

__device__ __forceinline__ bool bw_lane_wait(uint64_t *bar, uint32_t parity, BwBars *bars)
{
    const bool ok = wait_bounded(bar, parity, &bars->abort, kBwWaitNs);
    if (!ok) bw_timeout(bars);
    return ok;
}

__device__ __forceinline__ bool bw_warp_wait(uint64_t *bar, uint32_t parity, BwBars *bars)
{
    bool ok = wait_bounded(bar, parity, &bars->abort, kBwWaitNs);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) bw_timeout(bars);
    return ok;
}

// 128 x 128 x D product into TMEM columns, both operands K-major in shared
// memory (128-byte swizzled TMA tiles).
template <int D>
__device__ __forceinline__ void mma_kk(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc)
{
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        constexpr uint32_t box16 = Bt<D>::BOX_BYTES >> 4;
        const uint32_t off = (kk >> 2) * box16 + (kk & 3) * 2;
        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// 128 x D x 64 product: A (16-bit pairs, 32 columns) in TMEM, B MN-major in
// shared memory (64 rows along K); accumulate unless `first`.
__device__ __forceinline__ void mma_tm64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                         uint32_t idesc, bool first)
{
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
        mma_ts(d_tmem, a_tmem + kk * 8, b0 + kk * 128, idesc, (first && kk == 0) ? 0u : 1u);
}

// 128 x D x 128 product: A (16-bit pairs) in TMEM, B MN-major in shared
// memory; accumulate unless `first`.
__device__ __forceinline__ void mma_tm(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                       uint32_t idesc, bool first)
{
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(d_tmem, a_tmem + kk * 8, b0 + kk * 128, idesc, (first && kk == 0) ? 0u : 1u);
}

// Eight fp32 values x[0..8) * scale to global memory in one 32-byte store
// (p 32-byte aligned): a thread writing its own row fills whole sectors.
__device__ __forceinline__ void st_global_x8(float *ptr, const uint32_t *x, float scale)
{
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr),
                 "f"(__uint_as_float(x[0]) * scale), "f"(__uint_as_float(x[1]) * scale),
                 "f"(__uint_as_float(x[2]) * scale), "f"(__uint_as_float(x[3]) * scale),
                 "f"(__uint_as_float(x[4]) * scale), "f"(__uint_as_float(x[5]) * scale),
                 "f"(__uint_as_float(x[6]) * scale), "f"(__uint_as_float(x[7]) * scale)
                 : "memory");
}

// Four fp32 additions to global memory in one 16-byte reduction (p 16-byte
// aligned); the order among concurrent adders is unspecified.
__device__ __forceinline__ void red_add_v4(float *ptr, float a, float b, float c, float d)
{
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "f"(a),
                 "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// 1. D = rowsum(dO * O) and the fp16 copies --------------------------------

template <int D, bool OF32>
__global__ void bw_prep_kernel(const uint16_t *__restrict__ dO, const void *__restrict__ O,
                               const uint16_t *__restrict__ Q, float *__restrict__ Dv,
                               uint16_t *__restrict__ Q16, uint16_t *__restrict__ dO16,
                               int64_t rows)
{
    const int lane = threadIdx.x & 31;
    constexpr int DPL = D / 32;
    bool over = false;
    for (int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
         row < rows; row += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
        const int64_t base = row * D + lane * DPL;
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; e += 2) {
            const uint32_t g2 = *reinterpret_cast<const uint32_t *>(dO + base + e);
            const uint32_t q2 = *reinterpret_cast<const uint32_t *>(Q + base + e);
            float o0, o1;
            if (OF32) {
                const float2 o = *reinterpret_cast<const float2 *>(
                    static_cast<const float *>(O) + base + e);
                o0 = o.x;
                o1 = o.y;
            } else {
                const uint32_t o2 =
                    *reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(O) + base + e);
                o0 = bf16_lo(o2);
                o1 = bf16_hi(o2);
            }
            s = fmaf(bf16_lo(g2), o0, s);
            s = fmaf(bf16_hi(g2), o1, s);
            *reinterpret_cast<uint32_t *>(dO16 + base + e) =
                pack_f16x2(clamp_f16(bf16_lo(g2), over), clamp_f16(bf16_hi(g2), over));
            *reinterpret_cast<uint32_t *>(Q16 + base + e) =
                pack_f16x2(clamp_f16(bf16_lo(q2), over), clamp_f16(bf16_hi(q2), over));
        }
        s = warp_sum(s);
        if (lane == 0) Dv[row] = s;
    }
    if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(&g_backward_status, kStatusRange);
}

// 2. dQ ---------------------------------------------------------------------
//
// Work item: one 128-row query tile of one (batch, query head), latest tiles
// first.  Key tiles as in the forward: local (raw keys ws(t0) .. last row,
// bf16) then core (pooled keys 0 .. ws(last)/g - 1, fp16, against the fp16
// copies of Q and dO, reloaded at the switch).  Warps 0-7: the element-wise
// dS step, thread (w % 4) * 32 + lane owning one query row and warps w < 4 /
// w >= 4 its key columns [0, 64) / [64, 128) (a row needs no reduction);
// warp 8: TMA producer; warp 9: MMA issuer (one thread).  The issuer runs
// one tile ahead: S and dP of tile n+1 are issued once the dS warps have
// copied tile n's into registers, before dQ += dS K of tile n, so the tensor
// cores work while the dS step runs.
// TMEM: S [0,128), dP [128,256), dS [256,320) (16-bit pairs), dQ [320, +D).
constexpr int kDqSoftWarps = 8;
constexpr int kDqTmaWarp = 8, kDqMmaWarp = 9;
constexpr int kDqThreads = 320;
template <int D>
struct BqLayout {
    using T = Bt<D>;
    static constexpr int KST = D == 128 ? 3 : 4, VST = D == 128 ? 2 : 4;
    static constexpr int OFF_Q = 0, OFF_DO = T::TILE_BYTES;
    static constexpr int OFF_K = 2 * T::TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * T::TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * T::TILE_BYTES;
    static constexpr int SMEM = OFF_BAR + 512 + 1024;
    static constexpr uint32_t S_COL = 0, DP_COL = 128, DS_COL = 256, DQ_COL = 320;
};

struct QGeom {
    int b, hq, h, t0, tlast, ws_lo, n_local, n_core, n_tiles;
};

__device__ __forceinline__ QGeom q_geom(int item, const BwParams &p)
{
    QGeom G;
    const int bhq = p.B * p.Hq;
    const int qt = p.n_qt - 1 - item / bhq;
    const int x = item - (item / bhq) * bhq;
    G.b = x / p.Hq;
    G.hq = x - G.b * p.Hq;
    G.h = G.hq / p.r;
    G.t0 = qt * 128;
    G.tlast = min(G.t0 + 127, p.T - 1);
    G.ws_lo = ws_of(G.t0, p.g, p.w);
    G.n_local = (G.tlast - G.ws_lo + 1 + 127) / 128;
    G.n_core = (ws_of(G.tlast, p.g, p.w) / p.g + 127) / 128;
    G.n_tiles = G.n_local + G.n_core;
    return G;
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    bw_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmO16,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                 const BwParams p)
{
    using L = BqLayout<D>;
    using T = Bt<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::OFF_Q, *sO = smem + L::OFF_DO;
    uint8_t *sK = smem + L::OFF_K, *sV = smem + L::OFF_V;
    BwBars *bars = reinterpret_cast<BwBars *>(smem + L::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bhq = p.B * p.Hq;
    const int n_items = p.n_qt * bhq;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full[0], 1);
        mbar_init(&bars->q_empty[0], 1);
        for (int s = 0; s < L::KST; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < L::VST; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, kDqSoftWarps);
        mbar_init(&bars->p_full, kDqSoftWarps);
        mbar_init(&bars->mm_done, 1);
        mbar_init(&bars->acc_empty, kDqSoftWarps);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->never = 0;
        mbar_fence_init();
    }
    if (warp == kDqTmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    if (warp == kDqTmaWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc = 0, vc = 0, qc = 0;
            bool ok = true;
            auto load_q = [&](const CUtensorMap *mq, const CUtensorMap *mo, const QGeom &G) {
                if (qc > 0 && !(ok = bw_lane_wait(&bars->q_empty[0], (qc - 1) & 1, bars)))
                    return;
                mbar_arrive_expect_tx(&bars->q_full[0], 2 * T::TILE_BYTES);
                const int z = G.b * p.Hq + G.hq;
                for (int bx = 0; bx < T::NBOX; ++bx) {
                    tma_load_3d(sQ + bx * T::BOX_BYTES, mq, &bars->q_full[0], bx * 64, G.t0, z);
                    tma_load_3d(sO + bx * T::BOX_BYTES, mo, &bars->q_full[0], bx * 64, G.t0, z);
                }
                ++qc;
            };
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const QGeom G = q_geom(item, p);
                load_q(&tmQ, &tmO, G);
                const int z = G.b * p.Hkv + G.h;
                for (int j = 0; ok && j < G.n_tiles; ++j) {
                    const bool core = j >= G.n_local;
                    if (core && j == G.n_local) {
                        load_q(&tmQ16, &tmO16, G);
                        if (!ok) break;
                    }
                    const int key0 = core ? (j - G.n_local) * 128 : G.ws_lo + j * 128;
                    const int s = kc % L::KST;
                    if (!(ok = bw_lane_wait(&bars->k_empty[s], ((kc / L::KST) & 1) ^ 1, bars))) break;
                    mbar_arrive_expect_tx(&bars->k_full[s], T::TILE_BYTES);
                    for (int bx = 0; bx < T::NBOX; ++bx)
                        tma_load_3d(sK + s * T::TILE_BYTES + bx * T::BOX_BYTES, core ? &tmKc : &tmK,
                                    &bars->k_full[s], bx * 64, key0, z);
                    ++kc;
                    const int sv = vc % L::VST;
                    if (!(ok = bw_lane_wait(&bars->v_empty[sv], ((vc / L::VST) & 1) ^ 1, bars))) break;
                    mbar_arrive_expect_tx(&bars->v_full[sv], T::TILE_BYTES);
                    for (int bx = 0; bx < T::NBOX; ++bx)
                        tma_load_3d(sV + sv * T::TILE_BYTES + bx * T::BOX_BYTES, core ? &tmVc : &tmV,
                                    &bars->v_full[sv], bx * 64, key0, z);
                    ++vc;
                }
            }
            // drain: every issued copy has landed before the CTA exits
            const volatile int *never = &bars->never;
            for (uint32_t s = 0; s < L::KST && s < kc; ++s) {
                const uint32_t last = kc - 1 - ((kc - 1 - s) % L::KST);
                wait_bounded(&bars->k_full[last % L::KST], (last / L::KST) & 1, never, kBwWaitNs);
            }
            for (uint32_t s = 0; s < L::VST && s < vc; ++s) {
                const uint32_t last = vc - 1 - ((vc - 1 - s) % L::VST);
                wait_bounded(&bars->v_full[last % L::VST], (last / L::VST) & 1, never, kBwWaitNs);
            }
            if (qc > 0) wait_bounded(&bars->q_full[0], (qc - 1) & 1, never, kBwWaitNs);
        }
    } else if (warp == kDqMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s_bf = idesc_f32acc(128, 128, true, false, false);
            constexpr uint32_t id_s_h = idesc_f32acc(128, 128, false, false, false);
            constexpr uint32_t id_q_bf = idesc_f32acc(128, D, true, false, true);
            constexpr uint32_t id_q_h = idesc_f32acc(128, D, false, false, true);
            const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
            const uint64_t dO = smem_desc_sw128(smem_addr(sO), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_addr(sK), 16, 1024);
            const uint64_t dkm = smem_desc_sw128(smem_addr(sK), T::BOX_BYTES, 1024);
            const uint64_t dv = smem_desc_sw128(smem_addr(sV), 16, 1024);
            constexpr uint32_t kTile16 = T::TILE_BYTES >> 4;
            // Tiles are numbered n = 0, 1, ... over this CTA's items in
            // order; tile n uses K stage n % KST and V stage n % VST.  A(n)
            // issues S, dP of tile n; B(n) issues dQ += dS K of tile n.
            // Order: A(0), A(1), B(0), A(2), B(1), ...
            struct Cursor {
                int item, k, j;  // item index, its ordinal in this CTA, tile within it
                QGeom G;
                bool live;
            };
            auto start = [&](Cursor &c) {
                c.item = blockIdx.x;
                c.k = 0;
                c.j = 0;
                c.live = c.item < n_items;
                if (c.live) c.G = q_geom(c.item, p);
            };
            auto advance = [&](Cursor &c) {
                if (++c.j == c.G.n_tiles) {
                    c.item += gridDim.x;
                    ++c.k;
                    c.j = 0;
                    c.live = c.item < n_items;
                    if (c.live) c.G = q_geom(c.item, p);
                }
            };
            Cursor ca, cb;
            start(ca);
            start(cb);
            uint32_t na = 0, nb = 0, qc = 0;
            auto issue_a = [&]() -> bool {
                const bool core = ca.j >= ca.G.n_local;
                if (ca.j == 0 || (core && ca.j == ca.G.n_local)) {
                    // this item's query tiles (bf16), or their fp16 copies
                    if (!bw_lane_wait(&bars->q_full[0], qc & 1, bars)) return false;
                    ++qc;
                }
                const uint32_t s = na % L::KST, sv = na % L::VST;
                if (!bw_lane_wait(&bars->k_full[s], (na / L::KST) & 1, bars)) return false;
                if (!bw_lane_wait(&bars->v_full[sv], (na / L::VST) & 1, bars)) return false;
                if (na > 0 && !bw_lane_wait(&bars->s_free, (na - 1) & 1, bars)) return false;
                tc_fence_after_sync();
                mma_kk<D>(tmem + L::S_COL, dq, dk + s * kTile16, core ? id_s_h : id_s_bf);
                mma_kk<D>(tmem + L::DP_COL, dO, dv + sv * kTile16, core ? id_s_h : id_s_bf);
                mma_commit(&bars->s_full);
                mma_commit(&bars->v_empty[sv]);
                // the query tiles in shared memory are read for the last
                // time: before the switch to the fp16 copies, and at the
                // item's last tile
                if (ca.j + 1 == ca.G.n_tiles || (!core && ca.j + 1 == ca.G.n_local))
                    mma_commit(&bars->q_empty[0]);
                ++na;
                advance(ca);
                return true;
            };
            auto issue_b = [&]() -> bool {
                const bool core = cb.j >= cb.G.n_local;
                if (!bw_lane_wait(&bars->p_full, nb & 1, bars)) return false;
                if (cb.j == 0 && cb.k > 0 &&
                    !bw_lane_wait(&bars->acc_empty, (cb.k - 1) & 1, bars))
                    return false;
                tc_fence_after_sync();
                const uint32_t s = nb % L::KST;
                mma_tm(tmem + L::DQ_COL, tmem + L::DS_COL, dkm + s * kTile16,
                       core ? id_q_h : id_q_bf, cb.j == 0);
                mma_commit(&bars->mm_done);
                mma_commit(&bars->k_empty[s]);
                ++nb;
                advance(cb);
                return true;
            };
            bool ok = !ca.live || issue_a();
            while (ok && nb < na) {
                if (ca.live && !(ok = issue_a())) break;
                ok = issue_b();
            }
            mma_commit(&bars->drain);
            wait_bounded(&bars->drain, 0, &bars->never, kBwWaitNs);
        }
    } else {
        // ------------------------------------------------ dS warps
        const int row = threadIdx.x & 127;
        const int half = warp >> 2;  // key columns [64 half, 64 half + 64)
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const QGeom G = q_geom(item, p);
            const int t = G.t0 + row;
            const bool valid = t < p.T;
            const int64_t qrow = (static_cast<int64_t>(G.b) * p.Hq + G.hq) * p.T + t;
            const float lse = valid ? p.lse[qrow] : 0.f;
            const float dd = valid ? p.Dv[qrow] : 0.f;
            const int ws_t = ws_of(t, p.g, p.w);
            const int nc_t = ws_t / p.g;
            for (int j = 0; j < G.n_tiles; ++j, ++it) {
                if (!(ok = bw_warp_wait(&bars->s_full, it & 1, bars))) break;
                tc_fence_after_sync();
                const bool core = j >= G.n_local;
                const int key0 = core ? (j - G.n_local) * 128 : G.ws_lo + j * 128;
                const int lo = core ? 0 : ws_t, hi = core ? nc_t - 1 : t;
                uint32_t pk[2][16];
                // CORE: fp16 dS (core tiles) or bf16; MASK: test each key
                // against [lo, hi], skipped when every key of this half is
                // visible to every row of the warp
                auto elementwise = [&](auto core_c, auto mask_c) {
                    constexpr bool CORE = decltype(core_c)::value;
                    constexpr bool MASK = decltype(mask_c)::value;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = 2 * half + cc;
                        uint32_t us[32], ud[32];
                        tmem_ld32(tmem + lane_off + L::S_COL + c * 32, us);
                        tmem_ld32(tmem + lane_off + L::DP_COL + c * 32, ud);
                        tmem_wait_ld_dep(us);
                        tmem_wait_ld_dep(ud);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int key = key0 + c * 32 + e;
                            float p0 = fast_exp2(__uint_as_float(us[e]) * p.scale_log2 - lse);
                            float p1 = fast_exp2(__uint_as_float(us[e + 1]) * p.scale_log2 - lse);
                            if (MASK) {
                                p0 = valid && key >= lo && key <= hi ? p0 : 0.f;
                                p1 = valid && key + 1 >= lo && key + 1 <= hi ? p1 : 0.f;
                            }
                            const float d0 = p0 * (__uint_as_float(ud[e]) - dd);
                            const float d1 = p1 * (__uint_as_float(ud[e + 1]) - dd);
                            pk[cc][e / 2] = CORE ? pack_f16x2(d0, d1) : pack_bf16x2(d0, d1);
                        }
                    }
                };
                const int k_first = key0 + 64 * half;
                const bool full =
                    __all_sync(0xffffffffu, valid && k_first >= lo && k_first + 63 <= hi);
                if (core) {
                    if (full)
                        elementwise(std::true_type{}, std::false_type{});
                    else
                        elementwise(std::true_type{}, std::true_type{});
                } else {
                    if (full)
                        elementwise(std::false_type{}, std::false_type{});
                    else
                        elementwise(std::false_type{}, std::true_type{});
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_free);
                // the previous tile's dQ product has read dS
                if (it > 0) {
                    if (!(ok = bw_warp_wait(&bars->mm_done, (it - 1) & 1, bars))) break;
                    tc_fence_after_sync();
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    tmem_st16(tmem + lane_off + L::DS_COL + (2 * half + cc) * 16, pk[cc]);
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full);
            }
            if (!ok) break;
            // epilogue: dQ = (sum dS K) / sqrt(d)
            if (!(ok = bw_warp_wait(&bars->mm_done, (it - 1) & 1, bars))) break;
            tc_fence_after_sync();
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                const int c = half * (D / 64) + cc;
                uint32_t u[32];
                tmem_ld32_wait(tmem + lane_off + L::DQ_COL + c * 32, u);
                if (valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_global_x8(p.dQ + qrow * D + c * 32 + 8 * q, u + 8 * q, p.scale);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kDqTmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// 3. dK, dV (raw) and dKc, dVc (core) --------------------------------------
//
// Work item: one 128-key tile of one (batch, kv head) and a range of query
// tiles, for all r query heads of the kv head.  Core tiles come first, their
// query range (every later query sees a core key) cut into chunks of
// kCoreChunk tiles whose results are added into fp32 dKc, dVc; raw tiles
// take every query tile that sees one of their keys and store dK, dV.
// Each (key tile, query tile) pair runs as two 64-query halves h, so that
// the element-wise step of one half overlaps the MMAs of the other:
// warps 4h .. 4h+3 take half h (one key row per thread); warp 8: TMA
// producer; warp 9: issuer.  TMEM: S^T [0,128), half h in [64h, 64h+64),
// then that half's P^T over its first 32 columns; dP^T [128,256) the same
// way with dS^T; dK [256, 256+D); dV [256+D, 256+2D).
template <int D>
struct BkLayout {
    using T = Bt<D>;
    static constexpr int QST = 2;
    static constexpr int OFF_K = 0, OFF_V = T::TILE_BYTES;
    static constexpr int OFF_Q = 2 * T::TILE_BYTES;                 // QST stages
    static constexpr int OFF_O = OFF_Q + QST * T::TILE_BYTES;       // QST stages
    static constexpr int OFF_COL = OFF_O + QST * T::TILE_BYTES;     // per-column data
    static constexpr int OFF_BAR = OFF_COL + 2 * 128 * 8;
    static constexpr int SMEM = OFF_BAR + 512 + 1024;
    static constexpr uint32_t ST_COL = 0, DPT_COL = 128, DK_COL = 256, DV_COL = 256 + D;
};

constexpr int kDkvSoftWarps = 8;
constexpr int kDkvTmaWarp = 8, kDkvMmaWarp = 9;
constexpr int kDkvThreads = 320;

struct KGeom {
    bool core;
    int b, h, kt;   // key tile (raw: rows 128 kt..; core: groups 128 kt..)
    int qa, qb;     // query tiles [qa, qb)
};

// First query tile with a query that attends to core group j: query t sees
// group j iff j < ws(t) / g, i.e. t >= (j + 1) g + w.
__device__ __forceinline__ int core_first_qt(int j, const BwParams &p)
{
    return static_cast<int>((static_cast<int64_t>(j + 1) * p.g + p.w) / 128);
}

__device__ __forceinline__ KGeom k_geom(int item, const BwParams &p)
{
    KGeom G;
    const int pairs = p.B * p.Hkv;
    if (item < p.n_core_items) {
        int u = item;
        for (int ct = 0; ct < p.n_ct; ++ct) {
            const int qs = core_first_qt(ct * 128, p);
            const int nch = qs < p.n_qt ? (p.n_qt - qs + kCoreChunk - 1) / kCoreChunk : 0;
            if (u < nch * pairs) {
                const int chunk = u / pairs, pair = u - chunk * pairs;
                G.core = true;
                G.b = pair / p.Hkv;
                G.h = pair - G.b * p.Hkv;
                G.kt = ct;
                G.qa = qs + chunk * kCoreChunk;
                G.qb = min(G.qa + kCoreChunk, p.n_qt);
                return G;
            }
            u -= nch * pairs;
        }
    }
    const int u = item - p.n_core_items;
    const int kt = u / pairs, pair = u - kt * pairs;
    G.core = false;
    G.b = pair / p.Hkv;
    G.h = pair - G.b * p.Hkv;
    G.kt = kt;
    // key k is seen by queries k .. (floor(k / g) + 1) g + w - 1
    const int klast = min(kt * 128 + 127, p.T - 1);
    const int tmax = min((klast / p.g + 1) * p.g + p.w - 1, p.T - 1);
    G.qa = kt;
    G.qb = tmax / 128 + 1;
    return G;
}

template <int D>
__global__ void __launch_bounds__(kDkvThreads, 1)
    bw_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmO16,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                  const BwParams p)
{
    using L = BkLayout<D>;
    using T = Bt<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + L::OFF_K, *sV = smem + L::OFF_V;
    uint8_t *sQ = smem + L::OFF_Q, *sO = smem + L::OFF_O;
    // [2][128] (lse, D) of the current query tile's columns
    const uint32_t col_s = smem_addr(smem + L::OFF_COL);
    BwBars *bars = reinterpret_cast<BwBars *>(smem + L::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = p.n_items;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::QST; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->kv_empty, 1);
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars->hs_full[h], 1);
            mbar_init(&bars->hp_full[h], 4);
            mbar_init(&bars->hmm_done[h], 1);
        }
        mbar_init(&bars->acc_empty, kDkvSoftWarps);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->never = 0;
        mbar_fence_init();
    }
    if (warp == kDkvTmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    if (warp == kDkvTmaWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t qc = 0, kvc = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const KGeom G = k_geom(item, p);
                const int z = G.b * p.Hkv + G.h;
                if (kvc > 0 && !(ok = bw_lane_wait(&bars->kv_empty, (kvc - 1) & 1, bars))) break;
                mbar_arrive_expect_tx(&bars->kv_full, 2 * T::TILE_BYTES);
                for (int bx = 0; bx < T::NBOX; ++bx) {
                    tma_load_3d(sK + bx * T::BOX_BYTES, G.core ? &tmKc : &tmK, &bars->kv_full,
                                bx * 64, G.kt * 128, z);
                    tma_load_3d(sV + bx * T::BOX_BYTES, G.core ? &tmVc : &tmV, &bars->kv_full,
                                bx * 64, G.kt * 128, z);
                }
                ++kvc;
                for (int kh = 0; ok && kh < p.r; ++kh) {
                    const int zq = G.b * p.Hq + G.h * p.r + kh;
                    for (int qt = G.qa; qt < G.qb; ++qt) {
                        const int s = qc % L::QST;
                        if (!(ok = bw_lane_wait(&bars->q_empty[s], ((qc / L::QST) & 1) ^ 1, bars)))
                            break;
                        mbar_arrive_expect_tx(&bars->q_full[s], 2 * T::TILE_BYTES);
                        for (int bx = 0; bx < T::NBOX; ++bx) {
                            tma_load_3d(sQ + s * T::TILE_BYTES + bx * T::BOX_BYTES,
                                        G.core ? &tmQ16 : &tmQ, &bars->q_full[s], bx * 64,
                                        qt * 128, zq);
                            tma_load_3d(sO + s * T::TILE_BYTES + bx * T::BOX_BYTES,
                                        G.core ? &tmO16 : &tmO, &bars->q_full[s], bx * 64,
                                        qt * 128, zq);
                        }
                        ++qc;
                    }
                }
            }
            const volatile int *never = &bars->never;
            for (uint32_t s = 0; s < L::QST && s < qc; ++s) {
                const uint32_t last = qc - 1 - ((qc - 1 - s) % L::QST);
                wait_bounded(&bars->q_full[last % L::QST], (last / L::QST) & 1, never, kBwWaitNs);
            }
            if (kvc > 0) wait_bounded(&bars->kv_full, (kvc - 1) & 1, never, kBwWaitNs);
        }
    } else if (warp == kDkvMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s_bf = idesc_f32acc(128, 64, true, false, false);
            constexpr uint32_t id_s_h = idesc_f32acc(128, 64, false, false, false);
            constexpr uint32_t id_a_bf = idesc_f32acc(128, D, true, false, true);
            constexpr uint32_t id_a_h = idesc_f32acc(128, D, false, false, true);
            const uint64_t dk = smem_desc_sw128(smem_addr(sK), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_addr(sV), 16, 1024);
            const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
            const uint64_t dqm = smem_desc_sw128(smem_addr(sQ), T::BOX_BYTES, 1024);
            const uint64_t dO = smem_desc_sw128(smem_addr(sO), 16, 1024);
            const uint64_t dOm = smem_desc_sw128(smem_addr(sO), T::BOX_BYTES, 1024);
            constexpr uint32_t kTile16 = T::TILE_BYTES >> 4;
            constexpr uint32_t kHalf16 = (64 * 128) >> 4;  // 64 rows of a swizzled box
            // Per half h of tile n (tiles numbered over this CTA's items, Q
            // stage n % QST): A(h, n) issues S^T, dP^T; B(h, n) issues
            // dV += P^T dO, dK += dS^T Q.  Order within an item:
            //   A(0,0) A(1,0) | B(0,n) A(0,n+1) B(1,n) A(1,n+1) | ...
            // so each half runs its own chain and the halves overlap.  A(h,
            // n+1) waits until B(h, n) has read the half's P^T, dS^T.  No
            // look-ahead across items: the next item's K, V tiles reuse the
            // one key-side buffer.
            uint32_t kvc = 0, base = 0;
            int k = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++k) {
                const KGeom G = k_geom(item, p);
                const uint32_t ids = G.core ? id_s_h : id_s_bf, ida = G.core ? id_a_h : id_a_bf;
                auto issue_a = [&](int h, uint32_t n) -> bool {
                    if (n > 0 && !bw_lane_wait(&bars->hmm_done[h], (n - 1) & 1, bars)) return false;
                    tc_fence_after_sync();
                    const uint32_t s = n % L::QST;
                    mma_kk<D>(tmem + L::ST_COL + 64 * h, dk, dq + s * kTile16 + h * kHalf16, ids);
                    mma_kk<D>(tmem + L::DPT_COL + 64 * h, dv, dO + s * kTile16 + h * kHalf16, ids);
                    mma_commit(&bars->hs_full[h]);
                    return true;
                };
                auto issue_b = [&](int h, uint32_t n, bool first_tile) -> bool {
                    if (!bw_lane_wait(&bars->hp_full[h], n & 1, bars)) return false;
                    if (h == 0 && first_tile && k > 0 &&
                        !bw_lane_wait(&bars->acc_empty, (k - 1) & 1, bars))
                        return false;
                    tc_fence_after_sync();
                    const uint32_t s = n % L::QST;
                    const bool first = first_tile && h == 0;
                    mma_tm64(tmem + L::DV_COL, tmem + L::ST_COL + 64 * h,
                             dOm + s * kTile16 + h * 512, ida, first);
                    mma_tm64(tmem + L::DK_COL, tmem + L::DPT_COL + 64 * h,
                             dqm + s * kTile16 + h * 512, ida, first);
                    mma_commit(&bars->hmm_done[h]);
                    return true;
                };
                auto q_ready = [&](uint32_t n) {
                    return bw_lane_wait(&bars->q_full[n % L::QST], (n / L::QST) & 1, bars);
                };
                if (!(ok = bw_lane_wait(&bars->kv_full, kvc & 1, bars))) break;
                ++kvc;
                const int n_tiles = p.r * (G.qb - G.qa);
                if (!(ok = q_ready(base) && issue_a(0, base) && issue_a(1, base))) break;
                for (int i = 0; ok && i < n_tiles; ++i) {
                    const uint32_t n = base + i;
                    const bool more = i + 1 < n_tiles;
                    if (!(ok = issue_b(0, n, i == 0))) break;
                    if (more && !(ok = q_ready(n + 1) && issue_a(0, n + 1))) break;
                    if (!(ok = issue_b(1, n, i == 0))) break;
                    mma_commit(&bars->q_empty[n % L::QST]);
                    if (more && !(ok = issue_a(1, n + 1))) break;
                }
                if (!ok) break;
                base += n_tiles;
                mma_commit(&bars->kv_empty);
            }
            mma_commit(&bars->drain);
            wait_bounded(&bars->drain, 0, &bars->never, kBwWaitNs);
        }
    } else {
        // ------------------------------------------------ P^T, dS^T warps
        const int row = threadIdx.x & 127;
        const int half = warp >> 2;  // query columns [64 half, 64 half + 64)
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const KGeom G = k_geom(item, p);
            const int key = G.kt * 128 + row;  // raw key, or core group
            const bool kvalid = G.core ? key < p.m : key < p.T;
            const int n_tiles = p.r * (G.qb - G.qa);
            // the queries that see this key form one range [t_lo, t_hi]: a
            // raw key k is seen by t = k .. (floor(k / g) + 1) g + w - 1
            // (its window start ws(t) <= k), core group j by every
            // t >= (j + 1) g + w (j < ws(t) / g)
            int t_lo, t_hi;
            if (!kvalid) {
                t_lo = 1;
                t_hi = 0;
            } else if (G.core) {
                t_lo = (key + 1) * p.g + p.w;
                t_hi = p.T - 1;
            } else {
                t_lo = key;
                t_hi = min((key / p.g + 1) * p.g + p.w - 1, p.T - 1);
            }
            for (int i = 0; i < n_tiles; ++i, ++it) {
                const int kh = i / (G.qb - G.qa), qt = G.qa + (i - kh * (G.qb - G.qa));
                const int hq = G.h * p.r + kh;
                // per-column (log-sum-exp, D) of this half's 64 query
                // columns, staged in shared memory (double-buffered by tile)
                const uint32_t cb = col_s + (it & 1) * 128 * 8;
                if (row < 64) {
                    const int col = 64 * half + row;
                    const int t = qt * 128 + col;
                    const int64_t qrow = (static_cast<int64_t>(G.b) * p.Hq + hq) * p.T + t;
                    const bool tv = t < p.T;
                    const float lv = tv ? p.lse[qrow] : 0.f, dv_ = tv ? p.Dv[qrow] : 0.f;
                    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(cb + col * 8), "f"(lv),
                                 "f"(dv_)
                                 : "memory");
                }
                asm volatile("bar.sync %0, 128;" ::"r"(1 + half) : "memory");
                // this key's visible columns of the tile
                const int c_lo = max(t_lo - qt * 128, 0), c_hi = min(t_hi - qt * 128, 127);
                if (!(ok = bw_warp_wait(&bars->hs_full[half], it & 1, bars))) break;
                tc_fence_after_sync();
                // CORE: fp16 P, dS (core tiles) or bf16; MASK: test each
                // column against [c_lo, c_hi], skipped when every column of
                // this half is visible to every key row of the warp
                auto elementwise = [&](auto core_c, auto mask_c) {
                    constexpr bool CORE = decltype(core_c)::value;
                    constexpr bool MASK = decltype(mask_c)::value;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int c = 2 * half + h2;  // 32-column chunk of the tile
                        uint32_t us[32], ud[32], pp[16], pd[16];
                        tmem_ld32(tmem + lane_off + L::ST_COL + c * 32, us);
                        tmem_ld32(tmem + lane_off + L::DPT_COL + c * 32, ud);
                        tmem_wait_ld_dep(us);
                        tmem_wait_ld_dep(ud);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int cc = c * 32 + e;
                            float4 ld;  // (lse, D) of columns cc and cc + 1
                            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                         : "=f"(ld.x), "=f"(ld.y), "=f"(ld.z), "=f"(ld.w)
                                         : "r"(cb + cc * 8));
                            float p0 = fast_exp2(__uint_as_float(us[e]) * p.scale_log2 - ld.x);
                            float p1 = fast_exp2(__uint_as_float(us[e + 1]) * p.scale_log2 - ld.z);
                            if (MASK) {
                                p0 = cc >= c_lo && cc <= c_hi ? p0 : 0.f;
                                p1 = cc + 1 >= c_lo && cc + 1 <= c_hi ? p1 : 0.f;
                            }
                            const float d0 = p0 * (__uint_as_float(ud[e]) - ld.y);
                            const float d1 = p1 * (__uint_as_float(ud[e + 1]) - ld.w);
                            pp[e / 2] = CORE ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
                            pd[e / 2] = CORE ? pack_f16x2(d0, d1) : pack_bf16x2(d0, d1);
                        }
                        // over columns of this half this thread has already read
                        tmem_st16(tmem + lane_off + L::ST_COL + 64 * half + h2 * 16, pp);
                        tmem_st16(tmem + lane_off + L::DPT_COL + 64 * half + h2 * 16, pd);
                    }
                };
                const bool full =
                    __all_sync(0xffffffffu, c_lo <= 64 * half && c_hi >= 64 * half + 63);
                if (G.core) {
                    if (full)
                        elementwise(std::true_type{}, std::false_type{});
                    else
                        elementwise(std::true_type{}, std::true_type{});
                } else {
                    if (full)
                        elementwise(std::false_type{}, std::false_type{});
                    else
                        elementwise(std::false_type{}, std::true_type{});
                }
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->hp_full[half]);
            }
            if (!ok) break;
            // epilogue: dK = (sum dS^T Q) / sqrt(d), dV = sum P^T dO
            // The last tile's products.  A parity wait is sound only when
            // the phase before the awaited one is known to be complete.
            // Half 0's first: each group has seen the last tile's S^T of its
            // own half issued, A(1, last) follows A(0, last), and A(0, last)
            // is issued only once half 0's phase last - 1 is complete.
            // Then half 1's: B(0, last) follows B(1, last - 1), so its
            // completion implies half 1's phase last - 1.
            if (!(ok = bw_warp_wait(&bars->hmm_done[0], (it - 1) & 1, bars))) break;
            if (!(ok = bw_warp_wait(&bars->hmm_done[1], (it - 1) & 1, bars))) break;
            tc_fence_after_sync();
            const int64_t krow = (static_cast<int64_t>(G.b) * p.Hkv + G.h) * (G.core ? p.m : p.T) + key;
            float *dKo = (G.core ? p.dKc : p.dK) + krow * D;
            float *dVo = (G.core ? p.dVc : p.dV) + krow * D;
#pragma unroll
            for (int h2 = 0; h2 < D / 64; ++h2) {
                const int c = half * (D / 64) + h2;
                uint32_t uk[32], uv[32];
                tmem_ld32_wait(tmem + lane_off + L::DK_COL + c * 32, uk);
                tmem_ld32_wait(tmem + lane_off + L::DV_COL + c * 32, uv);
                if (!kvalid) continue;
                if (G.core) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        red_add_v4(dKo + c * 32 + 4 * q, __uint_as_float(uk[4 * q]) * p.scale,
                                   __uint_as_float(uk[4 * q + 1]) * p.scale,
                                   __uint_as_float(uk[4 * q + 2]) * p.scale,
                                   __uint_as_float(uk[4 * q + 3]) * p.scale);
                        red_add_v4(dVo + c * 32 + 4 * q, __uint_as_float(uv[4 * q]),
                                   __uint_as_float(uv[4 * q + 1]), __uint_as_float(uv[4 * q + 2]),
                                   __uint_as_float(uv[4 * q + 3]));
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        st_global_x8(dKo + c * 32 + 8 * q, uk + 8 * q, p.scale);
                        st_global_x8(dVo + c * 32 + 8 * q, uv + 8 * q, 1.0f);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kDkvTmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// 4. The pooling's chain rule ------------------------------------------------
//
// One warp per (batch, kv head, group j), lane l owning dims l*DPL ..: with
// the group's keys Kg, values Vg, the r scoring queries q_k (token jg+g-1)
// and softmax vectors s_k = softmax(Kg q_k / sqrt(d)), a = mean_k s_k:
//   dK_g += a dKc,  dV_g += a dVc,  da = Kg dKc + Vg dVc,
//   per head k: dz = s_k (da/r - s_k . da/r),
//   dq_k += (sum_i dz_i Kg_i) / sqrt(d),  dK_g += dz q_k / sqrt(d).
// Three passes over the group: scores and da (K, V rows read once from
// DRAM, 8 rows in flight), one read-modify-write of each dK, dV row, then
// dq per head (key rows again, now from L1).
template <int D>
struct BwVec;
template <>
struct BwVec<128> {
    using H = uint2;   // 4 bf16
    using F = float4;  // 4 fp32
    static __device__ __forceinline__ void h2f(H v, float (&f)[4])
    {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    }
    static __device__ __forceinline__ void ld(const float *p, float (&f)[4])
    {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&f)[4])
    {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};
template <>
struct BwVec<64> {
    using H = uint32_t;  // 2 bf16
    using F = float2;
    static __device__ __forceinline__ void h2f(H v, float (&f)[2])
    {
        f[0] = bf16_lo(v); f[1] = bf16_hi(v);
    }
    static __device__ __forceinline__ void ld(const float *p, float (&f)[2])
    {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        f[0] = v.x; f[1] = v.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&f)[2])
    {
        *reinterpret_cast<float2 *>(p) = make_float2(f[0], f[1]);
    }
};

template <int D>
__global__ void bw_pool_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                               const uint16_t *__restrict__ V, const BwParams p)
{
    constexpr int DPL = D / 32;
    using W = BwVec<D>;
    using H = typename W::H;
    extern __shared__ float pool_bw_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarp = blockDim.x >> 5;
    const int r = p.r, g = p.g;
    float *sc = pool_bw_smem + warp * (r + 2) * g;  // [r][g] softmax, then dz
    float *da = sc + r * g;                         // [g]
    float *aw = da + g;                             // [g] pooling weights
    const float inv_r = 1.0f / static_cast<float>(r);
    const int64_t n_groups = static_cast<int64_t>(p.B) * p.Hkv * p.m;
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * nwarp + warp; gid < n_groups;
         gid += static_cast<int64_t>(gridDim.x) * nwarp) {
        const int64_t pair = gid / p.m, j = gid - pair * p.m;
        const int64_t b = pair / p.Hkv, h = pair - b * p.Hkv;
        const int64_t row0 = pair * p.T + j * g;  // first key row of the group
        const int64_t last = j * g + g - 1;
        const int64_t lo = lane * DPL;
        auto qrow = [&](int k) { return ((b * p.Hq + h * r + k) * p.T + last) * D; };
        float dkc[DPL], dvc[DPL];
        W::ld(p.dKc + (pair * p.m + j) * D + lo, dkc);
        W::ld(p.dVc + (pair * p.m + j) * D + lo, dvc);
        // pass 1: logits of every head, da_i = (K_i . dKc + V_i . dVc) / r
        for (int i0 = 0; i0 < g; i0 += 8) {
            H kv[8], vv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (i0 + u < g) {
                    kv[u] = *reinterpret_cast<const H *>(K + (row0 + i0 + u) * D + lo);
                    vv[u] = *reinterpret_cast<const H *>(V + (row0 + i0 + u) * D + lo);
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (i0 + u < g) {
                    float kf[DPL], vf[DPL];
                    W::h2f(kv[u], kf);
                    W::h2f(vv[u], vf);
                    float t = 0.f;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) t = fmaf(kf[e], dkc[e], fmaf(vf[e], dvc[e], t));
                    t = warp_sum(t);
                    if (lane == 0) da[i0 + u] = t * inv_r;
                }
            }
            for (int k = 0; k < r; ++k) {
                float qf[DPL];
                W::h2f(*reinterpret_cast<const H *>(Q + qrow(k) + lo), qf);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (i0 + u < g) {
                        float kf[DPL];
                        W::h2f(kv[u], kf);
                        float t = 0.f;
#pragma unroll
                        for (int e = 0; e < DPL; ++e) t = fmaf(qf[e], kf[e], t);
                        t = warp_sum(t);
                        if (lane == 0) sc[k * g + i0 + u] = t * p.scale_log2;
                    }
                }
            }
        }
        __syncwarp();
        // softmax per head, weights a = mean over heads, then dz in place
        for (int i = lane; i < g; i += 32) aw[i] = 0.f;
        __syncwarp();
        for (int k = 0; k < r; ++k) {
            float mx = -INFINITY;
            for (int i = lane; i < g; i += 32) mx = fmaxf(mx, sc[k * g + i]);
            mx = warp_max(mx);
            float sum = 0.f;
            for (int i = lane; i < g; i += 32) {
                const float e = exp2f(sc[k * g + i] - mx);
                sc[k * g + i] = e;
                sum += e;
            }
            sum = warp_sum(sum);
            const float inv = 1.0f / sum;
            float sd = 0.f;
            for (int i = lane; i < g; i += 32) {
                const float sv = sc[k * g + i] * inv;
                sc[k * g + i] = sv;
                aw[i] += sv * inv_r;
                sd += sv * da[i];
            }
            sd = warp_sum(sd);
            for (int i = lane; i < g; i += 32) sc[k * g + i] *= da[i] - sd;  // dz
            __syncwarp();
        }
        // pass 2: dK_i += a_i dKc + (sum_k dz_ki q_k) / sqrt(d), dV_i += a_i dVc;
        // four rows' loads in flight before any of them is updated
        constexpr int RB = 4;
        for (int i0 = 0; i0 < g; i0 += RB) {
            float dk[RB][DPL], dv[RB][DPL];
#pragma unroll
            for (int u = 0; u < RB; ++u) {
                if (i0 + u < g) {
                    W::ld(p.dK + (row0 + i0 + u) * D + lo, dk[u]);
                    W::ld(p.dV + (row0 + i0 + u) * D + lo, dv[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < RB; ++u) {
                if (i0 + u < g) {
                    const float a = aw[i0 + u];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) {
                        dk[u][e] = fmaf(a, dkc[e], dk[u][e]);
                        dv[u][e] = fmaf(a, dvc[e], dv[u][e]);
                    }
                }
            }
            for (int k = 0; k < r; ++k) {
                float qf[DPL];
                W::h2f(*reinterpret_cast<const H *>(Q + qrow(k) + lo), qf);
#pragma unroll
                for (int u = 0; u < RB; ++u) {
                    if (i0 + u < g) {
                        const float c = sc[k * g + i0 + u] * p.scale;
#pragma unroll
                        for (int e = 0; e < DPL; ++e) dk[u][e] = fmaf(c, qf[e], dk[u][e]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < RB; ++u) {
                if (i0 + u < g) {
                    W::st(p.dK + (row0 + i0 + u) * D + lo, dk[u]);
                    W::st(p.dV + (row0 + i0 + u) * D + lo, dv[u]);
                }
            }
        }
        // pass 3: dq_k += (sum_i dz_ki K_i) / sqrt(d)
        for (int k = 0; k < r; ++k) {
            float dq[DPL];
#pragma unroll
            for (int e = 0; e < DPL; ++e) dq[e] = 0.f;
            for (int i = 0; i < g; ++i) {
                float kf[DPL];
                W::h2f(*reinterpret_cast<const H *>(K + (row0 + i) * D + lo), kf);
                const float c = sc[k * g + i];
#pragma unroll
                for (int e = 0; e < DPL; ++e) dq[e] = fmaf(c, kf[e], dq[e]);
            }
            float *dqr = p.dQ + qrow(k) + lo;
            float cur[DPL];
            W::ld(dqr, cur);
#pragma unroll
            for (int e = 0; e < DPL; ++e) cur[e] = fmaf(dq[e], p.scale, cur[e]);
            W::st(dqr, cur);
        }
        __syncwarp();
    }
}

template <int D>
cudaError_t launch_bw(const void *Q, const void *K, const void *V, const void *Kc,
                      const void *Vc, const void *O, bool o_f32, const float *lse,
                      const void *dO, float *dQ, float *dK, float *dV, int B, int Hq, int Hkv,
                      int64_t T, int g, int w, void *workspace, cudaStream_t s)
{
    const int64_t m = T / g;
    const int64_t rows = static_cast<int64_t>(B) * Hq * T;
    BwLayoutHost L = bw_layout(B, Hq, Hkv, T, D, g);
    char *ws = static_cast<char *>(workspace);
    uint16_t *Q16 = reinterpret_cast<uint16_t *>(ws + L.q16);
    uint16_t *dO16 = reinterpret_cast<uint16_t *>(ws + L.do16);
    float *Dv = reinterpret_cast<float *>(ws + L.dv);
    float *dKc = reinterpret_cast<float *>(ws + L.dkc);
    float *dVc = reinterpret_cast<float *>(ws + L.dvc);

    BwParams p;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.r = Hq / Hkv;
    p.T = static_cast<int>(T);
    p.g = g;
    p.w = w;
    p.m = static_cast<int>(m);
    p.scale = 1.0f / sqrtf(static_cast<float>(D));
    p.scale_log2 = kLog2e * p.scale;
    p.lse = lse;
    p.Dv = Dv;
    p.dQ = dQ;
    p.dK = dK;
    p.dV = dV;
    p.dKc = dKc;
    p.dVc = dVc;
    p.n_qt = static_cast<int>((T + 127) / 128);
    p.n_kt = p.n_qt;
    p.n_ct = static_cast<int>((m + 127) / 128);
    int core_items = 0;
    for (int ct = 0; ct < p.n_ct; ++ct) {
        const int qs = static_cast<int>((static_cast<int64_t>(ct * 128 + 1) * g + w) / 128);
        if (qs < p.n_qt) core_items += (p.n_qt - qs + kCoreChunk - 1) / kCoreChunk;
    }
    p.n_core_items = core_items * B * Hkv;
    p.n_items = p.n_core_items + p.n_kt * B * Hkv;

    cudaError_t e = cudaSuccess;
    if (m > 0) {
        e = cudaMemsetAsync(ws + L.dkc, 0, L.dvc + L.dvc_bytes - L.dkc, s);
        if (e != cudaSuccess) return e;
    }
    // 1. D and the fp16 copies
    {
        const int threads = 256;
        const int64_t want = (rows * 32 + threads - 1) / threads;
        const int blocks = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
        if (o_f32)
            bw_prep_kernel<D, true><<<blocks, threads, 0, s>>>(
                static_cast<const uint16_t *>(dO), O, static_cast<const uint16_t *>(Q), Dv, Q16,
                dO16, rows);
        else
            bw_prep_kernel<D, false><<<blocks, threads, 0, s>>>(
                static_cast<const uint16_t *>(dO), O, static_cast<const uint16_t *>(Q), Dv, Q16,
                dO16, rows);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    CUtensorMap mQ, mO, mQ16, mO16, mK, mV, mKc, mVc;
    const int64_t pq = static_cast<int64_t>(B) * Hq, pk = static_cast<int64_t>(B) * Hkv;
    bool ok = make_map(&mQ, Q, D, T, pq) && make_map(&mO, dO, D, T, pq) &&
              make_map(&mQ16, Q16, D, T, pq, true) && make_map(&mO16, dO16, D, T, pq, true) &&
              make_map(&mK, K, D, T, pk) && make_map(&mV, V, D, T, pk);
    if (m > 0)
        ok = ok && make_map(&mKc, Kc, D, m, pk, true) && make_map(&mVc, Vc, D, m, pk, true);
    else {
        mKc = mK;
        mVc = mV;
    }
    if (!ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // 2. dQ (attention part)
    {
        using LQ = BqLayout<D>;
        const int items = p.n_qt * B * Hq;
        const int grid = items < sms ? items : sms;
        if ((e = cudaFuncSetAttribute(bw_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      LQ::SMEM)) != cudaSuccess)
            return e;
        bw_dq_kernel<D><<<grid, kDqThreads, LQ::SMEM, s>>>(mQ, mO, mQ16, mO16, mK, mV, mKc, mVc,
                                                            p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 3. dK, dV and dKc, dVc
    {
        using LK = BkLayout<D>;
        const int grid = p.n_items < sms ? p.n_items : sms;
        if ((e = cudaFuncSetAttribute(bw_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      LK::SMEM)) != cudaSuccess)
            return e;
        bw_dkv_kernel<D><<<grid, kDkvThreads, LK::SMEM, s>>>(mQ, mO, mQ16, mO16, mK, mV, mKc,
                                                              mVc, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 4. the pooling
    if (m > 0) {
        // 8 warps per block, fewer when a warp's scratch is large (r, g)
        const size_t per_warp = sizeof(float) * (p.r + 2) * g;
        int warps = 8;
        while (warps > 1 && per_warp * warps > 200 * 1024) --warps;
        const size_t smem = per_warp * warps;
        const int64_t groups = static_cast<int64_t>(B) * Hkv * m;
        const int64_t want = (groups + warps - 1) / warps;
        const int blocks = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
        if (smem > 48 * 1024 &&
            (e = cudaFuncSetAttribute(bw_pool_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem))) != cudaSuccess)
            return e;
        bw_pool_kernel<D><<<blocks, warps * 32, smem, s>>>(
            static_cast<const uint16_t *>(Q), static_cast<const uint16_t *>(K),
            static_cast<const uint16_t *>(V), p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

BwLayoutHost bw_layout(int B, int Hq, int Hkv, int64_t T, int d, int g)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t qd = static_cast<size_t>(B) * Hq * T * d * 2;
    const size_t rows = static_cast<size_t>(B) * Hq * T * 4;
    const size_t core = static_cast<size_t>(B) * Hkv * (T / g) * d * 4;
    BwLayoutHost L;
    L.q16 = 0;
    L.do16 = L.q16 + up(qd);
    L.dv = L.do16 + up(qd);
    L.dkc = L.dv + up(rows);
    L.dvc = L.dkc + up(core);
    L.dvc_bytes = up(core);
    L.total = L.dvc + L.dvc_bytes;
    return L;
}

cudaError_t launch_backward(const void *Q, const void *K, const void *V, const void *Kc,
                            const void *Vc, const void *O, bool o_f32, const float *lse,
                            const void *dO, float *dQ, float *dK, float *dV, int B, int Hq,
                            int Hkv, int64_t T, int d, int g, int w, void *workspace,
                            cudaStream_t s)
{
    if (T == 0) return cudaSuccess;
    if (d == 128)
        return launch_bw<128>(Q, K, V, Kc, Vc, O, o_f32, lse, dO, dQ, dK, dV, B, Hq, Hkv, T, g,
                              w, workspace, s);
    return launch_bw<64>(Q, K, V, Kc, Vc, O, o_f32, lse, dO, dQ, dK, dV, B, Hq, Hkv, T, g, w,
                         workspace, s);
}

cudaError_t backward_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_backward_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_backward_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
