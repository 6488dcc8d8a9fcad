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
// Work item: a 256-row block of queries of one (batch, query head), split in
// two 128-row halves A and B that share every K/V tile.  Its key tiles are
// the local stream first (keys ws(t0) .. last row), then the core stream
// (pooled keys 0 .. ws(last row)/g - 1); rows mask the keys they do not see.
// Blocks are dealt round-robin to one persistent CTA per SM, latest blocks
// (most core tiles) first.
//
// CTA of 352 threads (168 registers a thread: registers are booked for warps
// in groups of four, so eleven warps count as twelve):
//   warps 0-3  softmax of half A, warps 4-7 softmax of half B: thread i owns
//              query row i of its half; copies its S row from tensor memory
//              into registers (which frees S for the next Q K^T), masks,
//              online softmax (fp32, exp2 on the MUFU unit, lazy rescale),
//              writes P into its half's P buffer, rescales O when its
//              reference max moved, and runs the epilogue O / l.  At the
//              switch from the local to the core stream each group turns its
//              half of the Q tile from bf16 into fp16 in place.
//   warp 8     TMA producer: the Q block, then per key tile one K and one V
//              tile into multi-stage shared-memory rings (128-byte swizzle).
//   warp 9     Q K^T issuer: ... S = Q_A K_j^T; S = Q_B K_j^T ...  (both
//              operands from shared memory).
//   warp 10    P V issuer: ... O_A += P_A V_j; O_B += P_B V_j ...  (P from
//              tensor memory).  An MMA-issuing thread stalls the tensor pipe
//              whenever it waits on a barrier, even one already complete;
//              with two issuers one keeps the pipe busy while the other
//              waits.
// Tensor memory: S [0,128) shared by the halves, P_A [128,192), P_B
// [192,256) (16-bit pairs), O_A [256, 256+D), O_B after.  One S buffer
// serves both halves because a half holds its S row in registers as soon as
// the MMA has written it; with separate P buffers the next tile's Q K^T then
// runs while the softmax of the current tile is still computing, so the
// tensor pipe is not left waiting on the exponentials.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tma_map.h"

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cca {

__device__ unsigned int g_prefill_status;  // kStatusTimeout | kStatusRange

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 15.0f;  // log2 units: P stays <= 2^15 (fp16 range)

template <int D>
struct Pf {
    static constexpr int NBOX = D / 64;          // 64-column swizzled boxes
    static constexpr int BOX_BYTES = 128 * 128;  // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;  // 128 rows x D
    static constexpr int KST = D == 128 ? 3 : 4;  // K ring stages
    static constexpr int VST = D == 128 ? 2 : 4;  // V ring stages
    static constexpr int OFF_Q = 0;               // Q halves A, B (bf16, then fp16)
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    static constexpr int SMEM = OFF_BAR + 512 + 1024;  // + barriers + align slack
    static constexpr uint32_t S_COL = 0;          // S, shared by the halves
    static constexpr uint32_t P_COL = 128;        // P of half h at 128 + h * 64
    static constexpr uint32_t O_COL = 256;        // O of half h at 256 + h * D
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 352;
};

struct Params {
    int B, Hq, Hkv, r;
    int T, g, w, m;
    int n_blocks, n_items;
    float scale_log2;
    void *O;
    int o_f32;
    float *lse;  // [B, Hq, T]: log2 of each row's softmax denominator (LSE instance)
};

__device__ __forceinline__ int ws_of(int t, int g, int w)
{
    const int lo = t > w ? t - w : 0;
    return (lo / g) * g;
}

// Geometry of one 256-row block.
struct Geom {
    int b, hq, h, t0, tlast;
    int ws_lo;                 // ws(t0): first local key
    int n_local, n_core_tiles, n_tiles;
};

// HM: head-major item order (all blocks of a head before the next head).
template <bool HM>
__device__ __forceinline__ Geom geom(int item, const Params &p)
{
    Geom G;
    const int bhq_count = p.B * p.Hq;
    // Latest blocks (most core tiles) first.  Across heads when the core
    // rows of all heads fit in L2, so that concurrent items have equal
    // costs; head by head when they do not, so that each head's core rows
    // are read from DRAM once (measured on B200 at 128K context: 4.2 GB of
    // DRAM reads instead of 15.6 GB, 4-5% faster; at 32K, 11% slower).
    int blk, bhq;
    if constexpr (HM) {
        bhq = item / p.n_blocks;
        blk = p.n_blocks - 1 - (item - bhq * p.n_blocks);
    } else {
        blk = p.n_blocks - 1 - item / bhq_count;
        bhq = item - (item / bhq_count) * bhq_count;
    }
    G.b = bhq / p.Hq;
    G.hq = bhq - G.b * p.Hq;
    G.h = G.hq / p.r;
    G.t0 = blk * 256;
    G.tlast = min(G.t0 + 255, p.T - 1);
    G.ws_lo = ws_of(G.t0, p.g, p.w);
    const int nc_hi = ws_of(G.tlast, p.g, p.w) / p.g;
    G.n_core_tiles = (nc_hi + 127) / 128;
    G.n_local = (G.tlast - G.ws_lo + 1 + 127) / 128;
    G.n_tiles = G.n_local + G.n_core_tiles;
    return G;
}

__device__ __forceinline__ bool tile_is_core(const Geom &G, int j) { return j >= G.n_local; }
__device__ __forceinline__ int tile_key0(const Geom &G, int j)
{
    return j >= G.n_local ? (j - G.n_local) * 128 : G.ws_lo + j * 128;
}

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t qh_full[2];
    uint64_t k_full[4], k_empty[4];
    uint64_t v_full[4], v_empty[4];
    uint64_t s_full[2];  // S holds half h's scores of its current tile
    uint64_t s_free[2];  // half h has read its S row into registers
    uint64_t p_full[2];
    uint64_t o_bar[2], o_empty[2];
    uint64_t mma_done, mma_done2;  // Q K^T issuer, P V issuer
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

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void load_chunk(uint32_t addr, float (&x)[32])
{
    uint32_t u[32];
    tmem_ld32_wait(addr, u);
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(u[e]);
}

// Softmax numerators of one 32-column chunk: p = 2^(x c - m) on the MUFU
// unit, packed to 16-bit pairs in pk (fp16 for core tiles, bf16 for raw
// ones).  For bf16 P (8 significant bits) the row sum adds exactly the
// rounded values P V will see, so that the rounding of a dominant weight
// cancels in O = (P V) / l; for fp16 P (11 bits) the fp32 values are summed.
template <bool F16>
__device__ __forceinline__ void exp_chunk(const float (&x)[32], float2 c2, float2 nm2,
                                          uint32_t (&pk)[16], float2 &acc)
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 y = __ffma2_rn(make_float2(x[2 * i], x[2 * i + 1]), c2, nm2);
        const float2 pv = make_float2(fast_exp2(y.x), fast_exp2(y.y));
        if (F16) {
            pk[i] = pack_f16x2(pv.x, pv.y);
            acc = __fadd2_rn(acc, pv);
        } else {
            pk[i] = pack_bf16x2(pv.x, pv.y);
            acc = __fadd2_rn(acc, make_float2(bf16_lo(pk[i]), bf16_hi(pk[i])));
        }
    }
}

__device__ __forceinline__ float row_max128(const float (&x)[128])
{
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmax3(x[16 * i], x[16 * i + 1], x[16 * i + 2]);
#pragma unroll
    for (int k = 3; k < 15; k += 2)
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = fmax3(m[i], x[16 * i + k], x[16 * i + k + 1]);
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], x[16 * i + 15]);
    return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// LSE: also write each row's log-sum-exp (log2 units: log2 of the sum of
// 2^(logit / ln 2) over the row's keys), which the backward kernels need;
// a separate instance, so that the inference kernel is unchanged.
// HM: item order (geom), a separate instance for the same reason.
template <int D, bool LSE, bool HM>
__global__ void __launch_bounds__(352, 1)
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
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < C::KST; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < C::VST; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars->qh_full[h], 4);
            mbar_init(&bars->s_full[h], 1);
            mbar_init(&bars->s_free[h], 4);
            mbar_init(&bars->p_full[h], 4);
            mbar_init(&bars->o_bar[h], 1);
            mbar_init(&bars->o_empty[h], 4);
        }
        mbar_init(&bars->mma_done, 1);
        mbar_init(&bars->mma_done2, 1);
        bars->abort = 0;
        bars->never = 0;
        mbar_fence_init();
    }
    if (warp == 8) {
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

    if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc = 0, vc = 0, qc = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                const Geom G = geom<HM>(item, p);
                if (qc > 0 && !(ok = lane_wait(&bars->q_empty, (qc - 1) & 1, bars))) break;
                mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE_BYTES);
                for (int hh = 0; hh < 2; ++hh)
                    for (int bx = 0; bx < C::NBOX; ++bx)
                        tma_load_3d(sQ + hh * C::TILE_BYTES + bx * C::BOX_BYTES, &tmQ,
                                    &bars->q_full, bx * 64, G.t0 + hh * 128,
                                    G.b * p.Hq + G.hq);
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
            // (the last fill of each ring stage, and the last Q block).
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
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------ tcgen05 issuers
        // Warp 9 issues S = Q K^T, warp 10 issues O += P V.  A thread that
        // issues MMAs stalls the tensor pipe while it waits on a barrier
        // (even a completed one); with two issuers one keeps the pipe busy
        // while the other waits.
        if (lane == 0) {
            constexpr uint32_t idesc_qk_bf = idesc_f32acc(128, 128, true, false, false);
            constexpr uint32_t idesc_qk_h = idesc_f32acc(128, 128, false, false, false);
            constexpr uint32_t idesc_pv_bf = idesc_f32acc(128, D, true, false, true);
            constexpr uint32_t idesc_pv_h = idesc_f32acc(128, D, false, false, true);
            // Shared-memory descriptors: the start-address field (bits
            // 0-13, 16-byte units) is advanced by plain addition.
            const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_addr(sK), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_addr(sV), C::BOX_BYTES, 1024);
            constexpr uint32_t kTile16 = C::TILE_BYTES >> 4;
            uint32_t it = 0;  // key tiles over all items
            int k = 0;
            bool ok = true;
            if (warp == 9) {
                uint32_t kc = 0, cq = 0;
                auto qk = [&](int hh, uint32_t s, bool core) {
                    const uint64_t a0 = dq + hh * kTile16, b0 = dk + s * kTile16;
                    const uint32_t idesc = core ? idesc_qk_h : idesc_qk_bf;
                    const uint32_t d_tmem = tmem + C::S_COL;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        constexpr uint32_t box16 = C::BOX_BYTES >> 4;
                        const uint32_t off = (kk >> 2) * box16 + (kk & 3) * 2;
                        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
                    }
                };
                for (int item = blockIdx.x; ok && item < p.n_items;
                     item += gridDim.x, ++k) {
                    const Geom G = geom<HM>(item, p);
                    if (!(ok = lane_wait(&bars->q_full, k & 1, bars))) break;
                    for (int j = 0; ok && j < G.n_tiles; ++j, ++it) {
                        const bool core = tile_is_core(G, j);
                        const uint32_t s = kc % C::KST;
                        if (!(ok = lane_wait(&bars->k_full[s], (kc / C::KST) & 1, bars))) break;
                        for (int hh = 0; hh < 2; ++hh) {
                            // S is free once its previous occupant has been
                            // read: half B's previous tile before S_A, half
                            // A's current tile before S_B.
                            if (hh == 1 || it > 0) {
                                const uint32_t prev = hh == 0 ? it - 1 : it;
                                if (!(ok = lane_wait(&bars->s_free[hh ^ 1], prev & 1, bars)))
                                    break;
                            }
                            if (core && j == G.n_local &&
                                !(ok = lane_wait(&bars->qh_full[hh], cq & 1, bars)))
                                break;
                            tc_fence_after_sync();
                            qk(hh, s, core);
                            mma_commit(&bars->s_full[hh]);
                        }
                        if (!ok) break;
                        mma_commit(&bars->k_empty[s]);
                        ++kc;
                        if (j == G.n_tiles - 1) mma_commit(&bars->q_empty);
                    }
                    if (G.n_core_tiles > 0) ++cq;
                }
                // Wait for every Q K^T this thread issued to finish.
                mma_commit(&bars->mma_done);
                wait_bounded(&bars->mma_done, 0, &bars->never, kWaitLimitNs);
            } else {
                uint32_t vc = 0;
                auto pv = [&](int hh, uint32_t sv, bool core, bool first) {
                    const uint64_t b0 = dv + sv * kTile16;
                    const uint32_t idesc = core ? idesc_pv_h : idesc_pv_bf;
                    const uint32_t d_tmem = tmem + C::O_COL + hh * D;
                    const uint32_t a_tmem = tmem + C::P_COL + hh * 64;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(d_tmem, a_tmem + kk * 8, b0 + kk * 128, idesc,
                               (first && kk == 0) ? 0u : 1u);
                };
                for (int item = blockIdx.x; ok && item < p.n_items;
                     item += gridDim.x, ++k) {
                    const Geom G = geom<HM>(item, p);
                    for (int j = 0; ok && j < G.n_tiles; ++j, ++it) {
                        const bool core = tile_is_core(G, j);
                        const uint32_t sv = vc % C::VST;
                        for (int hh = 0; hh < 2; ++hh) {
                            if (!(ok = lane_wait(&bars->p_full[hh], it & 1, bars))) break;
                            if (j == 0 && k > 0 &&
                                !(ok = lane_wait(&bars->o_empty[hh], (k - 1) & 1, bars)))
                                break;
                            if (hh == 0 &&
                                !(ok = lane_wait(&bars->v_full[sv], (vc / C::VST) & 1, bars)))
                                break;
                            tc_fence_after_sync();
                            pv(hh, sv, core, j == 0);
                            mma_commit(&bars->o_bar[hh]);
                        }
                        if (!ok) break;
                        mma_commit(&bars->v_empty[sv]);
                        ++vc;
                    }
                }
                // Wait for every P V this thread issued to finish.
                mma_commit(&bars->mma_done2);
                wait_bounded(&bars->mma_done2, 0, &bars->never, kWaitLimitNs);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------ softmax warps
        const int hh = warp >> 2;                  // half
        const int row = threadIdx.x & 127;         // tensor-memory lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + C::S_COL;
        const uint32_t p_addr = tmem + lane_off + C::P_COL + hh * 64;
        const uint32_t o_addr = tmem + lane_off + C::O_COL + hh * D;
        uint32_t it = 0;  // key tiles over all items
        bool ok = true;
        for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
            const Geom G = geom<HM>(item, p);
            const bool core_block = G.n_core_tiles > 0;
            const int t0h = G.t0 + hh * 128;       // first row of this half
            const int t = t0h + row;
            const int ws_t = ws_of(t, p.g, p.w);
            const int nc_t = ws_t / p.g;
            const int nc_lo = ws_of(t0h, p.g, p.w) / p.g;
            const int ws_hi = ws_of(t0h + 127, p.g, p.w);
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < G.n_tiles; ++j, ++it) {
                if (!(ok = warp_wait(&bars->s_full[hh], it & 1, bars))) break;
                tc_fence_after_sync();
                const bool core = tile_is_core(G, j);
                const int key0 = tile_key0(G, j);
                const bool need_mask = core ? (key0 + 128 > nc_lo)
                                            : (key0 < ws_hi || key0 + 127 > t0h);
                const int lo = core ? 0 : ws_t;
                const int hi = core ? nc_t - 1 : t;
                // The whole S row into registers; S is then free for the
                // other half's next Q K^T.
                float x[128];
                {
                    uint32_t u[128];
                    tmem_ld128_wait(s_addr, u);
#pragma unroll
                    for (int e = 0; e < 128; ++e) x[e] = __uint_as_float(u[e]);
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_free[hh]);
                if (need_mask) {
#pragma unroll
                    for (int e = 0; e < 128; ++e) {
                        const int key = key0 + e;
                        if (key < lo || key > hi) x[e] = -INFINITY;
                    }
                }
                const float m_tile = row_max128(x) * p.scale_log2;
                float alpha = 1.f;
                if (m_tile > m_run + kRescaleThreshold) {
                    alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_tile);
                    m_run = m_tile;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                // P = 2^(S c - m), packed.  P V of the previous tile (over
                // all items) must have read P_h and written O_h before
                // either is touched: the wait comes after three of the four
                // chunks, when that P V has almost always finished, and the
                // last chunk goes to tensor memory as soon as it is computed.
                // Measured on B200 at 128K context, waiting before the first
                // chunk is 7% slower, after the first 3% slower.
                const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
                const float2 nm2 = make_float2(-m_use, -m_use);
                float2 acc = make_float2(0.f, 0.f);
                uint32_t pk[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float xc[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) xc[e] = x[c * 32 + e];
                    if (core)
                        exp_chunk<true>(xc, c2, nm2, pk[c], acc);
                    else
                        exp_chunk<false>(xc, c2, nm2, pk[c], acc);
                    if (c == 2) {
                        if (it > 0) {
                            if (!(ok = warp_wait(&bars->o_bar[hh], (it - 1) & 1, bars))) break;
                            tc_fence_after_sync();
                        }
#pragma unroll
                        for (int q = 0; q < 3; ++q) tmem_st16(p_addr + q * 16, pk[q]);
                    } else if (c >= 3) {
                        tmem_st16(p_addr + c * 16, pk[c]);
                    }
                }
                if (!ok) break;
                l_run = fmaf(l_run, alpha, acc.x + acc.y);
                // the max moved (rare): rescale O before P V of this tile
                if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32_wait(o_addr + c * 32, u);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                        tmem_st32(o_addr + c * 32, u);
                    }
                }
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[hh]);
                if (core_block && j == G.n_local - 1) {
                    // Last local tile: its Q K^T, the last reader of the bf16
                    // Q half, is complete (its S was ready), so turn this
                    // half into fp16 in place for the core stream (16-byte
                    // chunks of 8 elements keep their swizzled places).  The
                    // first core Q K^T of the half waits for this.
                    bool over = false;
                    uint4 *q4 = reinterpret_cast<uint4 *>(sQ + hh * C::TILE_BYTES);
#pragma unroll 4
                    for (int c = row; c < C::TILE_BYTES / 16; c += 128) {
                        const uint4 v = q4[c];
                        uint4 h;
                        h.x = pack_f16x2(clamp_f16(bf16_lo(v.x), over), clamp_f16(bf16_hi(v.x), over));
                        h.y = pack_f16x2(clamp_f16(bf16_lo(v.y), over), clamp_f16(bf16_hi(v.y), over));
                        h.z = pack_f16x2(clamp_f16(bf16_lo(v.z), over), clamp_f16(bf16_hi(v.z), over));
                        h.w = pack_f16x2(clamp_f16(bf16_lo(v.w), over), clamp_f16(bf16_hi(v.w), over));
                        q4[c] = h;
                    }
                    if (over) atomicOr(&g_prefill_status, kStatusRange);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->qh_full[hh]);
                }
            }
            if (!ok) break;
            // Epilogue: O / l for this row, once P V of the item's last
            // tile (tile it - 1) is complete.
            if (!(ok = warp_wait(&bars->o_bar[hh], (it - 1) & 1, bars))) break;
            tc_fence_after_sync();
            // O / l for this row, 32 columns at a time; O is read completely
            // before its tensor memory is released
            const float inv = 1.0f / l_run;
            const int64_t orow = (static_cast<int64_t>(G.b) * p.Hq + G.hq) * p.T + t;
            const bool store = t < p.T;
            if (LSE && store) p.lse[orow] = (m_run == -INFINITY ? 0.f : m_run) + __log2f(l_run);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                load_chunk(o_addr + c * 32, o);
                if (c == D / 32 - 1) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->o_empty[hh]);
                }
                if (!store) continue;
                if (p.o_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.O) +
                                                             orow * D + c * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv,
                                             o[4 * q + 2] * inv, o[4 * q + 3] * inv);
                } else {
                    // 32-byte stores: each thread writes its own row, so a
                    // store fills whole sectors (measured on B200: 3-4%
                    // faster at 128K context than 16-byte stores)
                    uint16_t *dst = static_cast<uint16_t *>(p.O) + orow * D + c * 32;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[e] = pack_bf16x2(o[16 * q + 2 * e] * inv, o[16 * q + 2 * e + 1] * inv);
                        asm volatile(
                            "st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16 * q),
                            "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                            "r"(w[7])
                            : "memory");
                    }
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_d(const void *Q, const void *K, const void *V, const void *Kc,
                     const void *Vc, void *O, bool o_f32, int B, int Hq, int Hkv,
                     int64_t T, int g, int w, cudaStream_t s, float *lse)
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
    p.n_blocks = static_cast<int>((T + 255) / 256);
    p.n_items = p.n_blocks * B * Hq;
    p.scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
    p.O = O;
    p.o_f32 = o_f32 ? 1 : 0;
    p.lse = lse;
    int dev = 0, sms = 148, l2 = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    const int grid = p.n_items < sms ? p.n_items : sms;
    // head-major when the core keys and values of all heads (fp16) exceed
    // half the L2
    const bool hm = 4.0 * static_cast<double>(B) * Hkv * m * D > 0.5 * static_cast<double>(l2);
    auto kern = lse ? (hm ? prefill_kernel<D, true, true> : prefill_kernel<D, true, false>)
                    : (hm ? prefill_kernel<D, false, true> : prefill_kernel<D, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<grid, C::THREADS, C::SMEM, s>>>(mQ, mK, mV, mKc, mVc, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const void *Q, const void *K, const void *V,
                           const void *Kc, const void *Vc, void *O, bool o_f32,
                           int B, int Hq, int Hkv, int64_t T, int d, int g,
                           int w, cudaStream_t s, float *lse)
{
    if (T == 0) return cudaSuccess;
    if (d == 128) return launch_d<128>(Q, K, V, Kc, Vc, O, o_f32, B, Hq, Hkv, T, g, w, s, lse);
    return launch_d<64>(Q, K, V, Kc, Vc, O, o_f32, B, Hq, Hkv, T, g, w, s, lse);
}

cudaError_t prefill_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_prefill_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_prefill_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
