// Decode cache upkeep: filling the raw ring from a prefix, and appending one
// token (ring write, plus pooling of the group the token completes).
//
// The write-up (section 基于 Triton 的底层加速) states that the CCA kernel
// supports a KV cache for decoding; the cache here holds the core key/value
// of every completed group (slot j = group j) and the newest raw tokens in a
// ring (token p in slot p % tail_cap).  A group is pooled as soon as its
// last token arrives; that token's queries are the group's scoring queries
// (section 全局感知池化).  Core rows are fp16, raw rows bf16.
#include "internal.h"
#include "pool_warp.cuh"

namespace cca {

__device__ unsigned int g_append_status;  // kStatusRange, kStatusCapacity

namespace {

// One thread per 16-byte chunk of the copied rows.
__global__ void tail_fill_kernel(const uint4 *__restrict__ K,
                                 const uint4 *__restrict__ V,
                                 uint4 *__restrict__ k_tail,
                                 uint4 *__restrict__ v_tail, int64_t T,
                                 int64_t p0, int64_t tail_cap, int chunks_per_row,
                                 int64_t total)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         i < total; i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t n = T - p0;
        const int64_t c = i % chunks_per_row;
        const int64_t row = i / chunks_per_row;  // (bh, p - p0)
        const int64_t bh = row / n, p = p0 + (row - bh * n);
        const int64_t src = (bh * T + p) * chunks_per_row + c;
        const int64_t dst = (bh * tail_cap + p % tail_cap) * chunks_per_row + c;
        k_tail[dst] = K[src];
        v_tail[dst] = V[src];
    }
}

constexpr int kAppendWarps = 4;

// Append token t of pair bh = b * Hkv + h: its ring slot, and if it is the
// last token of group t / g, the pooling of that group into core slot t / g
// (the group's older tokens come from the ring, this one from the input
// rows).  One warp.
template <int D>
__device__ __forceinline__ void append_pair(
    const uint16_t *__restrict__ q_t, const uint16_t *__restrict__ k_t,
    const uint16_t *__restrict__ v_t, uint16_t *__restrict__ k_core,
    uint16_t *__restrict__ v_core, uint16_t *__restrict__ k_tail,
    uint16_t *__restrict__ v_tail, int Hq, int Hkv, int g, int64_t core_cap,
    int64_t tail_cap, int64_t t, int64_t bh, float scale_log2, float *scratch)
{
    const int lane = threadIdx.x & 31;
    const int r = Hq / Hkv;
    const int64_t b = bh / Hkv, h = bh - b * Hkv;
    using VT = typename RowVec<D>::T;
    const VT *kin = reinterpret_cast<const VT *>(k_t + bh * D);
    const VT *vin = reinterpret_cast<const VT *>(v_t + bh * D);
    const int64_t slot = t % tail_cap;
    reinterpret_cast<VT *>(k_tail + (bh * tail_cap + slot) * D)[lane] = kin[lane];
    reinterpret_cast<VT *>(v_tail + (bh * tail_cap + slot) * D)[lane] = vin[lane];
    if ((t + 1) % g != 0) return;
    const int64_t first = t - g + 1, j = t / g;
    const uint16_t *kt_base = k_tail + bh * tail_cap * D;
    const uint16_t *vt_base = v_tail + bh * tail_cap * D;
    const bool over = pool_group_warp<D>(
        [&](int i) {
            return i == g - 1 ? k_t + bh * D
                              : kt_base + ((first + i) % tail_cap) * D;
        },
        [&](int i) {
            return i == g - 1 ? v_t + bh * D
                              : vt_base + ((first + i) % tail_cap) * D;
        },
        [&](int k) { return q_t + (b * Hq + h * r + k) * D; }, r, g, scale_log2,
        scratch, k_core + (bh * core_cap + j) * D, v_core + (bh * core_cap + j) * D);
    if (over && lane == 0) atomicOr(&g_append_status, kStatusRange);
}

// One warp per (batch, key/value head); every row appends token t.
template <int D>
__global__ void __launch_bounds__(kAppendWarps * 32)
    append_kernel(const uint16_t *__restrict__ q_t,
                  const uint16_t *__restrict__ k_t,
                  const uint16_t *__restrict__ v_t, uint16_t *__restrict__ k_core,
                  uint16_t *__restrict__ v_core, uint16_t *__restrict__ k_tail,
                  uint16_t *__restrict__ v_tail, int B, int Hq, int Hkv, int g,
                  int64_t core_cap, int64_t tail_cap, int64_t t, float scale_log2)
{
    extern __shared__ float append_smem[];
    const int warp = threadIdx.x >> 5;
    const int64_t bh = static_cast<int64_t>(blockIdx.x) * kAppendWarps + warp;
    if (bh >= static_cast<int64_t>(B) * Hkv) return;
    const int r = Hq / Hkv;
    append_pair<D>(q_t, k_t, v_t, k_core, v_core, k_tail, v_tail, Hq, Hkv, g, core_cap,
                   tail_cap, t, bh, scale_log2, append_smem + warp * (r * g + g));
}

// One CTA per batch row b, one warp per key/value head; row b appends its
// token lens[b] and then advances lens[b] (device memory, so a captured
// CUDA graph can replay decode steps).  A row whose token would not fit the
// cache is left unchanged and reported (kStatusCapacity).
template <int D>
__global__ void append_rows_kernel(const uint16_t *__restrict__ q_t,
                                   const uint16_t *__restrict__ k_t,
                                   const uint16_t *__restrict__ v_t,
                                   uint16_t *__restrict__ k_core, uint16_t *__restrict__ v_core,
                                   uint16_t *__restrict__ k_tail, uint16_t *__restrict__ v_tail,
                                   long long *__restrict__ lens, int Hq, int Hkv, int g,
                                   int64_t core_cap, int64_t tail_cap, float scale_log2)
{
    extern __shared__ float append_smem[];
    __shared__ long long row_len;
    const int warp = threadIdx.x >> 5;
    const int64_t b = blockIdx.x;
    if (threadIdx.x == 0) row_len = lens[b];
    __syncthreads();
    const int64_t t = row_len;
    if (t < 0 || t / g >= core_cap) {
        if (threadIdx.x == 0) atomicOr(&g_append_status, kStatusCapacity);
        return;
    }
    const int r = Hq / Hkv;
    append_pair<D>(q_t, k_t, v_t, k_core, v_core, k_tail, v_tail, Hq, Hkv, g, core_cap,
                   tail_cap, t, b * Hkv + warp, scale_log2, append_smem + warp * (r * g + g));
    __syncthreads();  // every warp has read row_len before it moves on
    if (threadIdx.x == 0) lens[b] = t + 1;
}

}  // namespace

cudaError_t launch_tail_fill(const void *K, const void *V, void *k_tail,
                             void *v_tail, int B, int Hkv, int64_t T, int d,
                             int64_t p0, int64_t tail_cap, cudaStream_t s)
{
    const int cpr = d * 2 / 16;
    const int64_t total = static_cast<int64_t>(B) * Hkv * (T - p0) * cpr;
    if (total <= 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int blocks = static_cast<int>(want < 148LL * 32 ? want : 148LL * 32);
    tail_fill_kernel<<<blocks, threads, 0, s>>>(
        static_cast<const uint4 *>(K), static_cast<const uint4 *>(V),
        static_cast<uint4 *>(k_tail), static_cast<uint4 *>(v_tail), T, p0,
        tail_cap, cpr, total);
    return cudaGetLastError();
}

cudaError_t launch_append(const void *q_t, const void *k_t, const void *v_t,
                          void *k_core, void *v_core, void *k_tail,
                          void *v_tail, int B, int Hq, int Hkv, int d, int g,
                          int64_t core_cap, int64_t tail_cap, int64_t t,
                          cudaStream_t s)
{
    const int64_t pairs = static_cast<int64_t>(B) * Hkv;
    const int blocks = static_cast<int>((pairs + kAppendWarps - 1) / kAppendWarps);
    const int r = Hq / Hkv;
    const size_t smem = sizeof(float) * kAppendWarps * (r * g + g);
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    auto args = [&](auto kern) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        kern<<<blocks, kAppendWarps * 32, smem, s>>>(
            static_cast<const uint16_t *>(q_t), static_cast<const uint16_t *>(k_t),
            static_cast<const uint16_t *>(v_t), static_cast<uint16_t *>(k_core),
            static_cast<uint16_t *>(v_core), static_cast<uint16_t *>(k_tail),
            static_cast<uint16_t *>(v_tail), B, Hq, Hkv, g, core_cap, tail_cap, t,
            scale_log2);
    };
    if (d == 128)
        args(append_kernel<128>);
    else
        args(append_kernel<64>);
    return cudaGetLastError();
}

cudaError_t launch_append_rows(const void *q_t, const void *k_t, const void *v_t,
                               void *k_core, void *v_core, void *k_tail, void *v_tail,
                               long long *lens, int B, int Hq, int Hkv, int d, int g,
                               int64_t core_cap, int64_t tail_cap, cudaStream_t s)
{
    const int r = Hq / Hkv;
    const size_t smem = sizeof(float) * Hkv * (r * g + g);
    const float scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
    auto args = [&](auto kern) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        kern<<<B, Hkv * 32, smem, s>>>(
            static_cast<const uint16_t *>(q_t), static_cast<const uint16_t *>(k_t),
            static_cast<const uint16_t *>(v_t), static_cast<uint16_t *>(k_core),
            static_cast<uint16_t *>(v_core), static_cast<uint16_t *>(k_tail),
            static_cast<uint16_t *>(v_tail), lens, Hq, Hkv, g, core_cap, tail_cap,
            scale_log2);
    };
    if (d == 128)
        args(append_rows_kernel<128>);
    else
        args(append_rows_kernel<64>);
    return cudaGetLastError();
}

size_t append_rows_smem_bytes(int Hq, int Hkv, int g)
{
    return sizeof(float) * Hkv * ((Hq / Hkv) * g + g);
}

cudaError_t append_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_append_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_append_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
