// cca_pool: globally-aware pooling of every complete group (section
// 全局感知池化 of the CCA write-up).  HBM-bound segmented softmax-GEMV: one
// warp per (batch, key/value head, group), coalesced row loads, warp-shuffle
// reductions, fp32 softmax and accumulation, fp16 core rows out.
#include "internal.h"
#include "pool_warp.cuh"

namespace cca {

__device__ unsigned int g_pool_status;  // kStatusRange: a core value was clamped

namespace {

constexpr int kPoolWarps = 8;  // warps per block

// G > 0: register-resident fast path for that group size; G == 0: any g.
template <int D, int G>
__global__ void __launch_bounds__(kPoolWarps * 32, 2)
    pool_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                const uint16_t *__restrict__ V, uint16_t *__restrict__ Kc,
                uint16_t *__restrict__ Vc, int Hq, int Hkv, int64_t T, int g,
                int64_t m, int64_t out_rows, int64_t n_groups,
                float scale_log2)
{
    extern __shared__ float pool_smem[];
    const int warp = threadIdx.x >> 5;
    const int r = Hq / Hkv;
    float *scratch = pool_smem + warp * (r * g + g);
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * kPoolWarps + warp;
         gid < n_groups;
         gid += static_cast<int64_t>(gridDim.x) * kPoolWarps) {
        const int64_t bh = gid / m, j = gid - bh * m;
        const int64_t b = bh / Hkv, h = bh - b * Hkv;
        const uint16_t *Kg = K + (bh * T + j * g) * D;
        const uint16_t *Vg = V + (bh * T + j * g) * D;
        const int64_t last = j * g + g - 1;
        const uint16_t *Qb = Q + ((b * Hq + h * r) * T + last) * D;
        auto krow = [&](int i) { return Kg + static_cast<int64_t>(i) * D; };
        auto vrow = [&](int i) { return Vg + static_cast<int64_t>(i) * D; };
        auto qrow = [&](int k) { return Qb + static_cast<int64_t>(k) * T * D; };
        bool over;
        if constexpr (G > 0)
            over = pool_group_warp_fast<D, G>(krow, vrow, qrow, r, scale_log2, scratch,
                                              Kc + (bh * out_rows + j) * D,
                                              Vc + (bh * out_rows + j) * D);
        else
            over = pool_group_warp<D>(krow, vrow, qrow, r, g, scale_log2, scratch,
                                      Kc + (bh * out_rows + j) * D,
                                      Vc + (bh * out_rows + j) * D);
        if (over && (threadIdx.x & 31) == 0) atomicOr(&g_pool_status, kStatusRange);
    }
}

}  // namespace

cudaError_t launch_pool(const void *Q, const void *K, const void *V, void *Kc,
                        void *Vc, int B, int Hq, int Hkv, int64_t T, int d,
                        int g, int64_t out_rows, cudaStream_t s)
{
    const int64_t m = T / g;
    const int64_t n_groups = static_cast<int64_t>(B) * Hkv * m;
    if (n_groups == 0) return cudaSuccess;
    const int r = Hq / Hkv;
    const size_t smem = sizeof(float) * kPoolWarps * (r * g + g);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n_groups + kPoolWarps - 1) / kPoolWarps;
    const int blocks = static_cast<int>(want < 64LL * sms ? want : 64LL * sms);
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
        kern<<<blocks, kPoolWarps * 32, smem, s>>>(q, k, v, kc, vc, Hq, Hkv, T, g, m,
                                                    out_rows, n_groups, scale_log2);
    };
    if (d == 128) {
        if (g == 16)
            go(pool_kernel<128, 16>);
        else if (g == 32)
            go(pool_kernel<128, 32>);
        else
            go(pool_kernel<128, 0>);
    } else {
        if (g == 16)
            go(pool_kernel<64, 16>);
        else if (g == 32)
            go(pool_kernel<64, 32>);
        else
            go(pool_kernel<64, 0>);
    }
    return cudaGetLastError();
}

cudaError_t pool_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_pool_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_pool_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca
