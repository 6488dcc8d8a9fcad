// Host-side launchers of the CUDA kernels, called by the C ABI in api.cu
// after it has checked every argument.  Each returns the launch's
// cudaError_t.
#pragma once

#include <cuda_runtime_api.h>

#include <cstddef>
#include <cstdint>

namespace cca {

// Globally-aware pooling of all complete groups of Q/K/V [B,H,T,d] (bf16)
// into Kc/Vc [B, Hkv, out_rows, d] (fp16; rows 0..floor(T/g)-1 written).
cudaError_t launch_pool(const void *Q, const void *K, const void *V, void *Kc,
                        void *Vc, int B, int Hq, int Hkv, int64_t T, int d,
                        int g, int64_t out_rows, cudaStream_t s);

// Copy raw tokens p in [p0, T) of K/V [B,Hkv,T,d] into ring slots
// p % tail_cap of k_tail/v_tail [B,Hkv,tail_cap,d].
cudaError_t launch_tail_fill(const void *K, const void *V, void *k_tail,
                             void *v_tail, int B, int Hkv, int64_t T, int d,
                             int64_t p0, int64_t tail_cap, cudaStream_t s);

// Append token t (ring write; pool group t/g when (t+1) % g == 0).
cudaError_t launch_append(const void *q_t, const void *k_t, const void *v_t,
                          void *k_core, void *v_core, void *k_tail,
                          void *v_tail, int B, int Hq, int Hkv, int d, int g,
                          int64_t core_cap, int64_t tail_cap, int64_t t,
                          cudaStream_t s);

// Split-K decode over the cache for token t, then the merge.
struct DecodePlan {
    int64_t n_keys;   // keys of token t: core + raw
    int64_t n_core;   // core keys
    int64_t ws;       // window start
    int chunk;        // keys per split
    int nsplit;       // number of splits
};
DecodePlan decode_plan(int64_t t, int g, int w, int B, int Hkv);
int decode_max_splits(int64_t core_cap, int64_t tail_cap);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t core_cap,
                              int64_t tail_cap);
cudaError_t launch_decode(const void *k_core, const void *v_core,
                          const void *k_tail, const void *v_tail,
                          const void *q_t, void *o_t, bool o_f32,
                          void *workspace, int B, int Hq, int Hkv, int d,
                          int g, int w, int64_t core_cap, int64_t tail_cap,
                          int64_t t, cudaStream_t s);

// One decode step in one launch: append token t (k_t, v_t; ring slot, and
// pooling of the group it completes) and the attention of token t.  The
// workspace's tickets must be zero on entry (every decode launch leaves them
// so).
cudaError_t launch_decode_step(void *k_core, void *v_core, void *k_tail, void *v_tail,
                               const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               bool o_f32, void *workspace, int B, int Hq, int Hkv, int d,
                               int g, int w, int64_t core_cap, int64_t tail_cap, int64_t t,
                               cudaStream_t s);

// Fused core + local attention over a whole sequence (tcgen05 kernel).
// lse != nullptr: also write each row's log-sum-exp (log2 units), fp32
// [B, Hq, T], for the backward pass.
cudaError_t launch_prefill(const void *Q, const void *K, const void *V,
                           const void *Kc, const void *Vc, void *O, bool o_f32,
                           int B, int Hq, int Hkv, int64_t T, int d, int g,
                           int w, cudaStream_t s, float *lse = nullptr);

// Backward pass (training).  Workspace layout (byte offsets, 256-aligned):
// fp16 copies of Q and dO, D = rowsum(dO * O), fp32 dKc and dVc.
struct BwLayoutHost {
    size_t q16, do16, dv, dkc, dvc, dvc_bytes, total;
};
BwLayoutHost bw_layout(int B, int Hq, int Hkv, int64_t T, int d, int g);
cudaError_t launch_backward(const void *Q, const void *K, const void *V, const void *Kc,
                            const void *Vc, const void *O, bool o_f32, const float *lse,
                            const void *dO, float *dQ, float *dK, float *dV, int B, int Hq,
                            int Hkv, int64_t T, int d, int g, int w, void *workspace,
                            cudaStream_t s);
cudaError_t backward_status_read_clear(unsigned int *v);

// The LCA variant.  Condensation of all complete groups of Q/K/V into
// Kc/Vc [B, Hkv, out_rows, d] (fp16; rows 0..floor(T/g)-1 written).
cudaError_t launch_lca_pool(const void *Q, const void *K, const void *V, void *Kc, void *Vc,
                            int B, int Hq, int Hkv, int64_t T, int d, int g, int d_rope,
                            int64_t out_rows, cudaStream_t s);
// Append token t with the running query sums q_sum [B, Hq, d] (fp32).
cudaError_t launch_lca_append(const void *q_t, const void *k_t, const void *v_t, float *q_sum,
                              void *k_core, void *v_core, void *k_tail, void *v_tail, int B,
                              int Hq, int Hkv, int d, int g, int d_rope, int64_t core_cap,
                              int64_t tail_cap, int64_t t, cudaStream_t s);
// q_sum = sum of the query rows p0 .. T-1 of Q [B, Hq, T, d] (zero if none).
cudaError_t launch_lca_qsum_fill(const void *Q, float *q_sum, int B, int Hq, int d, int64_t T,
                                 int64_t p0, cudaStream_t s);
cudaError_t lca_status_read_clear(unsigned int *v);

// Device status words (bits kStatusTimeout, kStatusRange): read and clear.
cudaError_t prefill_status_read_clear(unsigned int *v);
cudaError_t pool_status_read_clear(unsigned int *v);
cudaError_t launch_append_rows(const void *q_t, const void *k_t, const void *v_t,
                               void *k_core, void *v_core, void *k_tail, void *v_tail,
                               long long *lens, int B, int Hq, int Hkv, int d, int g,
                               int64_t core_cap, int64_t tail_cap, cudaStream_t s);
size_t append_rows_smem_bytes(int Hq, int Hkv, int g);
cudaError_t launch_decode_rows(const void *k_core, const void *v_core,
                               const void *k_tail, const void *v_tail,
                               const void *q_t, void *o_t, bool o_f32,
                               void *workspace, const long long *lens, int B, int Hq,
                               int Hkv, int d, int g, int w, int64_t core_cap,
                               int64_t tail_cap, cudaStream_t s);
cudaError_t append_status_read_clear(unsigned int *v);
cudaError_t selftest_status_read_clear(unsigned int *v);
cudaError_t decode_status_read_clear(unsigned int *v);

}  // namespace cca
