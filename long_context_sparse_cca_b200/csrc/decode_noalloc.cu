// cca_attn_decode_noalloc: the decode attention of cca_attn_decode with its
// split-K workspace in a fixed, library-owned device array instead of
// caller-provided memory.
//
// Some callers cannot hand the library a workspace: runtimes that plan all
// device memory up front and forbid allocations outside their own pool,
// plug-in hosts that only pass input and output pointers through, and
// latency-critical loops where a cudaMalloc (which can synchronise the whole
// device) is not acceptable.  For them this entry point uses g_scratch below,
// a fixed array every GPU that loads the library holds until the process
// exits, and calls no allocating routine of the CUDA runtime or of any
// other library.
//
// The array's device address is looked up once per device, with that device
// current, on that device's first call (cudaGetSymbolAddress).  That first
// call should therefore come before any stream capture begins.  The contents
// left by one call are simply overwritten by the next: every partial result
// the merge reads is written earlier in the same call, and the call clears
// its own completion counters, so nothing needs to start at zero.  All calls
// share the one array, so calls whose kernels overlap on the GPU (different
// streams, no ordering between them) race.
#include <mutex>

#include "../../include/cca.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[CCA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device

// Device address of g_scratch on the current device (looked up on first use).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" cca_status cca_attn_decode_noalloc(const cca_cache *c, const void *q_t, void *o_t,
                                              cca_dtype o_dtype, cudaStream_t stream)
{
    // An invalid cache reports 0 bytes; cca_attn_decode then returns the
    // cache's own error before launching anything.
    const size_t need = cca_decode_workspace_bytes(c);
    if (need == 0) return cca_attn_decode(c, q_t, o_t, o_dtype, nullptr, 0, stream);
    if (need > CCA_NOALLOC_SCRATCH_BYTES) return CCA_ERR_SCRATCH;
    void *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return CCA_ERR_CUDA;
    return cca_attn_decode(c, q_t, o_t, o_dtype, ws, CCA_NOALLOC_SCRATCH_BYTES, stream);
}
