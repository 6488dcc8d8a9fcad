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
// The array's device address is looked up once per CUDA context, with that
// context current, on the first call made in it (cudaGetSymbolAddress): once
// per device for the runtime's primary contexts, and again after a context is
// re-created (for example after cudaDeviceReset, when the module may load at
// another address).  That first call should therefore come before any
// stream capture begins.  The contents left by one call are simply
// overwritten by the next: every partial result the merge reads is written
// earlier in the same call, and the call clears its own completion counters,
// so nothing needs to start at zero.  All calls share the one array, so calls
// whose kernels overlap on the GPU (different streams, no ordering between
// them) race.
#include <cuda.h>

#include <mutex>

#include "../../include/cca.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[CCA_NOALLOC_SCRATCH_BYTES];

// Device address of g_scratch per CUDA context, keyed by the context's
// unique ID (cuCtxGetId), which a re-created context never shares with an
// earlier one.
constexpr int kMaxContexts = 64;
struct Entry {
    unsigned long long ctx_id;
    void *addr;
};
std::mutex g_mu;
Entry g_entries[kMaxContexts];
int g_n_entries = 0;

using GetCurrentFn = CUresult (*)(CUcontext *);
using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// ID of the calling thread's current context: a context the caller made
// current, else the current device's primary context.
cudaError_t current_context_id(unsigned long long *id)
{
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void *f = nullptr, *g = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q1);
        if (e != cudaSuccess) return e;
        e = cudaGetDriverEntryPoint("cuCtxGetId", &g, cudaEnableDefault, &q2);
        if (e != cudaSuccess) return e;
        if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess)
            return cudaErrorNotSupported;
        get_current = reinterpret_cast<GetCurrentFn>(f);
        get_id = reinterpret_cast<GetIdFn>(g);
    }
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    if (ctx == nullptr) {
        // No context is current on this thread yet: the runtime would bind
        // the current device's primary context at its next call; bind it
        // now (cudaSetDevice initialises and binds it, and allocates
        // nothing).
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaSetDevice(dev);
        if (e != cudaSuccess) return e;
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    }
    if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// Device address of g_scratch in the current context (looked up on first use).
cudaError_t scratch_address(void **out)
{
    unsigned long long id = 0;
    cudaError_t e = current_context_id(&id);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_entries; ++i) {
        if (g_entries[i].ctx_id == id) {
            *out = g_entries[i].addr;
            return cudaSuccess;
        }
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    // a full table forgets its oldest entry (contexts of a long-gone past)
    if (g_n_entries == kMaxContexts) {
        for (int i = 1; i < kMaxContexts; ++i) g_entries[i - 1] = g_entries[i];
        --g_n_entries;
    }
    g_entries[g_n_entries++] = Entry{id, p};
    *out = p;
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
