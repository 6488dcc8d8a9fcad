// cca_selftest_wait_timeout: exercises the bounded-wait path that every
// kernel of the library takes when a barrier never completes.
//
// One CTA waits on a shared-memory mbarrier that nothing arrives at, with
// the same wait routine the prefill kernel uses (wait_bounded, here with a
// caller-chosen limit), records kStatusTimeout in its device status word
// when the wait runs out, and returns.  cca_device_status() then reports
// CCA_ERR_TIMEOUT, and the context stays usable: nothing faults, traps or
// hangs.  It lets a test check the failure path on a GPU without making a
// real kernel fail.
#include "../../include/cca.h"
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cca {

__device__ unsigned int g_selftest_status;  // kStatusTimeout

namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    // No thread arrives: the phase never completes and the wait runs out.
    const bool ok = wait_bounded(&bar, 0, &abort_flag, limit_ns);
    if (!ok && threadIdx.x == 0) atomicOr(&g_selftest_status, kStatusTimeout);
}

}  // namespace

cudaError_t selftest_status_read_clear(unsigned int *v)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(v, g_selftest_status, sizeof(*v));
    if (e == cudaSuccess && *v) e = cudaMemcpyToSymbol(g_selftest_status, &zero, sizeof(zero));
    return e;
}

}  // namespace cca

extern "C" cca_status cca_selftest_wait_timeout(unsigned int limit_us, cudaStream_t stream)
{
    if (limit_us == 0 || limit_us > 2000000u) return CCA_ERR_INVALID_ARG;
    cca::wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000u);
    return cudaGetLastError() == cudaSuccess ? CCA_OK : CCA_ERR_CUDA;
}
