// wq_selftest.cu -- failure-detection self-test of the bounded waits.
//
// The products never spin without a limit: every mbarrier wait gives up after a
// time limit, records the time-out in a device status word, skips the rest of
// the kernel's work and lets it exit, so the context stays usable and the host
// reads WQ_ERR_TIMEOUT.  This entry point runs that path on purpose, with no
// fault: one CTA waits, with the same bounded wait the products use, on an
// mbarrier that nothing ever completes.  The pages have no counterpart.
#include <cuda_runtime.h>

#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {
namespace {

__device__ unsigned int g_selftest_status = 0;

__global__ void wait_timeout_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none will come
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 of a fresh barrier completes only after an arrival
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicExch(&g_selftest_status, 1u);
    }
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000ull) return WQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(wq::g_selftest_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) !=
        cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    wq::wait_timeout_kernel<<<1, 32, 0, s>>>(limit_ns);
    if (cudaGetLastError() != cudaSuccess) return WQ_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, wq::g_selftest_status, sizeof(v), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return v ? WQ_ERR_TIMEOUT : WQ_OK;
}
