// wq_noalloc.cu -- wq_gemm_noalloc: wq_gemm with its split-K scratch in a fixed
// device array instead of a caller workspace.
//
// For callers that cannot allocate device memory at call time: a runtime that
// has handed all device memory to its own pool, or a plug-in whose host forbids
// allocation after initialisation (cudaMalloc also synchronises the device,
// which a per-token decode loop cannot afford).  The call allocates nothing:
// the scratch is a file-scope __device__ array of WQ_GEMM_NOALLOC_SCRATCH_BYTES
// in the library's device image, which the CUDA runtime instantiates once per
// device.  Nothing in it needs to start at zero: within one launch every slice
// the owners read was written first.  Calls that may run at the same time on
// one device share the array and race.
#include <atomic>

#include <cuda_runtime.h>

#include "wq_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_gemm_scratch[WQ_GEMM_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::atomic<void*> g_scratch_addr[MAX_DEVICES];

// Device address of the array on the current device, looked up on the first
// call per device (with that device current) and kept.
wq_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    if (dev < 0 || dev >= MAX_DEVICES) return WQ_ERR_UNSUPPORTED;
    void* a = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!a) {
        if (cudaGetSymbolAddress(&a, g_gemm_scratch) != cudaSuccess || !a) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
        g_scratch_addr[dev].store(a, std::memory_order_release);
    }
    *out = a;
    return WQ_OK;
}

}  // namespace

extern "C" wq_status wq_gemm_noalloc(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                                     const uint16_t* scales, const uint16_t* zeros,
                                     const uint16_t* bias, uint16_t* y, int M, int K, int N,
                                     int bits, int group_size, unsigned flags, void* stream) {
    // 0 for shapes that do not split K and for invalid arguments, which wq_gemm
    // then rejects without the scratch.
    const size_t need = wq_gemm_workspace_size(M, K, N, bits, group_size);
    if (need > WQ_GEMM_NOALLOC_SCRATCH_BYTES) return WQ_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if (need > 0) {
        const wq_status st = scratch_address(&scratch);
        if (st != WQ_OK) return st;
    }
    return wq_gemm(x, w_q, w_lo, scales, zeros, bias, y, M, K, N, bits, group_size, flags, scratch,
                   scratch ? (size_t)WQ_GEMM_NOALLOC_SCRATCH_BYTES : 0, stream);
}
