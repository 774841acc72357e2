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
#include <mutex>

#include <cuda_runtime.h>

#include "wq_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_gemm_scratch[WQ_GEMM_NOALLOC_SCRATCH_BYTES];

// The array's device address in the context current on each device, and the ID
// of that context.  A context that is destroyed and made again (cudaDeviceReset)
// loads the library's device image afresh, and the array may move: a new
// context ID makes the next call look the address up again.
struct ScratchSlot {
    std::mutex mu;
    uint64_t ctx = 0;
    void* addr = nullptr;
};
ScratchSlot g_slot[wq::MAX_DEVICES];

// Device address of the array in the current context, looked up (with that
// device current) on the first call in each context and kept.
wq_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    if (dev < 0 || dev >= wq::MAX_DEVICES) return WQ_ERR_UNSUPPORTED;
    const uint64_t id = wq::current_ctx_id();
    ScratchSlot& sl = g_slot[dev];
    std::lock_guard<std::mutex> lk(sl.mu);
    if (id == 0 || sl.ctx != id || !sl.addr) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_gemm_scratch) != cudaSuccess || !a) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
        sl.addr = a;
        sl.ctx = id;
    }
    *out = sl.addr;
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
