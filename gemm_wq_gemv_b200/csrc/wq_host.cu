// wq_host.cu -- host helpers shared by the launchers: TMA tensor maps, SM count.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>

#include "wq_internal.h"

namespace wq {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        else
            cudaGetLastError();
    }
    return fn;
}

}  // namespace

// A decode loop encodes the same descriptors for the same weights every step:
// a small per-thread cache keyed by every encoding argument returns them.
struct MapKey {
    const void* ptr;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int dt, sw;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && sw == o.sw;
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool valid;
};
constexpr int MAP_CACHE = 64;

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    static thread_local MapEntry cache[MAP_CACHE];
    const MapKey key{ptr, inner, outer, row_bytes, box_inner, box_outer, (int)dt, (int)sw};
    const size_t h = ((reinterpret_cast<uintptr_t>(ptr) >> 8) ^ (inner * 31) ^ (outer * 131) ^ (box_outer * 7) ^
                      (uint64_t)dt) % MAP_CACHE;
    if (cache[h].valid && cache[h].key == key) {
        *m = cache[h].map;
        return true;
    }
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    cache[h] = MapEntry{key, *m, true};
    return true;
}

// Unique ID of the CUDA context current on this thread (0 when there is none or
// the driver does not report one).  A context that is destroyed and created
// again (cudaDeviceReset) gets a new ID, so per-context state keyed on it --
// a kernel attribute, a symbol's device address -- is set up again.
uint64_t current_ctx_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static std::atomic<GetCurrent> get_current{nullptr};
    static std::atomic<GetId> get_id{nullptr};
    GetCurrent gc = get_current.load(std::memory_order_acquire);
    GetId gi = get_id.load(std::memory_order_acquire);
    if (!gc || !gi) {
        void* p1 = nullptr;
        void* p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return 0;
        }
        gc = reinterpret_cast<GetCurrent>(p1);
        gi = reinterpret_cast<GetId>(p2);
        get_current.store(gc, std::memory_order_release);
        get_id.store(gi, std::memory_order_release);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (gc(&ctx) != CUDA_SUCCESS || !ctx || gi(ctx, &id) != CUDA_SUCCESS) return 0;
    return (uint64_t)id;
}

// Raise a kernel's dynamic shared-memory limit once per context.  `done` is the
// caller's per-device record of the context the attribute was last set in; a
// concurrent first call may set it twice, which is harmless (the setting is
// idempotent), and no call launches before its own thread has set it.
wq_status ensure_smem_attr(const void* kern, int bytes, std::atomic<uint64_t>* done, int dev) {
    if (dev < 0 || dev >= MAX_DEVICES) return WQ_ERR_UNSUPPORTED;
    const uint64_t id = current_ctx_id();
    if (id != 0 && done[dev].load(std::memory_order_acquire) == id) return WQ_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return WQ_ERR_CUDA;
    if (id != 0) done[dev].store(id, std::memory_order_release);
    return WQ_OK;
}

// SM count of the current device, queried once per device (148 without a device).
int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace wq

namespace wq {

wq_status launch_prepared(const Prepared& pr, const void* x, void* y, cudaStream_t s) {
    alignas(64) unsigned char args[sizeof(pr.args)];
    std::memcpy(args, pr.args, sizeof(args));
    std::memcpy(args + pr.x_off, &x, sizeof(x));
    std::memcpy(args + pr.y_off, &y, sizeof(y));
    void* argv[6];
    for (int i = 0; i < pr.nargs; ++i) argv[i] = args + pr.arg_off[i];
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = pr.grid;
    cfg.blockDim = pr.block;
    cfg.dynamicSmemBytes = pr.smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (pr.cluster_y > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = pr.cluster_y;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pr.pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return from_cuda(cudaLaunchKernelExC(&cfg, pr.kern, argv));
}

}  // namespace wq
