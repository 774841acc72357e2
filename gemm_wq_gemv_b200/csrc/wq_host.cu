// wq_host.cu -- host helpers shared by the launchers: TMA tensor maps, SM count.
#include <cudaTypedefs.h>

#include <atomic>

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
