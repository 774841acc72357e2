// wq_abi.cu -- the C entry points of libwq.so: argument checks and dispatch.
//
// Every rule checked here is stated next to the entry point in include/wq.h.
// Nothing is launched unless every check passes.
#include <cuda_runtime.h>

#include <new>

#include "wq_internal.h"

namespace {

bool supported_bits(int b) { return b == 1 || b == 2 || b == 3 || b == 4 || b == 8; }

// Rows of K that one word row covers for the shape rules (3-bit: the lo plane's 32).
int k_quantum(int bits) { return bits == 3 ? 32 : 32 / bits; }

// Codes per word of the main plane (3-bit: the 2-bit plane, 16).
int main_eps(int bits) { return bits == 3 ? 16 : 32 / bits; }

bool aligned(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The library carries sm_100a code only: refuse any other device up front.
wq_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    static int ok[64] = {0};  // 0 unknown, 1 sm_100, 2 other
    if (dev >= 0 && dev < 64 && ok[dev]) return ok[dev] == 1 ? WQ_OK : WQ_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    const bool good = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) ok[dev] = good ? 1 : 2;
    return good ? WQ_OK : WQ_ERR_UNSUPPORTED;
}

wq_status check_plane_shape(int K, int N, int bits, const void* w_lo, bool need_lo_rule) {
    if (!supported_bits(bits)) return WQ_ERR_UNSUPPORTED;
    if (K < 1 || N < 1) return WQ_ERR_INVALID_ARG;
    if (K % k_quantum(bits) != 0) return WQ_ERR_INVALID_ARG;
    if ((long long)K * (long long)N > (1ll << 40)) return WQ_ERR_INVALID_ARG;
    if (need_lo_rule && ((bits == 3) != (w_lo != nullptr))) return WQ_ERR_INVALID_ARG;
    return WQ_OK;
}

// Shared checks of wq_gemv / wq_gemm; resolves G.
wq_status check_product(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                        const uint16_t* s, const uint16_t* z, const uint16_t* y, int M, int K,
                        int N, int bits, int group_size, unsigned flags, int& G) {
    wq_status st = check_plane_shape(K, N, bits, w_lo, true);
    if (st != WQ_OK) return st;
    if (M < 1) return WQ_ERR_INVALID_ARG;
    if (flags & ~WQ_FLAG_ALL) return WQ_ERR_INVALID_ARG;
    if (!x || !w_q || !s || !z || !y) return WQ_ERR_INVALID_ARG;
    if (group_size == -1) {
        G = K;
    } else {
        if (group_size < 1 || K % group_size != 0 || group_size % k_quantum(bits) != 0)
            return WQ_ERR_INVALID_ARG;
        G = group_size;
    }
    if (N % 8 != 0) return WQ_ERR_ALIGNMENT;
    if (!aligned(x, 16) || !aligned(w_q, 16) || !aligned(s, 16) || !aligned(z, 16) ||
        !aligned(y, 16) || (w_lo && !aligned(w_lo, 16)))
        return WQ_ERR_ALIGNMENT;
    return WQ_OK;
}

}  // namespace

extern "C" {

int wq_abi_version(void) { return WQ_ABI_VERSION; }

const char* wq_status_string(wq_status s) {
    switch (s) {
        case WQ_OK: return "ok";
        case WQ_ERR_INVALID_ARG: return "invalid argument";
        case WQ_ERR_UNSUPPORTED: return "unsupported bit width, group size or device";
        case WQ_ERR_ALIGNMENT: return "misaligned pointer or N not a multiple of 8";
        case WQ_ERR_CODE_RANGE: return "code does not fit in the bit width";
        case WQ_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
        case WQ_ERR_CUDA: return "CUDA runtime error";
        case WQ_ERR_SCRATCH_LIMIT: return "shape needs more split-K scratch than the static array holds";
        case WQ_ERR_CHECK: return "a bounds check of the checked build caught an access outside its array";
        case WQ_ERR_NOT_POSITIVE_DEFINITE: return "the damped Hessian is not positive definite";
    }
    return "unknown status";
}

wq_status wq_pack_kmajor(const uint8_t* codes_kn, int K, int N, int bits, uint32_t* w_q,
                         uint32_t* w_lo, uint32_t* bad_count, void* stream) {
    wq_status st = check_plane_shape(K, N, bits, w_lo, true);
    if (st != WQ_OK) return st;
    if (!codes_kn || !w_q) return WQ_ERR_INVALID_ARG;
    if (!aligned(w_q, 4) || (w_lo && !aligned(w_lo, 4)) || (bad_count && !aligned(bad_count, 4)))
        return WQ_ERR_ALIGNMENT;
    if ((st = check_device()) != WQ_OK) return st;
    return wq::launch_pack(codes_kn, K, N, bits, w_q, w_lo, bad_count, (cudaStream_t)stream);
}

wq_status wq_unpack_kmajor(const uint32_t* w_q, const uint32_t* w_lo, int K, int N, int bits,
                           uint8_t* codes_kn, void* stream) {
    wq_status st = check_plane_shape(K, N, bits, w_lo, true);
    if (st != WQ_OK) return st;
    if (!codes_kn || !w_q) return WQ_ERR_INVALID_ARG;
    if (!aligned(w_q, 4) || (w_lo && !aligned(w_lo, 4))) return WQ_ERR_ALIGNMENT;
    if ((st = check_device()) != WQ_OK) return st;
    return wq::launch_unpack(w_q, w_lo, K, N, bits, codes_kn, (cudaStream_t)stream);
}

wq_status wq_gemv(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                  const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias, uint16_t* y,
                  int M, int K, int N, int bits, int group_size, unsigned flags, void* stream) {
    int G = 0;
    wq_status st = check_product(x, w_q, w_lo, scales, zeros, y, M, K, N, bits, group_size, flags, G);
    if (st != WQ_OK) return st;
    if (bias && !aligned(bias, 2)) return WQ_ERR_ALIGNMENT;
    if (M > 16) return WQ_ERR_INVALID_ARG;
    if (G != K && G % (4 * main_eps(bits)) != 0) return WQ_ERR_UNSUPPORTED;
    if ((st = check_device()) != WQ_OK) return st;
    wq::Problem p{x, w_q, w_lo, scales, zeros, bias, y, M, K, N, bits, G, flags, nullptr, 0};
    return wq::launch_gemv(p, (cudaStream_t)stream);
}

struct wq_gemv_plan {
    wq::Prepared pr;
    int dev;
};

wq_status wq_gemv_plan_create(const uint32_t* w_q, const uint32_t* w_lo, const uint16_t* scales,
                              const uint16_t* zeros, const uint16_t* bias, int M, int K, int N, int bits,
                              int group_size, unsigned flags, wq_gemv_plan** plan) {
    if (!plan) return WQ_ERR_INVALID_ARG;
    *plan = nullptr;
    // x and y are bound at each run: w_q stands in for them in the shared checks
    const uint16_t* stand_in = reinterpret_cast<const uint16_t*>(w_q);
    int G = 0;
    wq_status st = check_product(stand_in, w_q, w_lo, scales, zeros, stand_in, M, K, N, bits, group_size, flags, G);
    if (st != WQ_OK) return st;
    if (bias && !aligned(bias, 2)) return WQ_ERR_ALIGNMENT;
    if (M > 16) return WQ_ERR_INVALID_ARG;
    if (G != K && G % (4 * main_eps(bits)) != 0) return WQ_ERR_UNSUPPORTED;
    if ((st = check_device()) != WQ_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    wq_gemv_plan* h = new (std::nothrow) wq_gemv_plan();
    if (!h) return WQ_ERR_CUDA;
    h->dev = dev;
    const wq::Problem p{nullptr, w_q, w_lo, scales, zeros, bias, nullptr, M, K, N, bits, G, flags, nullptr, 0};
    if ((st = wq::prepare_gemv(p, h->pr)) != WQ_OK) {
        delete h;
        return st;
    }
    *plan = h;
    return WQ_OK;
}

wq_status wq_gemv_plan_run(const wq_gemv_plan* plan, const uint16_t* x, uint16_t* y, void* stream) {
    if (!plan || !x || !y) return WQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return WQ_ERR_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->dev) return WQ_ERR_INVALID_ARG;
    return wq::launch_prepared(plan->pr, x, y, (cudaStream_t)stream);
}

void wq_gemv_plan_destroy(wq_gemv_plan* plan) { delete plan; }

wq_status wq_gemm(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                  const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias, uint16_t* y,
                  int M, int K, int N, int bits, int group_size, unsigned flags, void* workspace,
                  size_t workspace_bytes, void* stream) {
    int G = 0;
    wq_status st = check_product(x, w_q, w_lo, scales, zeros, y, M, K, N, bits, group_size, flags, G);
    if (st != WQ_OK) return st;
    if (bias && !aligned(bias, 2)) return WQ_ERR_ALIGNMENT;
    // the tensor-memory copy engine reads x in rows of K values: 16-byte multiples
    if (K % 8 != 0) return WQ_ERR_ALIGNMENT;
    if (workspace && !aligned(workspace, 16)) return WQ_ERR_ALIGNMENT;
    if ((st = check_device()) != WQ_OK) return st;
    wq::Problem p{x, w_q, w_lo, scales, zeros, bias, y, M, K, N, bits, G, flags, workspace,
                  workspace ? workspace_bytes : 0};
    return wq::launch_gemm(p, (cudaStream_t)stream);
}

size_t wq_gemm_workspace_size(int M, int K, int N, int bits, int group_size) {
    if (!supported_bits(bits) || M < 1 || N < 1 || K < 1 || K % k_quantum(bits) != 0 || K % 8 != 0) return 0;
    const int G = group_size == -1 ? K : group_size;
    if (G < 1 || K % G != 0 || G % k_quantum(bits) != 0) return 0;
    return wq::gemm_workspace_bytes(M, K, N, bits, G);
}

int wq_matmul_uses_gemv(int M, int K, int N, int bits, int group_size) {
    if (!supported_bits(bits) || M < 1 || K < 1 || N < 1) return 0;
    const int G = group_size == -1 ? K : group_size;
    const bool gemv_group = G == K || (G > 0 && G % (4 * main_eps(bits)) == 0);
    // 4- and 8-bit words: the lean GEMV takes up to 16 tokens (M = 16 of 4096 x 4096
    // in 3.4 us, below the GEMM's fixed cost per launch); other widths stage x on
    // chip, so M = 9..16 goes there only while M * K < 65536
    const bool lean = bits == 4 || bits == 8;
    const bool small_m = M <= 8 || (M <= 16 && (lean || (long long)M * K < 65536));
    return (gemv_group && small_m) ? 1 : 0;
}

size_t wq_matmul_workspace_size(int M, int K, int N, int bits, int group_size) {
    return wq_matmul_uses_gemv(M, K, N, bits, group_size) ? 0
                                                         : wq_gemm_workspace_size(M, K, N, bits, group_size);
}

wq_status wq_matmul(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                    const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias, uint16_t* y,
                    int M, int K, int N, int bits, int group_size, unsigned flags, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (wq_matmul_uses_gemv(M, K, N, bits, group_size))
        return wq_gemv(x, w_q, w_lo, scales, zeros, bias, y, M, K, N, bits, group_size, flags, stream);
    return wq_gemm(x, w_q, w_lo, scales, zeros, bias, y, M, K, N, bits, group_size, flags, workspace,
                   workspace_bytes, stream);
}

wq_status wq_gptqmodel_convert(const uint32_t* qweight, const uint32_t* qzeros, int K, int N, int bits,
                               int group_size, uint32_t* w_q, uint32_t* w_lo, uint16_t* zeros, unsigned flags,
                               void* stream) {
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return WQ_ERR_UNSUPPORTED;
    wq_status st = check_plane_shape(K, N, bits, w_lo, true);
    if (st != WQ_OK) return st;
    if (flags & ~WQ_FLAG_BF16) return WQ_ERR_INVALID_ARG;
    const int G = group_size == -1 ? K : group_size;
    if (G < 1 || K % G != 0) return WQ_ERR_INVALID_ARG;
    if (!qweight || !qzeros || !zeros || (bits == 3 && !w_q)) return WQ_ERR_INVALID_ARG;
    if (!aligned(qweight, 4) || !aligned(qzeros, 4) || !aligned(zeros, 2) || (w_q && !aligned(w_q, 4)) ||
        (w_lo && !aligned(w_lo, 4)))
        return WQ_ERR_ALIGNMENT;
    if ((st = check_device()) != WQ_OK) return st;
    return wq::launch_gptqmodel_convert(qweight, qzeros, K, N, bits, G, w_q, w_lo, zeros,
                                        (flags & WQ_FLAG_BF16) != 0, (cudaStream_t)stream);
}

wq_status wq_mse_search(const float* w, int rows, int cols, int group_size, int bits, int symmetric,
                        int steps, int grid, float norm, int patience, float* scale, float* zero,
                        int32_t* step, float* err, void* workspace, size_t workspace_bytes,
                        void* stream) {
    if (bits < 1 || bits > 8) return WQ_ERR_UNSUPPORTED;
    if (rows < 1 || cols < 1 || group_size < 1 || cols % group_size != 0) return WQ_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
    if (steps < 1 || steps > 32 || grid < 1 || patience < 0) return WQ_ERR_INVALID_ARG;
    if (!(norm > 0.0f) || !(norm < 3.0e38f)) return WQ_ERR_INVALID_ARG;  // rejects NaN and infinities
    if (!w || !scale || !zero || !step || !err) return WQ_ERR_INVALID_ARG;
    if (patience > 0 && (!workspace || workspace_bytes < 4)) return WQ_ERR_INVALID_ARG;
    if (!aligned(w, 4) || !aligned(scale, 4) || !aligned(zero, 4) || !aligned(step, 4) ||
        !aligned(err, 4) || (workspace && !aligned(workspace, 4)))
        return WQ_ERR_ALIGNMENT;
    wq_status st = check_device();
    if (st != WQ_OK) return st;
    return wq::launch_mse_search(w, rows, cols, group_size, bits, symmetric, steps, grid, norm, patience,
                                 scale, zero, step, err, static_cast<uint32_t*>(workspace),
                                 (cudaStream_t)stream);
}

size_t wq_gptq_workspace_size(int rows, int cols) {
    if (rows < 1 || cols < 1 || cols > 65536) return 0;
    return wq::gptq_workspace_bytes(rows, cols);
}

wq_status wq_gptq_quantize(const float* W, const float* H, const float* scale, const float* zero, int rows,
                           int cols, int group_size, int bits, int blocksize, float percdamp, float* Q,
                           uint8_t* codes, float* losses, void* workspace, size_t workspace_bytes,
                           void* stream) {
    if (bits < 1 || bits > 8) return WQ_ERR_UNSUPPORTED;
    if (rows < 1 || cols < 1 || cols > 65536 || group_size < 1 || blocksize < 1 || blocksize > 128)
        return WQ_ERR_INVALID_ARG;
    if ((size_t)rows * (size_t)cols > ((size_t)1 << 40)) return WQ_ERR_INVALID_ARG;
    if (!(percdamp >= 0.0f) || !(percdamp < 1.0e30f)) return WQ_ERR_INVALID_ARG;  // rejects NaN
    if (!W || !H || !scale || !zero || !losses || !workspace) return WQ_ERR_INVALID_ARG;
    if (workspace_bytes < wq::gptq_workspace_bytes(rows, cols)) return WQ_ERR_INVALID_ARG;
    if (!aligned(W, 4) || !aligned(H, 4) || !aligned(scale, 4) || !aligned(zero, 4) || !aligned(losses, 4) ||
        (Q && !aligned(Q, 4)) || !aligned(workspace, 256))
        return WQ_ERR_ALIGNMENT;
    wq_status st = check_device();
    if (st != WQ_OK) return st;
    return wq::launch_gptq(W, H, scale, zero, rows, cols, group_size, bits, blocksize, percdamp, Q, codes, losses,
                           workspace, (cudaStream_t)stream);
}

int wq_checked_build(void) {
#ifdef WQ_CHECKS
    return 1;
#else
    return 0;
#endif
}

wq_status wq_device_status(int reset) {
    const wq_status a = wq::gemm_device_status(reset);
    const wq_status b = wq::gemv_device_status(reset);
    const wq_status c = wq::gemv_lean_device_status(reset);
    const wq_status d = wq::gptq_device_status(reset);
    if (a == WQ_ERR_CUDA || b == WQ_ERR_CUDA || c == WQ_ERR_CUDA || d == WQ_ERR_CUDA) return WQ_ERR_CUDA;
    for (const wq_status e : {WQ_ERR_TIMEOUT, WQ_ERR_CHECK})
        if (a == e || b == e || c == e) return e;
    return d;
}

}  // extern "C"
