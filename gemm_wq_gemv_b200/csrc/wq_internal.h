// wq_internal.h -- declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/wq.h"

namespace wq {

// Problem description handed from the ABI layer to a launcher (already validated).
struct Problem {
    const uint16_t* x;
    const uint32_t* w_q;
    const uint32_t* w_lo;
    const uint16_t* scales;
    const uint16_t* zeros;
    const uint16_t* bias;  // (N,) fp16 or bf16 (WQ_FLAG_BF16), or null
    uint16_t* y;
    int M, K, N, bits, G;  // G resolved: group_size == -1 -> K
    unsigned flags;
    void* ws;              // wq_gemm split-K workspace (may be null)
    size_t ws_bytes;
};

wq_status launch_pack(const uint8_t* codes, int K, int N, int bits, uint32_t* w_q, uint32_t* w_lo,
                      uint32_t* bad_count, cudaStream_t s);
wq_status launch_unpack(const uint32_t* w_q, const uint32_t* w_lo, int K, int N, int bits,
                        uint8_t* codes, cudaStream_t s);
wq_status launch_gptqmodel_convert(const uint32_t* qweight, const uint32_t* qzeros, int K, int N, int bits,
                                   int G, uint32_t* w_q, uint32_t* w_lo, uint16_t* zeros, bool bf,
                                   cudaStream_t s);
wq_status launch_gemv(const Problem& p, cudaStream_t s);

// A GEMV launch prepared once for fixed weights, s, z, bias, shape and flags:
// the kernel, its launch shape and its arguments (tensor maps, then the
// parameter block), with the byte offsets of the x and y pointers inside the
// argument bytes.  launch_prepared patches x and y into a copy and launches.
struct Prepared {
    const void* kern = nullptr;
    dim3 grid{1, 1, 1}, block{1, 1, 1};
    size_t smem = 0;
    unsigned cluster_y = 1;   // CTAs per cluster along the grid's y extent (1: no cluster)
    bool pdl = false;         // programmatic stream serialisation attribute
    int nargs = 0;
    size_t arg_off[6] = {};   // byte offset of each kernel argument in `args`
    size_t x_off = 0, y_off = 0;
    alignas(64) unsigned char args[5 * sizeof(CUtensorMap) + 512] = {};
};
// Fill `pr` for problem p (x and y may be null) instead of launching.
wq_status prepare_gemv(const Problem& p, Prepared& pr);
wq_status launch_prepared(const Prepared& pr, const void* x, void* y, cudaStream_t s);
// GEMV with a small shared-memory footprint for 1-, 2-, 4- and 8-bit words and M <= 16
// (1-bit: M <= 8)
// (wq_gemv_lean.cu); launch_gemv routes the shapes it takes there.
bool gemv_lean_takes(const Problem& p);
wq_status launch_gemv_lean(const Problem& p, cudaStream_t s, Prepared* prep = nullptr);
wq_status launch_gemm(const Problem& p, cudaStream_t s);
size_t gemm_workspace_bytes(int M, int K, int N, int bits, int G);
wq_status launch_mse_search(const float* w, int rows, int cols, int group_size, int bits, int symmetric,
                            int steps, int grid, float norm, int patience, float* scale, float* zero,
                            int32_t* step, float* err, uint32_t* any_mask, cudaStream_t stream);

// Device status words (one per kernel file): nonzero once a bounded wait ran out.
// Reading synchronises the device; reset clears the word.
wq_status gemm_device_status(int reset);
wq_status gemv_device_status(int reset);
wq_status gemv_lean_device_status(int reset);
wq_status gptq_device_status(int reset);

// GPTQ block quantisation (wq_gptq.cu), arguments already validated.
size_t gptq_workspace_bytes(int R, int C);
wq_status launch_gptq(const float* W, const float* H, const float* scale, const float* zero, int R, int C, int G,
                      int bits, int blocksize, float percdamp, float* Q, uint8_t* codes, float* losses,
                      void* workspace, cudaStream_t s);

// 2-D tiled TMA descriptor for a row-major (outer, inner) array.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
int sm_count();

constexpr int MAX_DEVICES = 64;
uint64_t current_ctx_id();
wq_status ensure_smem_attr(const void* kern, int bytes, std::atomic<uint64_t>* done, int dev);

inline wq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

}  // namespace wq
