// wq_pack.cu -- bit-exact packing of codes into K-major words and back.
//
// Layout (dashq_kernel.py `_pack_kmajor` / `_unpack_kmajor`; 3-bit planes as in
// `TritonQuantLinear.__init__` and `dequantize_weight`): code q[k][n] of a b-bit
// plane lives in word [k / eps][n] at bit b * (k % eps), eps = 32 / b.  3-bit
// codes are split into a 2-bit plane of q >> 1 and a 1-bit plane of q & 1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "wq_internal.h"

namespace wq {
namespace {

// One thread per output word of one plane.  `src_shift` / `src_mask` select the
// bits of each code that go into this plane; codes above `range_max` are
// counted into *bad when `check` is set (and are masked either way).
__global__ void pack_plane_kernel(const uint8_t* __restrict__ codes, int N, size_t n_words,
                                  int plane_bits, int src_shift, uint32_t src_mask,
                                  uint32_t range_max, bool check, uint32_t* __restrict__ words,
                                  uint32_t* __restrict__ bad) {
    const int eps = 32 / plane_bits;
    uint32_t n_bad = 0;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_words;
         i += (size_t)gridDim.x * blockDim.x) {
        size_t r = i / N;
        int n = (int)(i - r * N);
        const uint8_t* src = codes + r * eps * (size_t)N + n;
        uint32_t w = 0;
        for (int j = 0; j < eps; ++j) {
            uint32_t c = src[(size_t)j * N];
            n_bad += (c > range_max);
            w |= ((c >> src_shift) & src_mask) << (plane_bits * j);
        }
        words[i] = w;
    }
    if (check && bad) {
        uint32_t tot = __reduce_add_sync(0xffffffffu, n_bad);
        if ((threadIdx.x & 31) == 0 && tot) atomicAdd(bad, tot);
    }
}

// One thread per code.
__global__ void unpack_kernel(const uint32_t* __restrict__ w_q, const uint32_t* __restrict__ w_lo,
                              int N, size_t n_codes, int bits, uint8_t* __restrict__ codes) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_codes;
         i += (size_t)gridDim.x * blockDim.x) {
        size_t k = i / N;
        size_t n = i - k * N;
        uint32_t q;
        if (bits == 3) {
            uint32_t hi = (w_q[(k / 16) * N + n] >> (2 * (k % 16))) & 3u;
            uint32_t lo = (w_lo[(k / 32) * N + n] >> (k % 32)) & 1u;
            q = (hi << 1) | lo;
        } else {
            int eps = 32 / bits;
            q = (w_q[(k / eps) * N + n] >> (bits * (k % eps))) & ((1u << bits) - 1u);
        }
        codes[i] = (uint8_t)q;
    }
}

// GPTQModel format ("GPTQModel-Compatible Triton Kernel" README, "Quantization
// Format"): V codes per word, code k of a column at bit bits * (k % V) of word
// k / V (3-bit: V = 10, bits 30-31 unused); qzeros pack a group's zero points
// along N the same way.
// One thread per (group, column): the zero point as a 16-bit float (fp16 or bf16).
__global__ void gq_zeros_kernel(const uint32_t* __restrict__ qzeros, int N, int NP, size_t n_out, int bits,
                                int V, bool bf, uint16_t* __restrict__ zeros) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_out;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t g = i / N;
        const int n = (int)(i - g * N);
        const uint32_t z = (qzeros[g * NP + n / V] >> (bits * (n % V))) & ((1u << bits) - 1u);
        zeros[i] = bf ? __bfloat16_as_ushort(__uint2bfloat16_rn(z)) : __half_as_ushort(__uint2half_rn(z));
    }
}

// 3-bit: one thread per (32-row block r, column n) reads the block's codes
// from the 10-per-word words and writes lo-plane word r and hi-plane words
// 2 r and 2 r + 1.
__global__ void gq_repack3_kernel(const uint32_t* __restrict__ qweight, int N, size_t n_blocks,
                                  uint32_t* __restrict__ w_q, uint32_t* __restrict__ w_lo) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_blocks;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t r = i / N;
        const size_t n = i - r * N;
        uint32_t lo = 0, hi0 = 0, hi1 = 0;
        for (int j = 0; j < 32; ++j) {
            const size_t k = 32 * r + j;
            const uint32_t q = (qweight[(k / 10) * N + n] >> (3 * (k % 10))) & 7u;
            lo |= (q & 1u) << j;
            if (j < 16) hi0 |= (q >> 1) << (2 * j);
            else hi1 |= (q >> 1) << (2 * (j - 16));
        }
        w_lo[r * N + n] = lo;
        w_q[(2 * r) * N + n] = hi0;
        w_q[(2 * r + 1) * N + n] = hi1;
    }
}

unsigned grid_for(size_t work, int block) {
    size_t b = (work + block - 1) / block;
    if (b > 148u * 64u) b = 148u * 64u;
    return (unsigned)(b ? b : 1);
}

}  // namespace

wq_status launch_pack(const uint8_t* codes, int K, int N, int bits, uint32_t* w_q, uint32_t* w_lo,
                      uint32_t* bad, cudaStream_t s) {
    const int block = 256;
    const uint32_t qmax = (1u << bits) - 1u;
    if (bits == 3) {
        size_t nh = (size_t)(K / 16) * N, nl = (size_t)(K / 32) * N;
        pack_plane_kernel<<<grid_for(nh, block), block, 0, s>>>(codes, N, nh, 2, 1, 3u, qmax, false,
                                                                w_q, bad);
        pack_plane_kernel<<<grid_for(nl, block), block, 0, s>>>(codes, N, nl, 1, 0, 1u, qmax, true,
                                                                w_lo, bad);
    } else {
        size_t nw = (size_t)(K / (32 / bits)) * N;
        pack_plane_kernel<<<grid_for(nw, block), block, 0, s>>>(codes, N, nw, bits, 0, qmax, qmax,
                                                                true, w_q, bad);
    }
    return from_cuda(cudaGetLastError());
}

wq_status launch_gptqmodel_convert(const uint32_t* qweight, const uint32_t* qzeros, int K, int N, int bits,
                                   int G, uint32_t* w_q, uint32_t* w_lo, uint16_t* zeros, bool bf,
                                   cudaStream_t s) {
    const int block = 256;
    const int V = bits == 3 ? 10 : 32 / bits;
    const int NP = (N + V - 1) / V;
    const size_t nz = (size_t)(K / G) * N;
    gq_zeros_kernel<<<grid_for(nz, block), block, 0, s>>>(qzeros, N, NP, nz, bits, V, bf, zeros);
    if (cudaGetLastError() != cudaSuccess) return WQ_ERR_CUDA;
    if (bits == 3) {
        const size_t nb = (size_t)(K / 32) * N;
        gq_repack3_kernel<<<grid_for(nb, block), block, 0, s>>>(qweight, N, nb, w_q, w_lo);
    } else if (w_q && w_q != qweight) {  // the same K-major words: a copy
        if (cudaMemcpyAsync(w_q, qweight, (size_t)(K / V) * N * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return WQ_ERR_CUDA;
    }
    return from_cuda(cudaGetLastError());
}

wq_status launch_unpack(const uint32_t* w_q, const uint32_t* w_lo, int K, int N, int bits,
                        uint8_t* codes, cudaStream_t s) {
    const int block = 256;
    size_t n = (size_t)K * N;
    unpack_kernel<<<grid_for(n, block), block, 0, s>>>(w_q, w_lo, N, n, bits, codes);
    return from_cuda(cudaGetLastError());
}

}  // namespace wq
