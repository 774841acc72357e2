// wq_dequant.cuh -- exact conversion of packed code pairs to fp16 (q - round(z)).
//
// Shared by the GEMV and the GEMM.  Codes j and j + E/2 of a word (E codes per
// word) sit at the same bit offset in the two 16-bit halves, so one LOP3 ORs
// both into the mantissa of the fp16 constant 1024 (0x6400), and one exact
// fp16x2 FMA brings them back to the integers q - zi, zi = round(z): every
// value involved is an integer below 2048, so nothing rounds.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_ptx.cuh"

namespace wq {

// ----------------------------------------------------------------- formats
// EPS: codes per word of the main plane (3-bit: the 2-bit plane).
// NC:  number of distinct fp16 bias constants per (group, column).
template <int BITS> struct Fmt;
template <> struct Fmt<1> { static constexpr int EPS = 32, NC = 10; };
template <> struct Fmt<2> { static constexpr int EPS = 16, NC = 5; };
template <> struct Fmt<3> { static constexpr int EPS = 16, NC = 8; };
template <> struct Fmt<4> { static constexpr int EPS = 8, NC = 2; };
template <> struct Fmt<8> { static constexpr int EPS = 4, NC = 1; };

// Per (group, column) record in shared memory: fp32 scale, fp32 fractional zero
// part, and NC bias constants as duplicated fp16 pairs.
template <int BITS> struct alignas(16) Rec {
    float s;
    float zr;
    uint32_t c[Fmt<BITS>::NC];
};

// Bias constant for a code that sits at mantissa bit p of a 0x6400 word and is
// brought back with multiplier 2^-p:  -(1024 * 2^-p + zi).
// 3-bit combines a hi field at bit ph (multiplier 2^(1-ph)) and a lo bit at
// bit j+1 (multiplier 2^-(j+1)): -(2^(11-ph) + 2^(9-j) + zi).
template <int BITS>
__device__ __forceinline__ float bias_magnitude(int i) {
    if constexpr (BITS == 1 || BITS == 2) {
        return 1024.0f / (float)(1 << (BITS * i));  // positions p = BITS * i
    } else if constexpr (BITS == 4) {
        return i == 0 ? 1024.0f : 64.0f;            // p = 0 and p = 4
    } else if constexpr (BITS == 8) {
        return 1024.0f;
    } else {
        const int ph = 2 * (i & 3) + 1;
        return (float)(1 << (11 - ph)) + (float)(1 << (9 - i));
    }
}

__device__ __forceinline__ uint32_t dup_half(float v) {
    __half h = __float2half_rn(v);
    uint16_t b = __half_as_ushort(h);
    return (uint32_t)b | ((uint32_t)b << 16);
}

// fp16x2 constant with the same value in both lanes (compile-time exact values).
__device__ __forceinline__ constexpr uint32_t h2c(uint32_t bits16) { return bits16 | (bits16 << 16); }

// fp16 bit patterns of 2^-p, p = 0..10
__device__ __forceinline__ constexpr uint32_t pow2neg_h(int p) { return (uint32_t)(15 - p) << 10; }

// ------------------------------------------------------- pair dequantisation
// Pair j of word w (codes j and j + EPS/2 in the low / high half) as fp16x2
// values q - zi, given the column's bias constants c[].
template <int BITS>
__device__ __forceinline__ uint32_t pair_q(uint32_t w, uint32_t w_hi, uint32_t lo_spread,
                                           const uint32_t (&c)[Fmt<BITS>::NC], int j) {
    constexpr uint32_t MAGIC = 0x64006400u;
    if constexpr (BITS == 8) {
        // bytes (j, j + 2) -> [b, 0x64] halves
        uint32_t v = prmt(w, 0x64646464u, j == 0 ? 0x4240u : 0x4341u);
        return hfma2_u32(v, h2c(0x3C00u), c[0]);
    } else if constexpr (BITS == 4) {
        // j = 0: bits 0-3, j = 1: bits 4-7, j = 2, 3: the same in w >> 8.
        const uint32_t src = (j < 2) ? w : w_hi;
        const int p = (j & 1) ? 4 : 0;
        uint32_t v = and_or(src, 0x000F000Fu << p, MAGIC);
        return hfma2_u32(v, h2c(pow2neg_h(p)), c[j & 1]);
    } else if constexpr (BITS == 2) {
        // j = 0..4: bits 2j, 2j+1 of w; j = 5..7: the same of w >> 10.
        const uint32_t src = (j < 5) ? w : w_hi;
        const int i = (j < 5) ? j : j - 5;
        const int p = 2 * i;
        uint32_t v = and_or(src, 0x00030003u << p, MAGIC);
        return hfma2_u32(v, h2c(pow2neg_h(p)), c[i]);
    } else if constexpr (BITS == 1) {
        const uint32_t src = (j < 10) ? w : w_hi;
        const int p = (j < 10) ? j : j - 10;
        uint32_t v = and_or(src, 0x00010001u << p, MAGIC);
        return hfma2_u32(v, h2c(pow2neg_h(p)), c[p]);
    } else {  // 3-bit: w = hi word << 1, w_hi = hi word >> 7, lo_spread = lo bits j at j+1 / j+17
        const uint32_t src = (j < 4) ? w : w_hi;
        const int ph = 2 * (j & 3) + 1;
        uint32_t H = and_or(src, 0x00030003u << ph, MAGIC);
        uint32_t L = and_or(lo_spread, 0x00010001u << (j + 1), MAGIC);
        uint32_t T = hfma2_u32(H, h2c(pow2neg_h(ph - 1)), c[j]);
        return hfma2_u32(L, h2c(pow2neg_h(j + 1)), T);
    }
}

// Per-word preparation for pair_q: the shifted copies each width needs.
// 3-bit: w becomes hi << 1, w_hi = hi >> 7, lo_spread = the lo bits of this hi
// word's 16 codes at bit j + 1 (codes 0-7) and j + 17 (codes 8-15); `lo_sel`
// picks the lower (0x7170) or upper (0x7372) half of the lo word.
template <int BITS>
__device__ __forceinline__ void prep_word(uint32_t& w, uint32_t& w_hi, uint32_t& lo_spread,
                                          uint32_t lo_word, uint32_t lo_sel) {
    if constexpr (BITS == 4) {
        w_hi = w >> 8;
    } else if constexpr (BITS == 2 || BITS == 1) {
        w_hi = w >> 10;
    } else if constexpr (BITS == 3) {
        w_hi = w >> 7;
        w <<= 1;
        lo_spread = prmt(lo_word, 0u, lo_sel) << 1;
    } else {
        w_hi = w;
    }
}

}  // namespace wq
