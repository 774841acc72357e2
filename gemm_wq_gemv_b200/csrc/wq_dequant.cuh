// wq_dequant.cuh -- exact conversion of packed code pairs to fp16 or bf16 (q - round(z)).
//
// Shared by the GEMV and the GEMM.  Codes j and j + E/2 of a word (E codes per
// word) sit at the same bit offset in the two 16-bit halves, so one LOP3 ORs
// both into the mantissa of the fp16 constant 1024 (0x6400), and one exact
// fp16x2 FMA brings them back to the integers q - zi, zi = round(z): every
// value involved is an integer below 2048, so nothing rounds.
//
// bf16 has 7 fraction bits: the constant is 128 (0x4300), whose fraction holds
// a code field only at bits 0-6, so each word is read through two to four
// shifted copies; zi is kept in [0, 2^bits - 1] so that q - zi (|.| <= 255)
// stays exact in bf16's 8 significant bits.  8-bit codes do not fit 7 bits:
// they go through the fp32 constant 2^23 instead and are packed to bf16 pairs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_ptx.cuh"

namespace wq {

// ----------------------------------------------------------------- formats
// EPS: codes per word of the main plane (3-bit: the 2-bit plane).
// NC:  number of distinct fp16 bias constants per (group, column); NCB: bf16.
template <int BITS> struct Fmt;
template <> struct Fmt<1> { static constexpr int EPS = 32, NC = 10, NCB = 7; };
template <> struct Fmt<2> { static constexpr int EPS = 16, NC = 5, NCB = 3; };
template <> struct Fmt<3> { static constexpr int EPS = 16, NC = 8, NCB = 8; };
template <> struct Fmt<4> { static constexpr int EPS = 8, NC = 2, NCB = 1; };
template <> struct Fmt<8> { static constexpr int EPS = 4, NC = 1, NCB = 1; };

template <int BITS, bool BF>
constexpr int ncons() { return BF ? Fmt<BITS>::NCB : Fmt<BITS>::NC; }

// Per (group, column) record in shared memory: the bias constants (duplicated
// fp16 / bf16 pairs; 8-bit bf16: one fp32), preceded by the fp32 scale and
// fractional zero part.  8-bit keeps "slim" records, the constant alone: the
// GEMV reads s and z from the raw s/z rows when a group ends, so the table is
// a quarter of the size.  On B200 that takes the 8192 x 8192 8-bit group-128
// decode plan from two CTAs per SM to three (25 us -> 14 us); the same for
// 4-bit would take the 4096 x 4096 decode plan from three to four CTAs per SM,
// which measured 4 % slower, so 4-bit keeps full records.
template <int BITS, bool BF>
constexpr bool slim_rec() { return BITS == 8; }

template <int BITS, bool BF, bool SLIM = slim_rec<BITS, BF>()> struct Rec;
template <int BITS, bool BF> struct alignas(16) Rec<BITS, BF, false> {
    float s;
    float zr;
    uint32_t c[ncons<BITS, BF>()];
};
template <int BITS, bool BF> struct Rec<BITS, BF, true> {
    uint32_t c[ncons<BITS, BF>()];
};

// ------------------------------------------------------------ element types
// x, scales, zeros, bias and y share one 16-bit type: fp16 (BF = false) or bf16.
template <bool BF> struct Dt;
template <> struct Dt<false> {
    static __device__ __forceinline__ float load(uint16_t v) { return __half2float(__ushort_as_half(v)); }
    static __device__ __forceinline__ uint16_t store(float v) { return __half_as_ushort(__float2half_rn(v)); }
    static __device__ __forceinline__ float2 pair(uint32_t u) {
        return __half22float2(*reinterpret_cast<const __half2*>(&u));
    }
};
template <> struct Dt<true> {
    static __device__ __forceinline__ float load(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }
    static __device__ __forceinline__ uint16_t store(float v) {
        return __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    static __device__ __forceinline__ float2 pair(uint32_t u) {
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
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

__device__ __forceinline__ uint32_t dup_bf16(float v) {
    const uint16_t b = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    return (uint32_t)b | ((uint32_t)b << 16);
}

template <bool BF>
__device__ __forceinline__ uint32_t dup_t(float v) { return BF ? dup_bf16(v) : dup_half(v); }

// bf16 pair j of a 3-bit word: the hi field sits at bit PH3(j) of its shifted
// copy, the lo bit at PL3(j).
__device__ __forceinline__ constexpr int ph3_bf(int j) { return 2 * (j % 3) + 1; }
__device__ __forceinline__ constexpr int pl3_bf(int j) { return j < 6 ? j + 1 : j - 5; }

// bf16 bias magnitude of constant i: 128 * 2^-p for a code at bit p of 0x4300
// (1-bit p = i; 2-bit p = 2 i; 4-bit p = 0).  3-bit: hi field at ph (multiplier
// 2^(1-ph)) and lo bit at pl (multiplier 2^-pl): 2^(8-ph) + 2^(7-pl).  With
// zi <= 2^bits - 1 every sum below has at most 8 significant bits.
template <int BITS>
__device__ __forceinline__ float bias_magnitude_bf(int i) {
    if constexpr (BITS == 1) {
        return (float)(128 >> i);
    } else if constexpr (BITS == 2) {
        return (float)(128 >> (2 * i));
    } else if constexpr (BITS == 4) {
        return 128.0f;
    } else {
        return (float)(1 << (8 - ph3_bf(i))) + (float)(1 << (7 - pl3_bf(i)));
    }
}

// The integer zero point the exact conversion subtracts; the rest, z - zi, is
// applied in fp32 (GEMV) or folded into the scale FMA (GEMM).
template <int BITS, bool BF>
__device__ __forceinline__ float zero_int(float z) {
    if constexpr (BF) return fminf(fmaxf(rintf(z), 0.0f), (float)((1 << BITS) - 1));
    else return fminf(fmaxf(rintf(z), -256.0f), 256.0f);
}

// Bias constant ci of a (group, column) whose integer zero point is zi.
template <int BITS, bool BF>
__device__ __forceinline__ uint32_t pair_const(int ci, float zi) {
    if constexpr (!BF) {
        return dup_half(-(bias_magnitude<BITS>(ci) + zi));
    } else if constexpr (BITS == 8) {
        return __float_as_uint(-(8388608.0f + zi));  // fp32: 2^23 + q minus 2^23 + zi
    } else {
        return dup_bf16(-(bias_magnitude_bf<BITS>(ci) + zi));
    }
}

// fp16x2 constant with the same value in both lanes (compile-time exact values).
__device__ __forceinline__ constexpr uint32_t h2c(uint32_t bits16) { return bits16 | (bits16 << 16); }

// fp16 bit patterns of 2^-p, p = 0..10
__device__ __forceinline__ constexpr uint32_t pow2neg_h(int p) { return (uint32_t)(15 - p) << 10; }

// bf16 bit patterns of 2^-p, p = 0..7
__device__ __forceinline__ constexpr uint32_t pow2neg_b(int p) { return (uint32_t)(127 - p) << 7; }

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

// ---------------------------------------------------- bf16 pair dequantisation
// A word and the shifted copies of it that pair_bf reads.
struct SrcB {
    uint32_t a, b, c, d;  // main plane copies
    uint32_t la, lb;      // 3-bit: lo plane copies
};

// 1-bit: w, w >> 7, w >> 14 (bits 0-6, 7-13, 14-15 of each half at bit 0);
// 2-bit: w, w >> 6, w >> 12; 4-bit: w, w >> 4, w >> 8, w >> 12; 8-bit: w.
// 3-bit: (hi << 1), hi >> 5, hi >> 11 put pair j's 2-bit field at bit
// 2 (j % 3) + 1; the lo bits of the hi word's 16 codes (selected by lo_sel
// as in prep_word) go to bit j + 1 (j < 6) or j - 5 (j >= 6).
template <int BITS>
__device__ __forceinline__ void prep_bf(uint32_t w, uint32_t lo_word, uint32_t lo_sel, SrcB& s) {
    s.a = w;
    s.b = s.c = s.d = s.la = s.lb = 0;
    if constexpr (BITS == 1) {
        s.b = w >> 7;
        s.c = w >> 14;
    } else if constexpr (BITS == 2) {
        s.b = w >> 6;
        s.c = w >> 12;
    } else if constexpr (BITS == 4) {
        s.b = w >> 4;
        s.c = w >> 8;
        s.d = w >> 12;
    } else if constexpr (BITS == 3) {
        s.a = w << 1;
        s.b = w >> 5;
        s.c = w >> 11;
        const uint32_t ls = prmt(lo_word, 0u, lo_sel);
        s.la = ls << 1;
        s.lb = ls >> 5;
    }
}

// Pair j (codes j and j + EPS/2 in the low / high half) as bf16x2 values q - zi.
template <int BITS>
__device__ __forceinline__ uint32_t pair_bf(const SrcB& s, const uint32_t (&c)[Fmt<BITS>::NCB], int j) {
    constexpr uint32_t MAGIC = 0x43004300u;
    if constexpr (BITS == 8) {
        // bytes j and j + 2 into the low byte of the fp32 constant 2^23 (0x4B000000)
        const float lo = __uint_as_float(prmt(s.a, 0x4B000000u, 0x7440u + j)) + __uint_as_float(c[0]);
        const float hi = __uint_as_float(prmt(s.a, 0x4B000000u, 0x7442u + j)) + __uint_as_float(c[0]);
        const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&v);
    } else if constexpr (BITS == 4) {
        const uint32_t src = j == 0 ? s.a : j == 1 ? s.b : j == 2 ? s.c : s.d;
        return bfma2_u32(and_or(src, 0x000F000Fu, MAGIC), h2c(pow2neg_b(0)), c[0]);
    } else if constexpr (BITS == 2) {
        const uint32_t src = j < 3 ? s.a : j < 6 ? s.b : s.c;
        const int i = j % 3;
        return bfma2_u32(and_or(src, 0x00030003u << (2 * i), MAGIC), h2c(pow2neg_b(2 * i)), c[i]);
    } else if constexpr (BITS == 1) {
        const uint32_t src = j < 7 ? s.a : j < 14 ? s.b : s.c;
        const int p = j % 7;
        return bfma2_u32(and_or(src, 0x00010001u << p, MAGIC), h2c(pow2neg_b(p)), c[p]);
    } else {
        const uint32_t srch = j < 3 ? s.a : j < 6 ? s.b : s.c;
        const uint32_t srcl = j < 6 ? s.la : s.lb;
        const int ph = ph3_bf(j), pl = pl3_bf(j);
        const uint32_t H = and_or(srch, 0x00030003u << ph, MAGIC);
        const uint32_t L = and_or(srcl, 0x00010001u << pl, MAGIC);
        const uint32_t T = bfma2_u32(H, h2c(pow2neg_b(ph - 1)), c[j]);
        return bfma2_u32(L, h2c(pow2neg_b(pl)), T);
    }
}

// ----------------------------------------------- one word, either element type
template <int BITS, bool BF> struct Word;
template <int BITS> struct Word<BITS, false> {
    uint32_t w, wh, ls;
    __device__ __forceinline__ void prep(uint32_t word, uint32_t lo_word, uint32_t lo_sel) {
        w = word;
        wh = ls = 0;
        prep_word<BITS>(w, wh, ls, lo_word, lo_sel);
    }
    __device__ __forceinline__ uint32_t pair(const uint32_t (&c)[Fmt<BITS>::NC], int j) const {
        return pair_q<BITS>(w, wh, ls, c, j);
    }
};
template <int BITS> struct Word<BITS, true> {
    SrcB s;
    __device__ __forceinline__ void prep(uint32_t word, uint32_t lo_word, uint32_t lo_sel) {
        prep_bf<BITS>(word, lo_word, lo_sel, s);
    }
    __device__ __forceinline__ uint32_t pair(const uint32_t (&c)[Fmt<BITS>::NCB], int j) const {
        return pair_bf<BITS>(s, c, j);
    }
};

}  // namespace wq
