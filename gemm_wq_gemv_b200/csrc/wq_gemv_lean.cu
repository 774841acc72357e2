// wq_gemv_lean.cu -- decode-time product y (M x N) = x (M x K) @ dequant(W_q) for
// 1 <= M <= 16 and 1-, 2-, 4- or 8-bit words, with a small shared-memory footprint.
//
// What is computed: dashq_kernel.py `_dashq_gemv_kernel` (one token there; up to
// 8 here): each output column n is sum_k x[k] * (q[k][n] - z[g][n]) * s[g][n],
// g = k / G, with fp32 accumulation and one rounding at the end.  x, s, z, the
// bias and y are all fp16 or all bf16.
//
// How (sm_100a).  The product reads every packed word once and is bound by
// HBM.  In a decode loop consecutive products overlap (programmatic dependent
// launch), and the time per product is set by how many bytes each SM keeps in
// flight while earlier products on the stream drain.  So shared memory holds
// only what is in flight: the weights and the s/z rows of the CTA.
//  * Work split.  A CTA of 8 warps owns 32 output columns and a K range (all of
//    K unless N is small; then a thread-block cluster splits K and sums its
//    partials through distributed shared memory).  A warp owns a run of quads
//    (4 word rows x 32 columns).
//  * Loads, all issued at kernel start.  Each warp requests its words with 2-D
//    TMA boxes (32 columns x R word rows, 128-byte swizzle, L2 evict-first)
//    into a ring of S slots; for the decode layers one box per warp covers its
//    whole range, so a CTA's words are all in flight at once.  Slots are
//    refilled as they are consumed when the range is longer.  One more TMA copy
//    brings the s and z rows of the CTA's groups.
//  * x is not staged: each lane reads the 16 (8-bit: 8, 2-bit: 32) bytes of x its word row
//    needs straight from global memory (L2-resident: every CTA reads the same
//    x), a group of quads ahead of their use, and permutes them into the MMA's
//    k order with PRMT.
//  * s and z: at the start of a group each lane turns the s and z of its 4
//    columns (two 8-byte shared-memory reads) into the conversion constants.
//  * Dequant and dot product (wq_dequant.cuh): a code pair becomes exact fp16 /
//    bf16 q - round(z) with one LOP3 and one FMA; those values are the A operand
//    of a warp MMA m16n8k16 with x as B.  Lane (g, t) (g = lane / 4, t = lane %
//    4) reads one 16-byte vector per quad, 4 adjacent columns of word row 4 q +
//    t; the chunk order keeps these reads free of bank conflicts.
//  * Per group, acc += s * (D - (z - round(z)) * X) in fp32, X = the sum of the
//    x values the warp's quads of that group cover (summed only when a zero
//    point of the group is fractional).
// Every mbarrier wait is bounded; on time-out the kernel records it in the
// GEMV's device status word and skips the rest of the warp's range.
#include <algorithm>
#include <cstddef>
#include <cstring>
#include <type_traits>

#include "wq_dequant.cuh"
#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {

// Device status of this kernel: 0, or 1 once a bounded wait ran out.
__device__ unsigned int g_gemv_lean_status = 0;

namespace {

constexpr int LCOLS = 32;  // output columns per CTA
constexpr int LWK = 8;     // warps per CTA (split along K)
constexpr int LMAXS = 4;   // ring slots per warp (at most)
constexpr uint64_t LWAIT_NS = 2000000000ull;

struct LeanParams {
    const uint16_t* x;
    const uint16_t* bias;  // (N,) or null
    uint16_t* y;
    int M, K, N, G;
    int Kw;         // word rows
    int Q;          // quads = ceil(Kw / 4)
    int QW;         // quads per warp (a multiple of the quads per box)
    int KS;         // CTAs per cluster along K (1: no cluster)
    int qpg;        // quads per group (a large number when one group spans K)
    int qpg_shift;  // log2(qpg) when qpg is a power of two, else -1
    int BQ;         // quads per TMA box (R = 4 BQ word rows)
    int S;          // ring slots per warp (a power of two)
    int sz_rows;    // s (and z) rows loaded per CTA: sz_box x (number of boxes)
    int sz_box;     // rows per s / z TMA box (<= 256)
    uint32_t off_sz;   // s rows (from the 1024-aligned base), then z rows at + sz_stride
    uint32_t sz_stride;  // sz_rows * 64 bytes rounded up to 128 (a TMA destination)
    uint32_t off_part, off_bar;
    uint32_t off_x;    // XS: the CTA's x slice, one row of xs_stride bytes per token
    uint32_t xs_stride;
    int late_wait;  // wait for the previous kernel only before writing y
};

// The x values of one word row: 16 bytes (4-bit; 8-bit: the first 8), 32
// bytes for the 16 values of a 2-bit word row, 64 for the 32 of a 1-bit one.
struct X16 {
    uint4 a, b;
};
struct X32 {
    uint4 a, b, c, d;
};
template <int EPS>
using XRow = std::conditional_t<(EPS == 32), X32, std::conditional_t<(EPS == 16), X16, uint4>>;

// The bytes of x that word row k0 / EPS needs, token row xr; zeros at and beyond K.
template <int EPS>
__device__ __forceinline__ XRow<EPS> ldg_x(const uint16_t* xr, int k0, int K) {
    const bool in = k0 < K;
    const uint16_t* src = xr + (in ? k0 : 0);  // a row past K reads row 0 and is zeroed below
    if constexpr (EPS == 32) {
        const uint4* v = reinterpret_cast<const uint4*>(src);
        X32 r{__ldg(v), __ldg(v + 1), __ldg(v + 2), __ldg(v + 3)};
        if (!in) r = X32{};
        return r;
    } else if constexpr (EPS == 16) {
        X16 r{__ldg(reinterpret_cast<const uint4*>(src)), __ldg(reinterpret_cast<const uint4*>(src) + 1)};
        if (!in) r = X16{};
        return r;
    } else {
        uint4 r;
        if constexpr (EPS == 8) {
            r = __ldg(reinterpret_cast<const uint4*>(src));
        } else {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
            r = make_uint4(v.x, v.y, 0u, 0u);
        }
        if (!in) r = make_uint4(0u, 0u, 0u, 0u);
        return r;
    }
}

// Conversion constants of a lane's 4 columns for one group, from the group's z
// values (uint2: columns 0-1 and 2-3 as 16-bit pairs).  fp16: two columns per
// fp16x2 instruction -- z is clamped to [-256, 256] and rounded to an integer by
// adding 1536 (fp16 spacing 1 on [1024, 2048), ties to even as rint, the same
// integer as zero_int), and the constants -(1024 + zi) and -(64 + zi) are
// differences of exact integers below 2048.  bf16: per column.
template <int BITS, bool BF>
struct GroupConsts {
    static constexpr int NC = ncons<BITS, BF>();
    uint32_t cc[4][NC];

    __device__ __forceinline__ void make(uint2 zv) {
        using T16 = Dt<BF>;
        if constexpr (!BF) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t z2 = h ? zv.y : zv.x;
                const uint32_t zc = hmin2_u32(hmax2_u32(z2, h2c(0xDC00u)), h2c(0x5C00u));  // [-256, 256]
                const uint32_t r = hadd2_u32(zc, h2c(0x6600u));                            // 1536 + zi
                const uint32_t c0 = hsub2_u32(h2c(0x6000u), r);  // 512 - 1536 - zi = -(1024 + zi)
                cc[2 * h][0] = prmt(c0, c0, 0x1010u);
                cc[2 * h + 1][0] = prmt(c0, c0, 0x3232u);
                if constexpr (BITS == 1) {  // -(1024 / 2^ci + zi) = (1536 - 1024 / 2^ci) - (1536 + zi), exact
                    constexpr uint32_t A[9] = {0x6400u, 0x6500u, 0x6580u, 0x65C0u, 0x65E0u,
                                               0x65F0u, 0x65F8u, 0x65FCu, 0x65FEu};  // 1024, 1280, ..., 1534
#pragma unroll
                    for (int ci = 1; ci < NC; ++ci) {
                        const uint32_t cx = hsub2_u32(h2c(A[ci - 1]), r);
                        cc[2 * h][ci] = prmt(cx, cx, 0x1010u);
                        cc[2 * h + 1][ci] = prmt(cx, cx, 0x3232u);
                    }
                } else if constexpr (BITS == 2) {  // -(1024 / 4^ci + zi) = (1536 - 1024 / 4^ci) - (1536 + zi), exact
                    constexpr uint32_t A[4] = {0x6500u, 0x65C0u, 0x65F0u, 0x65FCu};  // 1280, 1472, 1520, 1532
#pragma unroll
                    for (int ci = 1; ci < NC; ++ci) {
                        const uint32_t cx = hsub2_u32(h2c(A[ci - 1]), r);
                        cc[2 * h][ci] = prmt(cx, cx, 0x1010u);
                        cc[2 * h + 1][ci] = prmt(cx, cx, 0x3232u);
                    }
                } else if constexpr (NC > 1) {
                    const uint32_t c1 = hsub2_u32(h2c(0x65C0u), r);  // 1472 - 1536 - zi = -(64 + zi)
                    cc[2 * h][1] = prmt(c1, c1, 0x1010u);
                    cc[2 * h + 1][1] = prmt(c1, c1, 0x3232u);
                }
            }
        } else {
            const float2 z01 = T16::pair(zv.x), z23 = T16::pair(zv.y);
            const float zz[4] = {z01.x, z01.y, z23.x, z23.y};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float zi = zero_int<BITS, BF>(zz[c]);
#pragma unroll
                for (int ci = 0; ci < NC; ++ci) cc[c][ci] = pair_const<BITS, BF>(ci, zi);
            }
        }
    }
};

// ALIGNED: one box holds each warp's whole range (QW == BQ quads, all inside K)
// and groups start on the range's 4-quad blocks or hold 1 or 2 quads (1- and
// 2-bit words at group 128), so the main loop runs group by group without
// per-quad bookkeeping.
// XS: x is written by the previous kernel on the stream.  Every load that does
// not depend on it is issued and waited for first; after the grid dependency
// wait the CTA copies its slice of x into shared memory in one round trip, and
// the quads read it from there.
// TOK: 1 (one token), 8 (M <= 8) or 16 (M <= 16: two 8-token MMA tiles; not
// for 1-bit words, whose ten conversion constants per column leave no room).
template <int BITS, bool BF, int BQ, int TOK, bool ALIGNED, bool XS>
__global__ void __launch_bounds__(LWK * 32, (TOK > 8 || BITS == 1) ? 2 : 3)
gemv_lean_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                 const __grid_constant__ CUtensorMap tm_z, const LeanParams p) {
    using F = Fmt<BITS>;
    using T16 = Dt<BF>;
    constexpr int EPS = F::EPS;
    constexpr int MMAS = EPS / 4;  // MMAs per column pair per quad
    constexpr bool M1 = TOK == 1;
    constexpr int NT = TOK > 8 ? 2 : 1;  // 8-token MMA tiles
    constexpr int NE = M1 ? 1 : 2;       // tokens per lane and tile that can exist (2 t, 2 t + 1)
    constexpr uint32_t BOX_BYTES = (uint32_t)BQ * 4u * LCOLS * 4u;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base: the 128-byte swizzle of the TMA boxes repeats every 1024 bytes
    uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    // 16-byte column chunk of this lane (columns 4 cg .. 4 cg + 3): lanes g and
    // g + 1 of a quarter-warp differ in bit 2, which the row swizzle never
    // touches, so each quarter-warp's eight 16-byte reads hit distinct banks.
    const int cg = ((g & 1) << 2) | (g >> 1);
    const int rank = (int)blockIdx.y;  // the cluster spans the grid's y extent
    const int col0 = blockIdx.x * LCOLS;
    const int cta_q0 = rank * LWK * p.QW;
    const int q_begin = cta_q0 + warp * p.QW;
    const int nq = max(0, min(p.Q, q_begin + p.QW) - q_begin);
    // group of quad q (a shift for the usual power-of-two quads per group)
    auto gdiv = [&](int q) { return p.qpg_shift >= 0 ? (q >> p.qpg_shift) : q / p.qpg; };
    const int g_cta0 = gdiv(min(cta_q0, p.Q - 1));  // first group of the CTA's K range

    // ---- (1) every load of the CTA, issued first: the warp's words (boxes of BQ
    // quads into a ring of S slots) and, by warp 0, the s and z rows
    const int S = p.S;
    const uint32_t ring0 = smem_u32(smem) + (uint32_t)warp * (uint32_t)S * BOX_BYTES;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.off_bar) + warp * LMAXS;
    uint64_t* bar_sz = reinterpret_cast<uint64_t*>(smem + p.off_bar) + LWK * LMAXS;
    const int nbox = (nq + BQ - 1) / BQ;
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int b) {  // box b of this warp -> slot b % S
        const int slot = b & (S - 1);
        mbar_arrive_expect_tx(&bar[slot], BOX_BYTES);
        tma_load_2d_u32_hint(ring0 + (uint32_t)slot * BOX_BYTES, &tm_w, &bar[slot], col0, 4 * (q_begin + b * BQ),
                             pol);
    };
    const uint32_t sz_base = smem_u32(smem + p.off_sz);
    const uint32_t z_off = p.sz_stride;  // the z rows follow the s rows
    if (lane == 0) {
        for (int k = 0; k < S; ++k) mbar_init(&bar[k], 1);
        if (warp == 0) mbar_init(bar_sz, 1);
        fence_mbarrier_init();
        if (warp == 0) {
            const int nb = p.sz_rows / p.sz_box;
            mbar_arrive_expect_tx(bar_sz, 2u * (uint32_t)p.sz_rows * (LCOLS * 2u));
            for (int b = 0; b < nb; ++b) {
                const uint32_t d = sz_base + (uint32_t)(b * p.sz_box) * (LCOLS * 2u);
                tma_load_2d_u32(d, &tm_s, bar_sz, col0, g_cta0 + b * p.sz_box);
                tma_load_2d_u32(d + z_off, &tm_z, bar_sz, col0, g_cta0 + b * p.sz_box);
            }
        }
        for (int b = 0; b < S && b < nbox; ++b) issue(b);
    }
    __syncthreads();  // every mbarrier initialised before anyone waits on it
    // the next kernel on the stream may start now (it waits for this grid
    // before it touches anything this one writes)
    grid_launch_dependents();
    if (!XS && !p.late_wait) grid_dependency_wait();  // x may be the previous kernel's output

    // ---- (2) this lane's x: tokens g + 8 n (duplicates beyond M are harmless),
    // word row 4 i + t of the warp's quad i
    const uint16_t* xr[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) xr[n] = p.x + (M1 ? (size_t)0 : (size_t)min(g + 8 * n, p.M - 1) * (size_t)p.K);
    const int kx0 = (4 * q_begin + t) * EPS;
    // quads of this warp whose 4 word rows all lie inside K (the rest: the ragged end)
    const int nq_full = max(0, min(p.Kw / 4, q_begin + p.QW) - q_begin);

    // ---- (3) s and z.  Whether any zero point of the CTA's groups is
    // fractional is settled once, from the z rows in shared memory, and the
    // main loop is compiled for each case.
    bool ok_all = mbar_wait_bounded(bar_sz, 0, LWAIT_NS);
    if (!ok_all) atomicOr(&g_gemv_lean_status, 1u);
    ok_all = __all_sync(0xffffffffu, ok_all);
    const uint32_t sz_lane = sz_base + 2u * (uint32_t)(4 * cg);
    auto sz_addr = [&](int gi) {
        // the group's s / z row is one of the rows the CTA loaded
        if (!check(gi >= g_cta0 && gi - g_cta0 < p.sz_rows, &g_gemv_lean_status)) gi = g_cta0;
        return sz_lane + (LCOLS * 2u) * (uint32_t)(gi - g_cta0);
    };
    int gcur = gdiv(q_begin);
    // whether any zero point of the warp's groups is fractional (a warp vote)
    bool frac = false;
    if (ok_all && nq > 0) {
        const int g_last = gdiv(q_begin + nq - 1);
        const uint16_t* zt = reinterpret_cast<const uint16_t*>(smem + p.off_sz + z_off);
        for (int e = (gcur - g_cta0) * LCOLS + lane; e < (g_last - g_cta0 + 1) * LCOLS; e += 32) {
            const float z = T16::load(zt[e]);
            frac |= z != zero_int<BITS, BF>(z);
        }
    }
    frac = __any_sync(0xffffffffu, frac);
    GroupConsts<BITS, BF> k;
    uint2 sv = make_uint2(0u, 0u);  // the current group's s values of the lane's 4 columns
    auto consts = [&](int gi) {
        const uint32_t a = sz_addr(gi);
        sv = lds64_u32(a);
        k.make(lds64_u32(a + z_off));
    };
    int left = p.qpg - (q_begin - gcur * p.qpg);  // quads left in the current group
    if (ok_all && nq > 0) consts(gcur);

    // Per-lane offsets of this lane's 16-byte vector inside a slot: quad iq,
    // word row R = 4 iq + t, 16-byte chunk cg swizzled with (R & 7), whose
    // value only depends on the parity of iq.
    const uint32_t off_even = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)t) << 4);
    const uint32_t off_odd = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)(t + 4)) << 4);
    // XS: the weights, s and z are in flight or landed; now wait for the previous
    // kernel and copy the CTA's x slice (zeros past K) into shared memory
    const int kc0 = cta_q0 * 4 * EPS;  // first k of the CTA's range
    if constexpr (XS) {
        grid_dependency_wait();
        const int per_tok = LWK * p.QW * 4 * EPS / 8;  // 16-byte chunks of one token's slice
        for (int c = threadIdx.x; c < p.M * per_tok; c += LWK * 32) {
            const int m = c / per_tok, o = c - m * per_tok;
            const int kk = kc0 + 8 * o;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (kk < p.K) v = *reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + kk);  // K % 8 == 0
            if (check(m < p.M && 16u * (uint32_t)o + 16u <= p.xs_stride, &g_gemv_lean_status))
                *reinterpret_cast<uint4*>(smem + p.off_x + (size_t)m * p.xs_stride + 16 * o) = v;
        }
        __syncthreads();
    }
    uint32_t xs_lane[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n)
        xs_lane[n] = smem_u32(smem + p.off_x) + (uint32_t)(M1 ? 0 : min(g + 8 * n, p.M - 1)) * p.xs_stride +
                     2u * (uint32_t)(kx0 - kc0);
    // this lane's x values (token tile n) of quad i of the warp's range (all of its rows inside K)
    auto ldx = [&](int i, int n) {
        if constexpr (CHECKED) {  // the row lies inside K (and, staged, inside the CTA's slice)
            const int kl = kx0 + 4 * EPS * i;
            const bool ok = XS ? (kl - kc0 + EPS <= LWK * p.QW * 4 * EPS && (uint32_t)(kl - kc0 + EPS) * 2u <= p.xs_stride)
                               : (kl + EPS <= p.K);
            if (!check(ok, &g_gemv_lean_status)) return XRow<EPS>{};
        }
        if constexpr (EPS == 32) {  // 4 word rows = 128 values on per quad
            if constexpr (XS) {
                const uint32_t a = xs_lane[n] + 256u * i;
                return X32{lds128_u32(a), lds128_u32(a + 16u), lds128_u32(a + 32u), lds128_u32(a + 48u)};
            }
            const uint4* src = reinterpret_cast<const uint4*>(xr[n] + kx0) + 16 * i;
            return X32{__ldg(src), __ldg(src + 1), __ldg(src + 2), __ldg(src + 3)};
        } else if constexpr (EPS == 16) {  // 4 word rows = 64 values on per quad
            if constexpr (XS)
                return X16{lds128_u32(xs_lane[n] + 128u * i), lds128_u32(xs_lane[n] + 128u * i + 16u)};
            const uint4* src = reinterpret_cast<const uint4*>(xr[n] + kx0) + 8 * i;
            return X16{__ldg(src), __ldg(src + 1)};
        } else if constexpr (XS) {
            if constexpr (EPS == 8) return lds128_u32(xs_lane[n] + 64u * i);
            const uint2 v = lds64_u32(xs_lane[n] + 32u * i);
            return make_uint4(v.x, v.y, 0u, 0u);
        } else if constexpr (EPS == 8) {  // 4 word rows = 32 values on per quad
            return __ldg(reinterpret_cast<const uint4*>(xr[n] + kx0) + 4 * i);
        } else {                          // 16 values on per quad
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(xr[n] + kx0) + 4 * i);
            return make_uint4(v.x, v.y, 0u, 0u);
        }
    };
    // the same with a guard for rows past K (the ragged end of the range)
    auto ldx_guarded = [&](int i, int n) {
        if constexpr (XS) return ldx(i, n);  // the staged slice is zero past K
        return ldg_x<EPS>(xr[n], kx0 + 4 * EPS * i, p.K);
    };

    // ---- (4) main loop, FRAC: the CTA has fractional zero points
    float acc[4][NT][NE];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[c][n][e] = 0.0f;
    auto main_loop = [&](auto frac_tag) {
        constexpr bool FRAC = decltype(frac_tag)::value;
        float dsum[2][NT][4], xsum[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            xsum[n] = 0.0f;
#pragma unroll
            for (int T = 0; T < 2; ++T)
#pragma unroll
                for (int e = 0; e < 4; ++e) dsum[T][n][e] = 0.0f;
        }
        // fold the group's dot products into acc (scaled by s, fractional zero points applied)
        auto fold = [&]() {
            const float2 s01 = T16::pair(sv.x), s23 = T16::pair(sv.y);
            const float sc[4] = {s01.x, s01.y, s23.x, s23.y};
            float zr[4] = {0.0f, 0.0f, 0.0f, 0.0f}, X[NT][NE];
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < NE; ++e) X[n][e] = 0.0f;
            if constexpr (FRAC) {
                const uint2 zv = lds64_u32(sz_addr(gcur) + z_off);
                const float2 z01 = T16::pair(zv.x), z23 = T16::pair(zv.y);
                const float zz[4] = {z01.x, z01.y, z23.x, z23.y};
#pragma unroll
                for (int c = 0; c < 4; ++c) zr[c] = zz[c] - zero_int<BITS, BF>(zz[c]);
                // the x sum of token 8 n + 2 t + e over the group's quads of this warp
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    float tot = xsum[n] + __shfl_xor_sync(0xffffffffu, xsum[n], 1);
                    tot += __shfl_xor_sync(0xffffffffu, tot, 2);
#pragma unroll
                    for (int e = 0; e < NE; ++e) X[n][e] = __shfl_sync(0xffffffffu, tot, M1 ? 0 : 4 * (2 * t + e));
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int T = c >> 1, half = c & 1;
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        float d = dsum[T][n][2 * half + e];
                        if constexpr (FRAC) d = fmaf(-zr[c], X[n][e], d);
                        acc[c][n][e] = fmaf(sc[c], d, acc[c][n][e]);
                    }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                xsum[n] = 0.0f;
#pragma unroll
                for (int T = 0; T < 2; ++T)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dsum[T][n][e] = 0.0f;
            }
        };
        // one quad: the words hv (this lane's 16 bytes) and its x values xa[n]
        auto quad = [&](const uint4& hv, const XRow<EPS> (&xa)[NT]) {
            uint32_t bx[NT][EPS / 2];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if constexpr (EPS == 32) {  // pairs (j, j + 16) of the row's 32 values
                    const uint32_t lo[8] = {xa[n].a.x, xa[n].a.y, xa[n].a.z, xa[n].a.w,
                                            xa[n].b.x, xa[n].b.y, xa[n].b.z, xa[n].b.w};
                    const uint32_t hi[8] = {xa[n].c.x, xa[n].c.y, xa[n].c.z, xa[n].c.w,
                                            xa[n].d.x, xa[n].d.y, xa[n].d.z, xa[n].d.w};
#pragma unroll
                    for (int j = 0; j < 16; ++j) bx[n][j] = prmt(lo[j >> 1], hi[j >> 1], (j & 1) ? 0x7632u : 0x5410u);
                    if constexpr (FRAC) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float2 f = T16::pair(lo[u]), h = T16::pair(hi[u]);
                            xsum[n] += (f.x + f.y) + (h.x + h.y);
                        }
                    }
                } else if constexpr (EPS == 16) {  // pairs (j, j + 8) of the row's 16 values
                    const uint32_t lo[4] = {xa[n].a.x, xa[n].a.y, xa[n].a.z, xa[n].a.w};
                    const uint32_t hi[4] = {xa[n].b.x, xa[n].b.y, xa[n].b.z, xa[n].b.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) bx[n][j] = prmt(lo[j >> 1], hi[j >> 1], (j & 1) ? 0x7632u : 0x5410u);
                    if constexpr (FRAC) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 f = T16::pair(lo[u]), h = T16::pair(hi[u]);
                            xsum[n] += (f.x + f.y) + (h.x + h.y);
                        }
                    }
                } else {
                    if constexpr (EPS == 8) {  // pairs (0, 4), (1, 5), (2, 6), (3, 7) of the row's 8 values
                        bx[n][0] = prmt(xa[n].x, xa[n].z, 0x5410u);
                        bx[n][1] = prmt(xa[n].x, xa[n].z, 0x7632u);
                        bx[n][2] = prmt(xa[n].y, xa[n].w, 0x5410u);
                        bx[n][3] = prmt(xa[n].y, xa[n].w, 0x7632u);
                    } else {                   // pairs (0, 2), (1, 3) of the row's 4 values
                        bx[n][0] = prmt(xa[n].x, xa[n].y, 0x5410u);
                        bx[n][1] = prmt(xa[n].x, xa[n].y, 0x7632u);
                    }
                    if constexpr (FRAC) {  // this lane's row sum of x (fp32)
                        const uint32_t xv[4] = {xa[n].x, xa[n].y, xa[n].z, xa[n].w};
#pragma unroll
                        for (int u = 0; u < EPS / 2; ++u) {
                            const float2 f = T16::pair(xv[u]);
                            xsum[n] += f.x + f.y;
                        }
                    }
                }
            }
            const uint32_t wv[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int T = 0; T < 2; ++T) {
                Word<BITS, BF> WA, WB;
                WA.prep(wv[2 * T], 0u, 0u);
                WB.prep(wv[2 * T + 1], 0u, 0u);
#pragma unroll
                for (int h = 0; h < MMAS; ++h) {
                    uint32_t a[4];
                    a[0] = WA.pair(k.cc[2 * T], 2 * h);
                    a[1] = WB.pair(k.cc[2 * T + 1], 2 * h);
                    a[2] = WA.pair(k.cc[2 * T], 2 * h + 1);
                    a[3] = WB.pair(k.cc[2 * T + 1], 2 * h + 1);
#pragma unroll
                    for (int n = 0; n < NT; ++n) mma_16816<BF>(dsum[T][n], a, bx[n][2 * h], bx[n][2 * h + 1]);
                }
            }
        };
        // the four quads i4 .. i4 + 3 of a slot, quads i .. i + 3 of the warp
        auto block = [&](uint32_t slot_addr, int i4, int i) {
            const uint32_t wblk = slot_addr + 512u * (uint32_t)i4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                XRow<EPS> xa[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) xa[n] = ldx(i + j, n);
                quad(lds128_u32(wblk + 512u * j + ((j & 1) ? off_odd : off_even)), xa);
            }
        };
        // CNT (1 or 2) quads from quad i of the slot (a group of 1- or 2-bit words)
        auto block_short = [&](auto cnt_tag, uint32_t slot_addr, int i) {
            constexpr int CNT = decltype(cnt_tag)::value;
#pragma unroll
            for (int j = 0; j < CNT; ++j) {
                XRow<EPS> xa[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) xa[n] = ldx(i + j, n);
                quad(lds128_u32(slot_addr + 512u * (uint32_t)(i + j) + (((i + j) & 1) ? off_odd : off_even)), xa);
            }
        };

        if constexpr (ALIGNED) {
            if (ok_all && nq > 0) {
                const bool good = mbar_wait_bounded(&bar[0], 0u, LWAIT_NS);
                if (!good) atomicOr(&g_gemv_lean_status, 1u);
                ok_all = __all_sync(0xffffffffu, good);
            }
            if (!ok_all || nq == 0) return;
            const int seg = min(p.qpg, BQ);  // quads per group, or the whole range inside one group
#pragma unroll 1
            for (int q0 = 0; q0 < BQ; q0 += seg) {
                if (q0 > 0) consts(gcur);
                if (seg >= 4) {
#pragma unroll 1
                    for (int i = q0; i < q0 + seg; i += 4) block(ring0, i, i);
                } else if (seg == 2) {
                    block_short(std::integral_constant<int, 2>{}, ring0, q0);
                } else {
                    block_short(std::integral_constant<int, 1>{}, ring0, q0);
                }
                fold();
                ++gcur;
            }
        } else {
            // end of a group: fold, then the next group's constants
            auto group_end = [&](int i) {
                fold();
                left = p.qpg;
                ++gcur;
                if (i + 1 < nq) consts(gcur);
            };
            for (int b = 0; b < nbox && ok_all; ++b) {
                const int slot = b & (S - 1);
                const bool good = mbar_wait_bounded(&bar[slot], (uint32_t)((b / S) & 1), LWAIT_NS);
                if (!good) atomicOr(&g_gemv_lean_status, 1u);
                if (!__all_sync(0xffffffffu, good)) {  // give up this warp's range
                    ok_all = false;
                    break;
                }
                const uint32_t slot_addr = ring0 + (uint32_t)slot * BOX_BYTES;
                const int i0 = b * BQ;
#pragma unroll 1
                for (int i4 = 0; i4 < BQ && i0 + i4 < nq; i4 += 4) {
                    const int i = i0 + i4;
                    if (i + 4 <= nq_full && left >= 4) {  // four whole quads inside one group
                        block(slot_addr, i4, i);
                        left -= 4;
                        if (left == 0) group_end(i + 3);
                    } else {  // ragged end of the range, or groups shorter than four quads
                        const uint32_t wblk = slot_addr + 512u * (uint32_t)i4;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (i + j < nq) {
                                XRow<EPS> xa[NT];
#pragma unroll
                                for (int n = 0; n < NT; ++n) xa[n] = ldx_guarded(i + j, n);
                                quad(lds128_u32(wblk + 512u * j + ((j & 1) ? off_odd : off_even)), xa);
                                if (--left == 0) group_end(i + j);
                            }
                        }
                    }
                }
                // every lane has read this slot: refill it with box b + S
                __syncwarp();
                if (lane == 0 && b + S < nbox) {
                    fence_proxy_async_smem();
                    issue(b + S);
                }
            }
            if (ok_all && nq > 0 && left != p.qpg) fold();  // the warp's range ended inside a group
        }
    };
    if (frac)
        main_loop(std::true_type{});
    else
        main_loop(std::false_type{});

    // ---- (5) reduce over the warps of the CTA (and the CTAs of the cluster), write y.
    // Each warp's partials go to the first slot of its own ring, which it has consumed.
    const int nout = p.M * LCOLS;
    {
        float* red = reinterpret_cast<float*>(smem + (size_t)warp * S * BOX_BYTES);  // [M][LCOLS]
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < NE; ++e) {
                    const int m = 8 * n + 2 * t + e;
                    if (m < p.M && check((uint32_t)(m * LCOLS + LCOLS) * 4u <= S * BOX_BYTES, &g_gemv_lean_status))
                        red[m * LCOLS + 4 * cg + c] = acc[c][n][e];
                }
    }
    __syncthreads();
    auto warp_sum = [&](int i) {
        float v[LWK];
#pragma unroll
        for (int w = 0; w < LWK; ++w) v[w] = reinterpret_cast<const float*>(smem + (size_t)w * S * BOX_BYTES)[i];
#pragma unroll
        for (int h = LWK / 2; h >= 1; h >>= 1)
#pragma unroll
            for (int w = 0; w < h; ++w) v[w] += v[w + h];
        return v[0];
    };
    auto store = [&](int i, float v) {
        const int m = i / LCOLS, col = col0 + i % LCOLS;
        if (col < p.N && check(m < p.M, &g_gemv_lean_status)) {
            const float bv = p.bias ? T16::load(p.bias[col]) : 0.0f;
            p.y[(size_t)m * p.N + col] = T16::store(v + bv);
        }
    };
    if (p.KS > 1) {
        float* part = reinterpret_cast<float*>(smem + p.off_part);  // [M][LCOLS]
        for (int i = threadIdx.x; i < nout; i += LWK * 32) part[i] = warp_sum(i);
        cluster_sync();  // every CTA's partials are complete and visible
        if (p.late_wait) grid_dependency_wait();
        const uint32_t part_addr = smem_u32(part);
        for (int i = rank + p.KS * (int)threadIdx.x; i < nout; i += p.KS * LWK * 32) {
            float v = 0.0f;
            for (int r = 0; r < p.KS; ++r) v += ld_shared_cluster_f32(map_shared_rank(part_addr + 4u * i, r));
            store(i, v);
        }
        cluster_sync();  // peers keep their shared memory until every read is done
    } else {
        for (int i = threadIdx.x; i < nout; i += LWK * 32) {
            const float v = warp_sum(i);
            if (p.late_wait) grid_dependency_wait();  // a no-op after the first time
            store(i, v);
        }
    }
}

// One token, 4-bit fp16 words, groups of 128 (four quads), one TMA box per warp
// (QW = 8 or 16 quads), no cluster: the decode layers.  The same product as
// gemv_lean_kernel, written group by group with every loop bound known at
// compile time; it measured 2.15 us per overlapped 4096 x 4096 product against
// 2.73 us for the general kernel on B200 (the general kernel's bookkeeping for
// ragged ranges, other group sizes and up to 16 tokens costs issue slots that
// this shape does not need).  A warp whose groups hold a fractional zero point
// runs the second loop, which also sums x over each group.
template <int QW>
__global__ void __launch_bounds__(LWK * 32, 3)
gemv_decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_z, const LeanParams p) {
    constexpr uint32_t STAGE = (uint32_t)QW * 4u * LCOLS * 4u;  // one warp's words
    constexpr int GPW = QW / 4;                                  // groups per warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int cg = ((g & 1) << 2) | (g >> 1);
    const int col0 = blockIdx.x * LCOLS;
    const uint32_t st = smem_u32(sm) + (uint32_t)warp * STAGE;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + p.off_bar);
    const uint32_t sz_base = smem_u32(sm + p.off_sz);
    if (lane == 0) {
        mbar_init(&bar[warp], 1);
        if (warp == 0) mbar_init(&bar[LWK], 1);
        fence_mbarrier_init();
        if (warp == 0) {  // the s and z rows of the CTA's groups, first in line
            mbar_arrive_expect_tx(&bar[LWK], 2u * (uint32_t)p.sz_rows * (LCOLS * 2u));
            tma_load_2d_u32(sz_base, &tm_s, &bar[LWK], col0, 0);
            tma_load_2d_u32(sz_base + p.sz_stride, &tm_z, &bar[LWK], col0, 0);
        }
        mbar_arrive_expect_tx(&bar[warp], STAGE);
        tma_load_2d_u32_hint(st, &tm_w, &bar[warp], col0, 4 * QW * warp, policy_evict_first());
    }
    __syncthreads();  // every mbarrier initialised before anyone waits on it
    grid_launch_dependents();
    const uint32_t off_even = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)t) << 4);
    const uint32_t off_odd = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)(t + 4)) << 4);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    bool good = mbar_wait_bounded(&bar[LWK], 0, LWAIT_NS) && mbar_wait_bounded(&bar[warp], 0, LWAIT_NS);
    if (!good) atomicOr(&g_gemv_lean_status, 1u);
    good = __all_sync(0xffffffffu, good);
    const uint16_t* xg = p.x + 8 * (4 * QW * warp + t);  // word row 4 iq + t of the warp's quad iq
    // s of the lane's 4 columns for group gl of the warp at sz, z at + sz_stride
    const uint32_t sz = sz_base + 2u * (uint32_t)(GPW * warp * LCOLS + 4 * cg);
    bool frac = false;  // a fractional zero point among the warp's groups
    if (good) {
        const uint16_t* zt = reinterpret_cast<const uint16_t*>(sm + p.off_sz + p.sz_stride) + GPW * warp * LCOLS;
#pragma unroll
        for (int e = 0; e < GPW; ++e) {
            const float z = __half2float(__ushort_as_half(zt[e * LCOLS + lane]));
            frac |= z != zero_int<4, false>(z);
        }
    }
    frac = __any_sync(0xffffffffu, frac);
    auto run = [&](auto frac_tag) {
        constexpr bool FRAC = decltype(frac_tag)::value;
#pragma unroll 1
        for (int gl = 0; gl < GPW; ++gl) {
            const uint2 sv = lds64_u32(sz + 64u * gl), zv = lds64_u32(sz + p.sz_stride + 64u * gl);
            uint32_t cc[4][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t z2 = h ? zv.y : zv.x;
                const uint32_t zc = hmin2_u32(hmax2_u32(z2, h2c(0xDC00u)), h2c(0x5C00u));  // [-256, 256]
                const uint32_t r = hadd2_u32(zc, h2c(0x6600u));                            // 1536 + zi
                const uint32_t c0 = hsub2_u32(h2c(0x6000u), r);  // -(1024 + zi)
                const uint32_t c1 = hsub2_u32(h2c(0x65C0u), r);  // -(64 + zi)
                cc[2 * h][0] = prmt(c0, c0, 0x1010u);
                cc[2 * h + 1][0] = prmt(c0, c0, 0x3232u);
                cc[2 * h][1] = prmt(c1, c1, 0x1010u);
                cc[2 * h + 1][1] = prmt(c1, c1, 0x3232u);
            }
            float dsum[2][4] = {};
            float xsum = 0.0f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int iq = 4 * gl + qq;
                const uint4 hv = lds128_u32(st + 512 * iq + ((qq & 1) ? off_odd : off_even));
                uint4 a;  // (volatile: the load stays at the start of its quad)
                asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w)
                             : "l"(xg + 32 * iq));
                uint32_t bx[4];  // pairs (0, 4), (1, 5), (2, 6), (3, 7) of the row's 8 values
                bx[0] = prmt(a.x, a.z, 0x5410u);
                bx[1] = prmt(a.x, a.z, 0x7632u);
                bx[2] = prmt(a.y, a.w, 0x5410u);
                bx[3] = prmt(a.y, a.w, 0x7632u);
                if constexpr (FRAC) {
                    const uint32_t xv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xv[u]));
                        xsum += f.x + f.y;
                    }
                }
                const uint32_t wv[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int T = 0; T < 2; ++T) {
                    Word<4, false> WA, WB;
                    WA.prep(wv[2 * T], 0u, 0u);
                    WB.prep(wv[2 * T + 1], 0u, 0u);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t aa[4];
                        aa[0] = WA.pair(cc[2 * T], 2 * h);
                        aa[1] = WB.pair(cc[2 * T + 1], 2 * h);
                        aa[2] = WA.pair(cc[2 * T], 2 * h + 1);
                        aa[3] = WB.pair(cc[2 * T + 1], 2 * h + 1);
                        mma_16816<false>(dsum[T], aa, bx[2 * h], bx[2 * h + 1]);
                    }
                }
            }
            const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
            const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
            float d[4] = {dsum[0][0], dsum[0][2], dsum[1][0], dsum[1][2]};
            if constexpr (FRAC) {  // acc += s (D - (z - zi) X), X the group's x sum over the warp's rows
                float X = xsum + __shfl_xor_sync(0xffffffffu, xsum, 1);
                X += __shfl_xor_sync(0xffffffffu, X, 2);
                X = __shfl_sync(0xffffffffu, X, 0);
                const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&zv.x));
                const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&zv.y));
                const float zz[4] = {z01.x, z01.y, z23.x, z23.y};
#pragma unroll
                for (int c = 0; c < 4; ++c) d[c] = fmaf(-(zz[c] - zero_int<4, false>(zz[c])), X, d[c]);
            }
            acc[0] = fmaf(s01.x, d[0], acc[0]);
            acc[1] = fmaf(s01.y, d[1], acc[1]);
            acc[2] = fmaf(s23.x, d[2], acc[2]);
            acc[3] = fmaf(s23.y, d[3], acc[3]);
        }
    };
    if (good) {
        if (frac)
            run(std::true_type{});
        else
            run(std::false_type{});
    }
    // reduce over the 8 warps: each warp's partials into its own (consumed) stage
    __syncwarp();
    float* red = reinterpret_cast<float*>(sm + warp * STAGE);
    if (t == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) red[4 * cg + c] = acc[c];
    }
    __syncthreads();
    if (warp == 0) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < LWK; ++w) v += reinterpret_cast<const float*>(sm + w * STAGE)[lane];
        const int col = col0 + lane;
        if (col < p.N) {
            if (p.bias) v += __half2float(__ushort_as_half(p.bias[col]));
            if (p.late_wait) grid_dependency_wait();
            p.y[col] = __half_as_ushort(__float2half_rn(v));
        }
    }
}

static_assert(3 * sizeof(CUtensorMap) + sizeof(LeanParams) <= sizeof(Prepared::args), "prepared launch arguments");

// Shared-memory plan of one launch: the rings, the s / z rows, the cluster
// partials and the mbarriers.
size_t lean_layout(LeanParams& p, bool xs) {
    size_t off = (size_t)LWK * p.S * p.BQ * 4 * LCOLS * 4;  // the rings (1024-byte multiples)
    p.off_sz = (uint32_t)off;
    p.sz_stride = ((uint32_t)p.sz_rows * LCOLS * 2u + 127u) & ~127u;
    off += (size_t)p.sz_stride + (size_t)p.sz_rows * LCOLS * 2;
    off = (off + 15) & ~(size_t)15;
    p.off_part = (uint32_t)off;
    off += (size_t)p.M * LCOLS * 4;
    off = (off + 7) & ~(size_t)7;
    p.off_bar = (uint32_t)off;
    off += (size_t)(LWK * LMAXS + 1) * 8;
    off = (off + 15) & ~(size_t)15;
    p.off_x = (uint32_t)off;
    off += xs ? (size_t)p.M * p.xs_stride : 0;
    return off + 1024;  // slack for aligning the base to 1024 bytes
}

template <int BITS, bool BF, int BQ, int TOK, bool ALIGNED, bool XS>
wq_status launch_lean(const CUtensorMap& mw, const CUtensorMap& ms, const CUtensorMap& mz, const LeanParams& p,
                      size_t smem, const Problem& pb, cudaStream_t stream, Prepared* prep) {
    auto kern = gemv_lean_kernel<BITS, BF, BQ, TOK, ALIGNED, XS>;
    // context the smem limit was raised in, one per kernel this function launches
    static std::atomic<uint64_t> attr_ctx_lean[MAX_DEVICES], attr_ctx_decode[MAX_DEVICES];
    std::atomic<uint64_t>* attr_ctx = attr_ctx_lean;
    if constexpr (BITS == 4 && !BF && TOK == 1 && ALIGNED && !XS) {
        // the decode layers: one token, groups of 128, one box per warp, no cluster,
        // one s / z box from group 0
        if (p.KS == 1 && p.S == 1 && p.QW == BQ && p.qpg == 4 && p.sz_rows == p.sz_box && p.sz_rows == 2 * BQ) {
            kern = gemv_decode_kernel<BQ>;
            attr_ctx = attr_ctx_decode;
        }
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (const wq_status st = ensure_smem_attr((const void*)kern, 227 * 1024, attr_ctx, dev); st != WQ_OK) return st;
    if (prep) {  // record the launch instead of making it
        Prepared& r = *prep;
        r.kern = (const void*)kern;
        r.grid = dim3((pb.N + LCOLS - 1) / LCOLS, p.KS, 1);
        r.block = dim3(LWK * 32, 1, 1);
        r.smem = smem;
        r.cluster_y = p.KS > 1 ? (unsigned)p.KS : 1u;
        r.pdl = (pb.flags & (WQ_FLAG_PDL | WQ_FLAG_PDL_INPUTS_READY)) != 0;
        r.nargs = 4;
        const size_t mo = sizeof(CUtensorMap);
        std::memcpy(r.args, &mw, mo);
        std::memcpy(r.args + mo, &ms, mo);
        std::memcpy(r.args + 2 * mo, &mz, mo);
        std::memcpy(r.args + 3 * mo, &p, sizeof(p));
        r.arg_off[0] = 0; r.arg_off[1] = mo; r.arg_off[2] = 2 * mo; r.arg_off[3] = 3 * mo;
        r.x_off = 3 * mo + offsetof(LeanParams, x);
        r.y_off = 3 * mo + offsetof(LeanParams, y);
        return WQ_OK;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((pb.N + LCOLS - 1) / LCOLS, p.KS, 1);
    cfg.blockDim = dim3(LWK * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (p.KS > 1) {  // a cluster of one CTA is no cluster: launch without the attribute
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = p.KS;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pb.flags & (WQ_FLAG_PDL | WQ_FLAG_PDL_INPUTS_READY)) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, mw, ms, mz, p));
}

template <int BITS, bool BF>
wq_status run_lean(const Problem& pb, cudaStream_t stream, Prepared* prep) {
    constexpr int EPS = Fmt<BITS>::EPS;
    constexpr int QK = 4 * EPS;
    LeanParams p{};
    p.x = pb.x; p.bias = pb.bias; p.y = pb.y;
    p.M = pb.M; p.K = pb.K; p.N = pb.N; p.G = pb.G;
    p.late_wait = (pb.flags & WQ_FLAG_PDL_INPUTS_READY) ? 1 : 0;
    p.Kw = pb.K / EPS;
    p.Q = (p.Kw + 3) / 4;
    p.qpg = (pb.G == pb.K) ? (1 << 29) : pb.G / QK;
    p.qpg_shift = -1;
    for (int sh = 0; sh < 30; ++sh)
        if (p.qpg == (1 << sh)) p.qpg_shift = sh;
    const int n_groups = (pb.K + pb.G - 1) / pb.G;
    const int colblocks = (pb.N + LCOLS - 1) / LCOLS;
    const int sms = sm_count();
    // Split K over a cluster only when the column blocks leave most SMs idle.
    int KS = 1;
    while (KS < 8 && colblocks * KS * 2 <= sms && LWK * KS * 2 <= p.Q) KS *= 2;
    p.KS = KS;
    const int qw = (p.Q + LWK * KS - 1) / (LWK * KS);  // quads per warp before rounding to boxes
    // Ring: up to 8 KB of words in flight per warp.  One box of 16 (or 8) quads
    // covers the warp's range when it fits -- all of a CTA's words requested at
    // once -- else two slots of 8 quads stream it.
    int BQ;
    if (qw <= 8) {
        BQ = 8;
        p.S = 1;
    } else if (qw <= 16) {
        BQ = 16;
        p.S = 1;
    } else {
        BQ = 8;
        p.S = 2;
    }
    p.BQ = BQ;
    p.QW = (qw + BQ - 1) / BQ * BQ;
    // s / z rows a CTA's quads touch (at most): from the group of its first quad
    // to the group of its last
    int rows = 1;
    for (int r = 0; r < KS; ++r) {
        const int q0 = r * LWK * p.QW;
        if (q0 >= p.Q) break;
        const int q1 = std::min(p.Q, q0 + LWK * p.QW) - 1;
        rows = std::max(rows, q1 / p.qpg - q0 / p.qpg + 1);
    }
    rows = std::min(rows, n_groups);
    p.sz_box = std::min(rows, 256);
    p.sz_rows = (rows + p.sz_box - 1) / p.sz_box * p.sz_box;
    // x written by the previous kernel (WQ_FLAG_PDL): stage it once per CTA
    const bool xs = (pb.flags & WQ_FLAG_PDL) && !(pb.flags & WQ_FLAG_PDL_INPUTS_READY);
    p.xs_stride = (uint32_t)(LWK * p.QW * 4 * EPS * 2) + (pb.M > 1 ? 16u : 0u);  // pad: tokens on other banks
    const size_t smem = lean_layout(p, xs);
    if (smem > 227 * 1024) return WQ_ERR_UNSUPPORTED;

    CUtensorMap mw, ms, mz;
    bool ok = make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_q, pb.N, p.Kw, (uint64_t)pb.N * 4, LCOLS, 4 * BQ,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.scales, pb.N, n_groups, (uint64_t)pb.N * 2, LCOLS,
                        p.sz_box, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_map(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.zeros, pb.N, n_groups, (uint64_t)pb.N * 2, LCOLS,
                        p.sz_box, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return WQ_ERR_CUDA;
    // ALIGNED: one box per warp covering its QW quads, every warp of every rank
    // full and inside K, and groups starting on 4-quad blocks of the ranges
    const bool aligned = p.S == 1 && p.QW == BQ && p.Q == KS * LWK * p.QW && p.Kw == 4 * p.Q &&
                         ((p.qpg <= p.QW && p.QW % p.qpg == 0 && (p.qpg % 4 == 0 || p.qpg <= 2)) ||
                          (p.qpg > p.QW && (p.qpg % p.QW == 0 || p.qpg >= p.Q)));
    auto go = [&](auto bq, auto a) {
        constexpr int B = decltype(bq)::value;
        constexpr bool A = decltype(a)::value;
        auto tok = [&](auto xs_tag) {
            constexpr bool X = decltype(xs_tag)::value;
            if (pb.M == 1) return launch_lean<BITS, BF, B, 1, A, X>(mw, ms, mz, p, smem, pb, stream, prep);
            if (pb.M <= 8) return launch_lean<BITS, BF, B, 8, A, X>(mw, ms, mz, p, smem, pb, stream, prep);
            if constexpr (BITS == 1) return WQ_ERR_UNSUPPORTED;  // two 1-bit token tiles spill: not routed here
            else return launch_lean<BITS, BF, B, 16, A, X>(mw, ms, mz, p, smem, pb, stream, prep);
        };
        return xs ? tok(std::true_type{}) : tok(std::false_type{});
    };
    using I16 = std::integral_constant<int, 16>;
    using I8 = std::integral_constant<int, 8>;
    if (BQ == 16) return aligned ? go(I16{}, std::true_type{}) : go(I16{}, std::false_type{});
    return aligned ? go(I8{}, std::true_type{}) : go(I8{}, std::false_type{});
}

}  // namespace

wq_status gemv_lean_device_status(int reset) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_gemv_lean_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_gemv_lean_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return (v & 1u) ? WQ_ERR_TIMEOUT : (v & 2u) ? WQ_ERR_CHECK : WQ_OK;
}

bool gemv_lean_takes(const Problem& p) {
    if (p.bits == 3) return false;
    if (p.M > (p.bits == 1 ? 8 : 16)) return false;  // 1-bit with two token tiles would spill registers
    // x written by the previous kernel on the stream: the staged copy of x is
    // read in 16-byte rows
    if ((p.flags & WQ_FLAG_PDL) && !(p.flags & WQ_FLAG_PDL_INPUTS_READY) && p.K % 8 != 0) return false;
    const int qk = 4 * (32 / p.bits);
    return p.G == p.K || p.G % qk == 0;
}

wq_status launch_gemv_lean(const Problem& p, cudaStream_t s, Prepared* prep) {
    const bool bf = (p.flags & WQ_FLAG_BF16) != 0;
    switch (p.bits) {
        case 1: return bf ? run_lean<1, true>(p, s, prep) : run_lean<1, false>(p, s, prep);
        case 2: return bf ? run_lean<2, true>(p, s, prep) : run_lean<2, false>(p, s, prep);
        case 4: return bf ? run_lean<4, true>(p, s, prep) : run_lean<4, false>(p, s, prep);
        case 8: return bf ? run_lean<8, true>(p, s, prep) : run_lean<8, false>(p, s, prep);
        default: return WQ_ERR_UNSUPPORTED;
    }
}

}  // namespace wq
