// wq_gemv_lean.cu -- decode-time product y (M x N) = x (M x K) @ dequant(W_q) for
// 1 <= M <= 8 and 4- or 8-bit words, with a small shared-memory footprint.
//
// What is computed: dashq_kernel.py `_dashq_gemv_kernel` (one token there; up to
// 8 here): each output column n is sum_k x[k] * (q[k][n] - z[g][n]) * s[g][n],
// g = k / G, with fp32 accumulation and one rounding at the end.  x, s, z, the
// bias and y are all fp16 or all bf16.
//
// How (sm_100a).  The product reads every packed word once and is bound by
// HBM.  In a decode loop consecutive products overlap (programmatic dependent
// launch), and the time per product is set by how many bytes each SM keeps in
// flight while earlier products on the stream drain.  So every byte of shared
// memory a CTA holds is there to carry weights in flight:
//  * Work split.  A CTA of 8 warps owns 32 output columns and a K range (all of
//    K unless N is small; then a thread-block cluster splits K and sums its
//    partials through distributed shared memory).  A warp owns a run of quads
//    (4 word rows x 32 columns).
//  * Loads.  At kernel start each warp requests its words with 2-D TMA boxes
//    (32 columns x R word rows, 128-byte swizzle, L2 evict-first) into a ring of
//    S slots; for the decode layers one box per warp covers its whole range, so
//    a CTA's words are all in flight at once.  Slots are refilled as they are
//    consumed when the range is longer.
//  * s and z.  Each lane reads the s and z of its 4 columns (8 bytes each) one
//    group ahead from global memory and turns them into the conversion constants
//    itself: no table in shared memory and no barrier before the first product.
//  * Dequant and dot product (wq_dequant.cuh): a code pair becomes exact fp16 /
//    bf16 q - round(z) with one LOP3 and one FMA; those values are the A operand
//    of a warp MMA m16n8k16 with x (staged once per CTA in shared memory, in the
//    matching k order) as B.  Lane (g, t) (g = lane / 4, t = lane % 4) reads one
//    16-byte vector per quad, 4 adjacent columns of word row 4 q + t; the chunk
//    order keeps these reads free of bank conflicts.
//  * Per group, acc += s * (D - (z - round(z)) * X) in fp32, X = the sum of the
//    x values the warp's quads of that group cover (read from per-quad sums in
//    shared memory only when a zero point of the group is fractional).
// Every mbarrier wait is bounded; on time-out the kernel records it in the
// GEMV's device status word and skips the rest of the warp's range.
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
// Independent MMA accumulator chains per column pair.  A warp's MMAs into one
// accumulator form a dependency chain, and on B200 the warp-level MMA takes
// long enough from issue to result that a single chain per pair, 2 MMAs per
// quad for 16 quads, leaves the warp mostly waiting; the quads' MMAs rotate
// over LACC accumulators instead, summed when a group ends.
constexpr int LACC = 1;
constexpr uint64_t LWAIT_NS = 2000000000ull;

struct LeanParams {
    const uint16_t* x;
    const uint16_t* s;
    const uint16_t* z;
    const uint16_t* bias;  // (N,) or null
    uint16_t* y;
    int M, K, N, G;
    int Kw;         // word rows
    int Q;          // quads = ceil(Kw / 4)
    int QW;         // quads per warp (a multiple of the quads per box)
    int KS;         // CTAs per cluster along K (1: no cluster)
    int qpg;        // quads per group (a large number when one group spans K)
    int BQ;         // quads per TMA box (R = 4 BQ word rows)
    int S;          // ring slots per warp (a power of two)
    int xs_stride;  // bytes between tokens in the x stage
    int quads_cta;  // LWK * QW
    uint32_t off_x, off_xq, off_red, off_part, off_bar;  // from the 1024-aligned base (stages at 0)
    int late_wait;  // wait for the previous kernel only before writing y
};

__device__ __forceinline__ uint2 ldg_u2(const uint16_t* p) { return *reinterpret_cast<const uint2*>(p); }

// Conversion constants, scales and fractional zero parts of a lane's 4 columns
// for one group, from the group's s and z values (uint2: columns 0-1 and 2-3
// as 16-bit pairs).  fp16: two columns per fp16x2 instruction -- z is clamped
// to [-256, 256] and rounded to an integer by adding 1536 (fp16 spacing 1 on
// [1024, 2048), ties to even as rint), and the constants -(1024 + zi) and
// -(64 + zi) are differences of exact integers below 2048.  bf16: per column.
template <int BITS, bool BF>
struct GroupConsts {
    static constexpr int NC = ncons<BITS, BF>();
    uint32_t cc[4][NC];
    float sc[4];
    float zr[4];
    bool frac;

    __device__ __forceinline__ void make(uint2 sv, uint2 zv) {
        using T16 = Dt<BF>;
        const float2 s01 = T16::pair(sv.x), s23 = T16::pair(sv.y);
        sc[0] = s01.x; sc[1] = s01.y; sc[2] = s23.x; sc[3] = s23.y;
        bool f = false;
        if constexpr (!BF) {
            uint32_t zi2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t z2 = h ? zv.y : zv.x;
                const uint32_t zc = hmin2_u32(hmax2_u32(z2, h2c(0xDC00u)), h2c(0x5C00u));  // [-256, 256]
                const uint32_t r = hadd2_u32(zc, h2c(0x6600u));                            // 1536 + zi
                zi2[h] = hsub2_u32(r, h2c(0x6600u));
                f |= zi2[h] != z2;
                const uint32_t c0 = hsub2_u32(h2c(0x6000u), r);  // 512 - 1536 - zi = -(1024 + zi)
                cc[2 * h][0] = prmt(c0, c0, 0x1010u);
                cc[2 * h + 1][0] = prmt(c0, c0, 0x3232u);
                if constexpr (NC > 1) {
                    const uint32_t c1 = hsub2_u32(h2c(0x65C0u), r);  // 1472 - 1536 - zi = -(64 + zi)
                    cc[2 * h][1] = prmt(c1, c1, 0x1010u);
                    cc[2 * h + 1][1] = prmt(c1, c1, 0x3232u);
                }
            }
            frac = __any_sync(0xffffffffu, f);
            if (frac) {
                const float2 z01 = T16::pair(zv.x), z23 = T16::pair(zv.y);
                const float2 i01 = T16::pair(zi2[0]), i23 = T16::pair(zi2[1]);
                zr[0] = z01.x - i01.x; zr[1] = z01.y - i01.y;
                zr[2] = z23.x - i23.x; zr[3] = z23.y - i23.y;
            }
        } else {
            const float2 z01 = T16::pair(zv.x), z23 = T16::pair(zv.y);
            const float zz[4] = {z01.x, z01.y, z23.x, z23.y};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float zi = zero_int<BITS, BF>(zz[c]);
                zr[c] = zz[c] - zi;
                f |= zr[c] != 0.0f;
#pragma unroll
                for (int ci = 0; ci < NC; ++ci) cc[c][ci] = pair_const<BITS, BF>(ci, zi);
            }
            frac = __any_sync(0xffffffffu, f);
        }
    }
};

template <int BITS, bool BF, int BQ, bool M1>
__global__ void __launch_bounds__(LWK * 32, 3)
gemv_lean_kernel(const __grid_constant__ CUtensorMap tm_w, const LeanParams p) {
    using F = Fmt<BITS>;
    using T16 = Dt<BF>;
    constexpr int EPS = F::EPS;
    constexpr int QK = 4 * EPS;    // k values per quad
    constexpr int MMAS = EPS / 4;  // MMAs per column pair per quad
    constexpr int NE = M1 ? 1 : 2; // tokens per lane that can exist (2 t, 2 t + 1)
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

    // ---- (1) the warp's words: boxes of BQ quads into a ring of S slots
    const int S = p.S;
    const uint32_t ring0 = smem_u32(smem) + (uint32_t)warp * (uint32_t)S * BOX_BYTES;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.off_bar) + warp * LMAXS;
    const int nbox = (nq + BQ - 1) / BQ;
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int b) {  // box b of this warp -> slot b % S
        const int slot = b & (S - 1);
        mbar_arrive_expect_tx(&bar[slot], BOX_BYTES);
        tma_load_2d_u32_hint(ring0 + (uint32_t)slot * BOX_BYTES, &tm_w, &bar[slot], col0, 4 * (q_begin + b * BQ),
                             pol);
    };
    if (lane == 0) {
        for (int k = 0; k < S; ++k) mbar_init(&bar[k], 1);
        fence_mbarrier_init();
        for (int b = 0; b < S && b < nbox; ++b) issue(b);
    }

    // ---- (2) s and z, read by the warp SZG groups at a time: lane l holds group
    // gb + l / 8, columns col0 + 4 (l % 8) .. + 3 (8 bytes of s and 8 of z), and
    // every lane takes its own columns' values from there by shuffle.  The next
    // chunk is always in flight, SZG groups of work ahead of its use.
    constexpr int SZG = 4;
    const int n_groups = (p.K + p.G - 1) / p.G;
    const int ld_col = col0 + 4 * (lane & 7);
    auto load_chunk = [&](int gb, uint2& sv, uint2& zv) {
        const int gi = gb + (lane >> 3);
        if (ld_col < p.N && gi < n_groups) {
            sv = ldg_u2(p.s + (size_t)gi * p.N + ld_col);
            zv = ldg_u2(p.z + (size_t)gi * p.N + ld_col);
        } else {
            sv = zv = make_uint2(0u, 0u);
        }
    };
    const int g_first = q_begin / p.qpg;
    int gb = g_first;  // first group of the chunk in (sA, zA)
    uint2 sA, zA, sB, zB;
    load_chunk(gb, sA, zA);
    load_chunk(gb + SZG, sB, zB);

    // the next kernel on the stream may start now (it waits for this grid
    // before it touches anything this one writes)
    grid_launch_dependents();

    // ---- (3) x, staged per token in k-slot order: word row r holds the pairs
    // (x[r*EPS + j], x[r*EPS + j + EPS/2]), j < EPS/2.  A chunk is one word row
    // (two for 8-bit), read as 16-byte vectors; values beyond K are zero.
    if (!p.late_wait) grid_dependency_wait();  // x may be the previous kernel's output
    constexpr int CH = EPS >= 8 ? EPS : 8;  // halves per chunk
    constexpr int UPC = CH / 8;             // 16-byte vectors per chunk
    const int row_cta0 = cta_q0 * 4;
    const int cpt = p.quads_cta * 4 * EPS / CH;  // chunks per token
    const int nchunk = p.M * cpt;
    uint8_t* xs = smem + p.off_x;
    for (int c = threadIdx.x; c < nchunk; c += LWK * 32) {
        const int m = M1 ? 0 : c / cpt, ci = M1 ? c : c - m * cpt;
        const int k0 = (row_cta0 + ci * (CH / EPS)) * EPS;
        const uint16_t* src = p.x + (size_t)m * p.K + k0;
        uint4 v[UPC];
#pragma unroll
        for (int w = 0; w < UPC; ++w) v[w] = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (EPS >= 8) {
            if (k0 < p.K) {
#pragma unroll
                for (int w = 0; w < UPC; ++w) v[w] = *reinterpret_cast<const uint4*>(src + 8 * w);
            }
        } else {  // two word rows of 4 values, each 8-byte aligned
            if (k0 < p.K) {
                const uint2 a = *reinterpret_cast<const uint2*>(src);
                v[0].x = a.x; v[0].y = a.y;
            }
            if (k0 + 4 < p.K) {
                const uint2 b = *reinterpret_cast<const uint2*>(src + 4);
                v[0].z = b.x; v[0].w = b.y;
            }
        }
        uint32_t W[CH / 2], P[CH / 2];
#pragma unroll
        for (int w = 0; w < UPC; ++w) {
            W[4 * w + 0] = v[w].x; W[4 * w + 1] = v[w].y;
            W[4 * w + 2] = v[w].z; W[4 * w + 3] = v[w].w;
        }
#pragma unroll
        for (int rr = 0; rr < CH / EPS; ++rr)
#pragma unroll
            for (int j = 0; j < EPS / 2; ++j) {
                const uint32_t* Wr = W + rr * (EPS / 2);
                P[rr * (EPS / 2) + j] = prmt(Wr[j / 2], Wr[j / 2 + EPS / 4], (j & 1) ? 0x7632u : 0x5410u);
            }
        uint8_t* dst = xs + m * p.xs_stride + (size_t)ci * CH * 2;
#pragma unroll
        for (int w = 0; w < UPC; ++w)
            *reinterpret_cast<uint4*>(dst + 16 * w) = make_uint4(P[4 * w], P[4 * w + 1], P[4 * w + 2], P[4 * w + 3]);
    }
    __syncthreads();  // x staged; every mbarrier initialised
    // per-quad sums of x (fp32), for fractional zero points
    float* xq = reinterpret_cast<float*>(smem + p.off_xq);
    for (int i = threadIdx.x; i < p.M * p.quads_cta; i += LWK * 32) {
        const int m = i / p.quads_cta, ql = i - m * p.quads_cta;
        const uint4* src = reinterpret_cast<const uint4*>(xs + m * p.xs_stride + (size_t)ql * QK * 2);
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int w = 0; w < QK / 8; ++w) {
            const uint4 u = src[w];
            const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = T16::pair(e[h]);
                a0 += f.x;
                a1 += f.y;
            }
        }
        xq[i] = a0 + a1;
    }
    __syncthreads();

    // ---- (4) main loop
    float acc[4][NE], dsum[LACC][2][4], xsum[NE];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < NE; ++e) acc[c][e] = 0.0f;
#pragma unroll
    for (int c = 0; c < LACC; ++c)
#pragma unroll
        for (int T = 0; T < 2; ++T)
#pragma unroll
            for (int e = 0; e < 4; ++e) dsum[c][T][e] = 0.0f;
#pragma unroll
    for (int e = 0; e < NE; ++e) xsum[e] = 0.0f;
    // B fragment address: token g (duplicates beyond M are harmless), word row t of quad 0
    uint32_t xaddr = smem_u32(xs) + (uint32_t)(min(g, p.M - 1) * p.xs_stride + (4 * (q_begin - cta_q0) + t) * EPS * 2);
    uint32_t xqa[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e)
        xqa[e] = smem_u32(xq) + 4u * (uint32_t)(min(2 * t + e, p.M - 1) * p.quads_cta + (q_begin - cta_q0));

    GroupConsts<BITS, BF> k;
    auto consts = [&](int gi) {  // gi: gb <= gi <= gb + SZG (warp-uniform)
        if (gi >= gb + SZG) {
            gb += SZG;
            sA = sB;
            zA = zB;
            load_chunk(gb + SZG, sB, zB);
        }
        const int src = ((gi - gb) << 3) | cg;
        uint2 sv, zv;
        sv.x = __shfl_sync(0xffffffffu, sA.x, src);
        sv.y = __shfl_sync(0xffffffffu, sA.y, src);
        zv.x = __shfl_sync(0xffffffffu, zA.x, src);
        zv.y = __shfl_sync(0xffffffffu, zA.y, src);
        k.make(sv, zv);
    };
    int gcur = g_first;
    consts(gcur);
    int left = p.qpg - (q_begin - g_first * p.qpg);  // quads left in the current group
    // fold the group's dot products into acc (scaled by s, fractional zero points applied)
    auto fold = [&]() {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int T = c >> 1, half = c & 1;
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                float d = dsum[0][T][2 * half + e];
#pragma unroll
                for (int ch = 1; ch < LACC; ++ch) d += dsum[ch][T][2 * half + e];
                if (k.frac) d = fmaf(-k.zr[c], xsum[e], d);
                acc[c][e] = fmaf(k.sc[c], d, acc[c][e]);
            }
        }
#pragma unroll
        for (int ch = 0; ch < LACC; ++ch)
#pragma unroll
            for (int T = 0; T < 2; ++T)
#pragma unroll
                for (int e = 0; e < 4; ++e) dsum[ch][T][e] = 0.0f;
#pragma unroll
        for (int e = 0; e < NE; ++e) xsum[e] = 0.0f;
    };

    // Per-lane offsets of this lane's 16-byte vector inside a slot: quad iq,
    // word row R = 4 iq + t, 16-byte chunk cg swizzled with (R & 7), whose
    // value only depends on the parity of iq.
    const uint32_t off_even = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)t) << 4);
    const uint32_t off_odd = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)(t + 4)) << 4);

    // one quad: iq = i4 + j is the quad within the slot (j < 4 compile-time, i4 a
    // multiple of 4), i the quad within the warp
    auto quad = [&](uint32_t slot_addr, int i4, int j, int i) {
        const int iq = i4 + j;
        const uint4 hv = lds128_u32(slot_addr + 512 * iq + ((j & 1) ? off_odd : off_even));
        uint32_t bx[EPS / 2];
        if constexpr (EPS >= 8) {
#pragma unroll
            for (int v = 0; v < EPS / 8; ++v) {
                const uint4 u = lds128_u32(xaddr + QK * 2 * iq + 16 * v);
                bx[4 * v + 0] = u.x; bx[4 * v + 1] = u.y; bx[4 * v + 2] = u.z; bx[4 * v + 3] = u.w;
            }
        } else {
            const uint2 u = lds64_u32(xaddr + QK * 2 * iq);
            bx[0] = u.x;
            bx[1] = u.y;
        }
        if (k.frac) {
#pragma unroll
            for (int e = 0; e < NE; ++e) xsum[e] += __uint_as_float(lds32_u32(xqa[e] + 4 * i));
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
                mma_16816<BF>(dsum[(j * MMAS + h) % LACC][T], a, bx[2 * h], bx[2 * h + 1]);
            }
        }
        if (--left == 0) {  // end of a group: fold, then the next group's constants
            fold();
            left = p.qpg;
            consts(++gcur);
        }
    };

    bool ok_all = true;
    for (int b = 0; b < nbox; ++b) {
        const int slot = b & (S - 1);
        const bool good = mbar_wait_bounded(&bar[slot], (uint32_t)((b / S) & 1), LWAIT_NS);
        if (!good) atomicExch(&g_gemv_lean_status, 1u);
        if (!__all_sync(0xffffffffu, good)) {  // give up this warp's range
            ok_all = false;
            break;
        }
        const uint32_t slot_addr = ring0 + (uint32_t)slot * BOX_BYTES;
        const int i0 = b * BQ;
        if (i0 + BQ <= nq) {
#pragma unroll 1
            for (int i4 = 0; i4 < BQ; i4 += 4)
#pragma unroll
                for (int j = 0; j < 4; ++j) quad(slot_addr, i4, j, i0 + i4 + j);
        } else {
#pragma unroll 1
            for (int i4 = 0; i4 < BQ; i4 += 4)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (i0 + i4 + j < nq) quad(slot_addr, i4, j, i0 + i4 + j);
        }
        xaddr += QK * 2 * BQ;
        // every lane has read this slot: refill it with box b + S
        __syncwarp();
        if (lane == 0 && b + S < nbox) {
            fence_proxy_async_smem();
            issue(b + S);
        }
    }
    if (ok_all && nq > 0 && left != p.qpg) fold();  // the warp's range ended inside a group

    // ---- (5) reduce over the warps of the CTA (and the CTAs of the cluster), write y
    float* red = reinterpret_cast<float*>(smem + p.off_red);  // [LWK][M][LCOLS]
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            const int m = 2 * t + e;
            if (m < p.M) red[(warp * p.M + m) * LCOLS + 4 * cg + c] = acc[c][e];
        }
    __syncthreads();
    const int nout = p.M * LCOLS;
    auto warp_sum = [&](int i) {
        float v[LWK];
#pragma unroll
        for (int w = 0; w < LWK; ++w) v[w] = red[w * nout + i];
#pragma unroll
        for (int h = LWK / 2; h >= 1; h >>= 1)
#pragma unroll
            for (int w = 0; w < h; ++w) v[w] += v[w + h];
        return v[0];
    };
    auto store = [&](int i, float v) {
        const int m = i / LCOLS, col = col0 + i % LCOLS;
        if (col < p.N) {
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
        if (p.late_wait) grid_dependency_wait();
        for (int i = threadIdx.x; i < nout; i += LWK * 32) store(i, warp_sum(i));
    }
}

// Shared-memory plan of one launch: the ring, x and the small buffers.
size_t lean_layout(LeanParams& p, int EPS) {
    size_t off = (size_t)LWK * p.S * p.BQ * 4 * LCOLS * 4;  // the rings (1024-byte multiples)
    p.off_x = (uint32_t)off;
    off += (size_t)p.M * p.xs_stride;
    off = (off + 15) & ~(size_t)15;
    p.off_xq = (uint32_t)off;
    off += (size_t)p.M * p.quads_cta * 4;
    off = (off + 15) & ~(size_t)15;
    p.off_red = (uint32_t)off;
    off += (size_t)LWK * p.M * LCOLS * 4;
    p.off_part = (uint32_t)off;
    off += (size_t)p.M * LCOLS * 4;
    off = (off + 7) & ~(size_t)7;
    p.off_bar = (uint32_t)off;
    off += (size_t)LWK * LMAXS * 8;
    (void)EPS;
    return off + 1024;  // slack for aligning the base to 1024 bytes
}

template <int BITS, bool BF, int BQ, bool M1>
wq_status launch_lean(const CUtensorMap& mw, const LeanParams& p, size_t smem, const Problem& pb,
                      cudaStream_t stream) {
    auto kern = gemv_lean_kernel<BITS, BF, BQ, M1>;
    static std::atomic<uint64_t> attr_ctx[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (const wq_status st = ensure_smem_attr((const void*)kern, 227 * 1024, attr_ctx, dev); st != WQ_OK) return st;
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
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, mw, p));
}

template <int BITS, bool BF>
wq_status run_lean(const Problem& pb, cudaStream_t stream) {
    constexpr int EPS = Fmt<BITS>::EPS;
    constexpr int QK = 4 * EPS;
    LeanParams p{};
    p.x = pb.x; p.s = pb.scales; p.z = pb.zeros; p.bias = pb.bias; p.y = pb.y;
    p.M = pb.M; p.K = pb.K; p.N = pb.N; p.G = pb.G;
    p.late_wait = (pb.flags & WQ_FLAG_PDL_INPUTS_READY) ? 1 : 0;
    p.Kw = pb.K / EPS;
    p.Q = (p.Kw + 3) / 4;
    p.qpg = (pb.G == pb.K) ? (1 << 29) : pb.G / QK;
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
    p.quads_cta = LWK * p.QW;
    p.xs_stride = p.quads_cta * 4 * EPS * 2 + (pb.M > 1 ? 64 : 0);  // pad: tokens on other banks
    const size_t smem = lean_layout(p, EPS);
    if (smem > 227 * 1024) return WQ_ERR_UNSUPPORTED;

    CUtensorMap mw;
    if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_q, pb.N, p.Kw, (uint64_t)pb.N * 4, LCOLS, 4 * BQ,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    const bool m1 = pb.M == 1;
    if (BQ == 16)
        return m1 ? launch_lean<BITS, BF, 16, true>(mw, p, smem, pb, stream)
                  : launch_lean<BITS, BF, 16, false>(mw, p, smem, pb, stream);
    return m1 ? launch_lean<BITS, BF, 8, true>(mw, p, smem, pb, stream)
              : launch_lean<BITS, BF, 8, false>(mw, p, smem, pb, stream);
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
    return v ? WQ_ERR_TIMEOUT : WQ_OK;
}

bool gemv_lean_takes(const Problem& p) {
    if (p.bits != 4 && p.bits != 8) return false;
    if (p.M > 8) return false;
    // one 4-bit token: the kernel of wq_gemv.cu measured faster on B200 (4096 x 4096)
    if (p.bits == 4 && p.M == 1 && p.K >= 1024) return false;
    const int qk = 4 * (32 / p.bits);
    return p.G == p.K || p.G % qk == 0;
}

wq_status launch_gemv_lean(const Problem& p, cudaStream_t s) {
    const bool bf = (p.flags & WQ_FLAG_BF16) != 0;
    if (p.bits == 4) return bf ? run_lean<4, true>(p, s) : run_lean<4, false>(p, s);
    if (p.bits == 8) return bf ? run_lean<8, true>(p, s) : run_lean<8, false>(p, s);
    return WQ_ERR_UNSUPPORTED;
}

}  // namespace wq
