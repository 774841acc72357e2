// wq_gemv.cu -- decode-time product y (M x N) = x (M x K) @ dequant(W_q), 1 <= M <= 16.
//
// What is computed: dashq_kernel.py `_dashq_gemv_kernel` (one token there; up to
// 16 here): each output column n is sum_k x[k] * (q[k][n] - z[g][n]) * s[g][n],
// g = k / G, with fp32 accumulation and one rounding at the end.  x, s, z, the
// bias and y are all fp16 or all bf16 (the module's `out_dtype`).
//
// How (sm_100a):
//  * Work split.  A CTA owns 32 output columns and a contiguous K range, split
//    again over its WK warps; a warp owns a run of "quads" (4 packed word rows
//    x 32 columns).  When there are few column blocks, the CTAs of a
//    thread-block cluster split K further and reduce their fp32 partial sums
//    through distributed shared memory.  One launch, no workspace, no atomics.
//  * Loads.  Each warp streams its K range with 2-D TMA boxes of 32 word rows
//    x 32 columns (8 quads, 128-byte swizzle) into one or two shared-memory stages,
//    completing on an mbarrier: the bytes in flight cost neither registers nor
//    L1 request slots.  Lane (g, t) (g = lane / 4, t = lane % 4) then reads one
//    16-byte vector per quad (4 adjacent columns of one word row); the column
//    chunk each lane reads is chosen so that these reads are free of bank
//    conflicts.
//  * Dequant.  A code pair (code j, code j + eps/2) sits at the same offset in
//    the two 16-bit halves of a word: one LOP3 ORs both into the mantissa of
//    fp16 1024 and one exact fp16x2 FMA gives the integers q - round(z) (bf16:
//    the same with bf16 128 on shifted copies of the word; see wq_dequant.cuh).
//  * Dot product.  Those exact values are the A operand of a warp MMA m16n8k16
//    (fp16 or bf16 in, fp32 accumulate) with x as B: A rows are 16 output columns and
//    the 16 k-slots are 4 word rows x 4 codes, a permutation of k; x is staged
//    once per CTA in shared memory in the same permuted order.
//  * Per group, acc += s * (D - (z - round(z)) * X) in fp32, X = the sum of the
//    x values of that group slice, so fractional zero points are exact and
//    q == z gives exactly 0.
//  * s and z of the CTA's groups arrive with one TMA copy each and become
//    per-(group, column) records in shared memory; the optional bias is added
//    to the fp32 sum before the final rounding.
#include <algorithm>
#include <array>
#include <cstddef>
#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>

#include "wq_dequant.cuh"
#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {

// Device status of the GEMV: 0, or 1 once a bounded wait ran out.
__device__ unsigned int g_gemv_status = 0;

namespace {

constexpr int COLS = 32;     // output columns per CTA
constexpr int MAXW = 16;     // warps per CTA (split along K)
constexpr int SQ = 8;        // quads per TMA stage (32 word rows x 32 columns = 4 KB)
constexpr int MAXST = 2;     // stages per warp (at most)
constexpr uint64_t WAIT_NS = 2000000000ull;

struct Params {
    const uint16_t* x;
    const uint32_t* w_q;
    const uint32_t* w_lo;
    const uint16_t* s;
    const uint16_t* z;
    const uint16_t* bias;  // (N,) fp16 / bf16 or null
    uint16_t* y;
    int M, K, N, G;
    int Kw;        // word rows of the main plane
    int Q;         // quads = ceil(Kw / 4)
    int QW;        // quads per warp (a power of two)
    int WK;        // warps per CTA
    int CS;        // CTAs per cluster (along K)
    int qpg;       // quads per group (a large number when one group spans K)
    int qpg_shift; // log2(qpg) when qpg is a power of two, else -1
    int n_groups;  // ceil(K / G)
    int cpt_shift; // log2(x chunks per token staged by a CTA)
    int qc_shift;  // log2(quads per CTA)
    int groups_cta;
    int nst;       // TMA stages per warp: 1 or 2
    int late_wait; // wait for the previous kernel only before writing y
    int xs_tok_stride;  // bytes between tokens in the x stage (padded)
    uint32_t off_x, off_xq, off_tab, off_red, off_part, off_bar;  // smem byte offsets (stages at 0)
    uint32_t off_sz;  // raw s rows then z rows of the CTA's groups (sz_rows x COLS fp16 each)
    int sz_rows;      // rows loaded per tile: sz_box x sz_nbox >= groups_cta
    int sz_box;       // rows per TMA box (<= 256)
    uint32_t sz_stride;  // bytes from the s tile to the z tile (128-byte multiple)
};

// bytes of one stage: 32 x 32 words of the main plane (+ 16 x 32 lo-plane words)
template <int BITS>
constexpr int stage_bytes() { return BITS == 3 ? 6144 : 4096; }

// Sum of red[w * stride + i] over the wk (<= MAXW) warps: all loads issued
// first, then a pairwise tree, so the latency is paid once.
__device__ __forceinline__ float sum_warps(const float* red, int wk, int stride, int i) {
    float v[MAXW];
#pragma unroll
    for (int w = 0; w < MAXW; ++w) v[w] = (w < wk) ? red[w * stride + i] : 0.0f;
#pragma unroll
    for (int h = MAXW / 2; h >= 1; h >>= 1)
#pragma unroll
        for (int w = 0; w < h; ++w) v[w] += v[w + h];
    return v[0];
}

template <int BITS, int NT, bool BF>
__global__ void __launch_bounds__(MAXW * 32, (NT == 1 && BITS != 1) ? 2 : 1)
gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_lo,
            const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_z, const Params p) {
    using F = Fmt<BITS>;
    using T16 = Dt<BF>;
    using R = Rec<BITS, BF>;
    constexpr bool SLIM = slim_rec<BITS, BF>();
    constexpr uint32_t COFF = SLIM ? 0u : 8u;  // byte offset of the constants in a record
    constexpr int EPS = F::EPS;
    constexpr int NC = ncons<BITS, BF>();
    constexpr int QK = 4 * EPS;  // k values per quad
    constexpr int MMAS = EPS / 4;
    constexpr int SB = stage_bytes<BITS>();
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base: the 128-byte swizzle of the TMA stages repeats every 1024 bytes
    uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    // 16-byte column chunk this lane reads (columns 4 cg .. 4 cg + 3): lanes g and
    // g + 1 of a quarter-warp then differ in bit 2, which the row swizzle never
    // touches, so each quarter-warp's eight 16-byte reads hit distinct banks.
    const int cg = ((g & 1) << 2) | (g >> 1);
    const int rank = (int)blockIdx.y;  // the cluster spans the grid's y extent
    const int col0 = blockIdx.x * COLS;

    const int cta_q0 = rank * p.WK * p.QW;
    const int q_begin = cta_q0 + warp * p.QW;
    const int q_end = min(p.Q, q_begin + p.QW);
    const int nq = max(0, q_end - q_begin);

    // ---- s, z of the CTA's (group, column) records
    // group of quad q (G = qpg * QK): a shift for the usual power-of-two group sizes
    auto gdiv = [&](int q) { return p.qpg_shift >= 0 ? (q >> p.qpg_shift) : q / p.qpg; };
    const int g_cta0 = gdiv(min(cta_q0, p.Q - 1));
    const int nrec = p.groups_cta * COLS;
    R* tab = reinterpret_cast<R*>(smem + p.off_tab);
    bool any_frac = false;
    // Record slot sl of a group holds column 4 (sl % 8) + sl / 8: the eight lanes
    // reading one column offset c of their chunks then read consecutive records.
    // Built from the raw s and z tiles that one TMA copy brought in (columns or
    // groups outside the matrix read as 0: s = 0 and z = 0).
    const uint16_t* s_raw = reinterpret_cast<const uint16_t*>(smem + p.off_sz);
    const uint16_t* z_raw = reinterpret_cast<const uint16_t*>(smem + p.off_sz + p.sz_stride);
    auto tab_build = [&]() {
        for (int i = threadIdx.x; i < nrec; i += blockDim.x) {
            const int sl = i & (COLS - 1);
            const int o = (i & ~(COLS - 1)) + 4 * (sl & 7) + (sl >> 3);
            const float sv = T16::load(s_raw[o]);
            const float zv = T16::load(z_raw[o]);
            const float zi = zero_int<BITS, BF>(zv);
            R rec;
            if constexpr (!SLIM) {
                rec.s = sv;
                rec.zr = zv - zi;
            }
            any_frac |= (zv - zi != 0.0f);
#pragma unroll
            for (int ci = 0; ci < NC; ++ci) rec.c[ci] = pair_const<BITS, BF>(ci, zi);
            tab[i] = rec;
        }
    };
    // ---- (2) weights: each warp streams its K range with 2-D TMA boxes of 32
    // word rows x 32 columns (8 quads, 128-byte swizzle) into nst stages
    const int nst = p.nst;
    const uint32_t st0 = smem_u32(smem) + (uint32_t)(warp * nst * SB);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.off_bar) + warp * MAXST;
    const int nst_w = (nq + SQ - 1) / SQ;  // stages this warp consumes
    auto issue = [&](int k) {              // stage number k of this warp -> slot k % nst
        const int slot = k & (nst - 1);
        const uint32_t dst = st0 + slot * SB;
        mbar_arrive_expect_tx(&bar[slot], (uint32_t)SB);
        tma_load_2d_u32(dst, &tm_w, &bar[slot], col0, 4 * (q_begin + k * SQ));
        if constexpr (BITS == 3) tma_load_2d_u32(dst + 4096, &tm_lo, &bar[slot], col0, 2 * (q_begin + k * SQ));
    };
    uint64_t* bar_sz = reinterpret_cast<uint64_t*>(smem + p.off_bar) + p.WK * MAXST;
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < MAXST; ++k) mbar_init(&bar[k], 1);
        if (warp == 0) mbar_init(bar_sz, 1);
        fence_mbarrier_init();
        prefetch_tmap(&tm_w);
        if (warp == 0) {  // ---- (1) the raw s and z rows of the CTA's groups, first in line
            const int nbox = p.sz_rows / p.sz_box;
            mbar_arrive_expect_tx(bar_sz, (uint32_t)(2 * p.sz_rows * COLS * 2));
            for (int b = 0; b < nbox; ++b) {
                const uint32_t d = smem_u32(smem + p.off_sz) + (uint32_t)(b * p.sz_box * COLS * 2);
                tma_load_2d_u32(d, &tm_s, bar_sz, col0, g_cta0 + b * p.sz_box);
                tma_load_2d_u32(d + p.sz_stride, &tm_z, bar_sz, col0, g_cta0 + b * p.sz_box);
            }
        }
        for (int k = 0; k < nst && k < nst_w; ++k) issue(k);
    }
    __syncthreads();  // every mbarrier above is initialised before anyone waits on it
    // the next kernel on the stream may start now (it waits for this grid before reading its x)
    grid_launch_dependents();

    // x is staged per token in k-slot order: word row r holds the pairs
    // (x[r*EPS + j], x[r*EPS + j + EPS/2]), j < EPS/2.  A chunk is one word row
    // (two for 8-bit), read as 16-byte vectors.
    constexpr int CH = EPS >= 8 ? EPS : 8;        // halves per chunk
    constexpr int UPC = CH / 8;                   // 16-byte vectors per chunk
    constexpr int XB = UPC >= 2 ? 1 : 2;          // chunks per thread per round
    const int row_cta0 = cta_q0 * 4;
    const int cpt = 1 << p.cpt_shift;             // chunks per token
    const int nchunk = p.M * cpt;
    uint8_t* xs = smem + p.off_x;
    auto x_load = [&](int base, uint4 (&v)[XB][UPC]) {
#pragma unroll
        for (int u = 0; u < XB; ++u) {
            const int c = base + u * (int)blockDim.x + (int)threadIdx.x;
            const int m = c >> p.cpt_shift, ci = c & (cpt - 1);
            const int k0 = (row_cta0 + ci * (CH / EPS)) * EPS;
            const uint16_t* src = p.x + (size_t)m * p.K + k0;
#pragma unroll
            for (int w = 0; w < UPC; ++w) v[u][w] = make_uint4(0, 0, 0, 0);
            if (c < nchunk && check(m < p.M, &g_gemv_status)) {
                if constexpr (EPS >= 8) {
                    if (k0 < p.K) {
#pragma unroll
                        for (int w = 0; w < UPC; ++w) v[u][w] = *reinterpret_cast<const uint4*>(src + 8 * w);
                    }
                } else {  // two rows of 4 halves, each 8-byte aligned
                    if (k0 < p.K) {
                        const uint2 a = *reinterpret_cast<const uint2*>(src);
                        v[u][0].x = a.x; v[u][0].y = a.y;
                    }
                    if (k0 + 4 < p.K) {
                        const uint2 b = *reinterpret_cast<const uint2*>(src + 4);
                        v[u][0].z = b.x; v[u][0].w = b.y;
                    }
                }
            }
        }
    };
    auto x_store = [&](int base, const uint4 (&v)[XB][UPC]) {
#pragma unroll
        for (int u = 0; u < XB; ++u) {
            const int c = base + u * (int)blockDim.x + (int)threadIdx.x;
            if (c < nchunk) {
                const int m = c >> p.cpt_shift, ci = c & (cpt - 1);
                uint32_t W[CH / 2];
#pragma unroll
                for (int w = 0; w < UPC; ++w) {
                    W[4 * w + 0] = v[u][w].x; W[4 * w + 1] = v[u][w].y;
                    W[4 * w + 2] = v[u][w].z; W[4 * w + 3] = v[u][w].w;
                }
                uint32_t P[CH / 2];
#pragma unroll
                for (int rr = 0; rr < CH / EPS; ++rr) {
#pragma unroll
                    for (int j = 0; j < EPS / 2; ++j) {
                        const uint32_t* Wr = W + rr * (EPS / 2);
                        P[rr * (EPS / 2) + j] = prmt(Wr[j / 2], Wr[j / 2 + EPS / 4], (j & 1) ? 0x7632u : 0x5410u);
                    }
                }
                uint8_t* dst = xs + m * p.xs_tok_stride + (size_t)ci * CH * 2;
#pragma unroll
                for (int w = 0; w < UPC; ++w)
                    *reinterpret_cast<uint4*>(dst + 16 * w) = make_uint4(P[4 * w], P[4 * w + 1], P[4 * w + 2], P[4 * w + 3]);
            }
        }
    };
    auto stage_x = [&]() {
    for (int base = 0; base < nchunk; base += XB * (int)blockDim.x) {
        uint4 xv[XB][UPC];
        x_load(base, xv);
        x_store(base, xv);
    }
    };
    auto table = [&]() {
        const bool good = mbar_wait_bounded(bar_sz, 0, WAIT_NS);
        if (!good) atomicOr(&g_gemv_status, 1u);
        if (good) tab_build();
    };
    // ---- (3) the records, and x.  x may come from the previous kernel on the
    // stream (WQ_FLAG_PDL): build the records while that kernel runs, then wait.
    // Without that dependency stage x first, while the s/z copy lands.
    if (!p.late_wait) {
        table();
        grid_dependency_wait();
        stage_x();
    } else {
        stage_x();
        table();
    }
    // fractional zero points anywhere in this CTA's records?  (CTA-uniform; the
    // barrier also publishes the staged x and the records)
    const bool frac = __syncthreads_or(any_frac) != 0;

    // ---- (4) per-quad x sums (fp32), only needed for fractional zero points
    const int quads_cta = 1 << p.qc_shift;
    float* xq = reinterpret_cast<float*>(smem + p.off_xq);
    if (frac) {
        for (int i = threadIdx.x; i < p.M * quads_cta; i += blockDim.x) {
            const int m = i >> p.qc_shift, ql = i & (quads_cta - 1);
            const uint4* src = reinterpret_cast<const uint4*>(xs + m * p.xs_tok_stride + (size_t)ql * QK * 2);
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
    }
    float acc[4][NT][2];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[c][n][0] = acc[c][n][1] = 0.0f;
    int tok[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        tok[n][0] = 2 * t + 8 * n;
        tok[n][1] = 2 * t + 1 + 8 * n;
    }

    // The main loop, specialised on whether fractional zero-point terms are needed.
    auto main_loop = [&](auto frac_tag) {
        constexpr bool FRAC = decltype(frac_tag)::value;
        constexpr uint32_t RS = sizeof(R);
        float dsum[2][NT][4];
        float xs_sum[NT][2];
#pragma unroll
        for (int T = 0; T < 2; ++T)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) dsum[T][n][e] = 0.0f;
#pragma unroll
        for (int n = 0; n < NT; ++n) xs_sum[n][0] = xs_sum[n][1] = 0.0f;

        // B-fragment addresses (token rows; duplicates beyond M are harmless)
        uint32_t xaddr[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n)
            xaddr[n] = smem_u32(xs) + (uint32_t)(min(g + 8 * n, p.M - 1) * p.xs_tok_stride +
                                                 (4 * (q_begin - cta_q0) + t) * EPS * 2);
        uint32_t xqaddr[NT][2];
        if constexpr (FRAC) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    xqaddr[n][e] = smem_u32(xq) + 4u * (uint32_t)((min(tok[n][e], p.M - 1) << p.qc_shift) +
                                                                  (q_begin - cta_q0));
        }
        // group bookkeeping without divisions in the loop
        const int g_first = gdiv(q_begin);
        int left = p.qpg - (q_begin - g_first * p.qpg);  // quads left in the current group
        uint32_t rc = smem_u32(tab) + RS * (uint32_t)((g_first - g_cta0) * COLS + cg);
        constexpr uint32_t CS8 = 8 * RS;  // record stride between the lane's columns
        // slim records: the raw s row of the lane's 4 columns (z at + sz_stride)
        [[maybe_unused]] uint32_t sz_row = smem_u32(s_raw) + 2u * (uint32_t)((g_first - g_cta0) * COLS + 4 * cg);
        // bias constants of the lane's 4 columns, in registers for narrow records
        constexpr bool CREG = NC <= 2;
        [[maybe_unused]] uint32_t creg[4][CREG ? NC : 1];
        auto load_creg = [&]() {
            if constexpr (CREG) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int ci = 0; ci < NC; ++ci) creg[c][ci] = lds32_u32(rc + c * CS8 + COFF + 4 * ci);
            }
        };
        if (nq > 0) load_creg();
        const uint32_t lo_sel = (t & 1) ? 0x7372u : 0x7170u;  // 3-bit: which half of the lo word
        // Per-lane offsets of this lane's 16-byte vector inside a stage: quad iq,
        // word row R = 4 iq + t, 16-byte chunk cg swizzled with (R & 7), whose
        // value only depends on the parity of iq.
        const uint32_t off_even = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)t) << 4);
        const uint32_t off_odd = (uint32_t)t * 128 + (((uint32_t)cg ^ (uint32_t)(t + 4)) << 4);
        // 3-bit lo plane: row R >> 1 = 2 iq + (t >> 1), swizzled with ((R >> 1) & 7)
        const uint32_t tl = (uint32_t)(t >> 1);
        [[maybe_unused]] const uint32_t lo_off[4] = {tl * 128 + (((uint32_t)cg ^ tl) << 4), tl * 128 + (((uint32_t)cg ^ (tl + 2)) << 4),
                                    tl * 128 + (((uint32_t)cg ^ (tl + 4)) << 4), tl * 128 + (((uint32_t)cg ^ (tl + 6)) << 4)};

        auto quad = [&](uint32_t stage, int iq, int i) {
            const uint4 hv = lds128_u32(stage + 512 * iq + ((iq & 1) ? off_odd : off_even));
            uint4 lv = make_uint4(0, 0, 0, 0);
            if constexpr (BITS == 3) lv = lds128_u32(stage + 4096 + 256 * iq + lo_off[iq & 3]);
            // B fragments: this lane's word row of the quad, all MMAS pairs
            uint32_t bx[NT][EPS / 2];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
#pragma unroll
                for (int v = 0; v < EPS / 8; ++v) {
                    const uint4 u = lds128_u32(xaddr[n] + QK * 2 * iq + 16 * v);
                    bx[n][4 * v + 0] = u.x;
                    bx[n][4 * v + 1] = u.y;
                    bx[n][4 * v + 2] = u.z;
                    bx[n][4 * v + 3] = u.w;
                }
                if constexpr (EPS / 8 == 0) {
                    const uint2 u = lds64_u32(xaddr[n] + QK * 2 * iq);
                    bx[n][0] = u.x;
                    bx[n][1] = u.y;
                }
            }
            if constexpr (FRAC) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) xs_sum[n][e] += __uint_as_float(lds32_u32(xqaddr[n][e] + 4 * iq));
            }

            const uint32_t wv[4] = {hv.x, hv.y, hv.z, hv.w};
            const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
            for (int T = 0; T < 2; ++T) {
                const int ca = 2 * T, cb = 2 * T + 1;
                uint32_t cA[NC], cB[NC];
#pragma unroll
                for (int ci = 0; ci < NC; ++ci) {
                    if constexpr (CREG) {
                        cA[ci] = creg[ca][ci];
                        cB[ci] = creg[cb][ci];
                    } else {
                        cA[ci] = lds32_u32(rc + ca * CS8 + COFF + 4 * ci);
                        cB[ci] = lds32_u32(rc + cb * CS8 + COFF + 4 * ci);
                    }
                }
                Word<BITS, BF> WA, WB;
                WA.prep(wv[ca], lw[ca], lo_sel);
                WB.prep(wv[cb], lw[cb], lo_sel);
#pragma unroll
                for (int h = 0; h < MMAS; ++h) {
                    uint32_t a[4];
                    a[0] = WA.pair(cA, 2 * h);
                    a[1] = WB.pair(cB, 2 * h);
                    a[2] = WA.pair(cA, 2 * h + 1);
                    a[3] = WB.pair(cB, 2 * h + 1);
#pragma unroll
                    for (int n = 0; n < NT; ++n) mma_16816<BF>(dsum[T][n], a, bx[n][2 * h], bx[n][2 * h + 1]);
                }
            }

            // end of a group (or of this warp's range): scale and fold into acc
            if (--left == 0 || i == nq - 1) {
                [[maybe_unused]] float s4[4], zr4[4];
                if constexpr (SLIM) {  // columns 4 cg .. 4 cg + 3 of the raw rows: one 8-byte read each
                    const uint2 su = lds64_u32(sz_row);
                    const float2 s01 = T16::pair(su.x), s23 = T16::pair(su.y);
                    s4[0] = s01.x; s4[1] = s01.y; s4[2] = s23.x; s4[3] = s23.y;
                    if constexpr (FRAC) {
                        const uint2 zu = lds64_u32(sz_row + p.sz_stride);
                        const float2 z01 = T16::pair(zu.x), z23 = T16::pair(zu.y);
                        const float zv[4] = {z01.x, z01.y, z23.x, z23.y};
#pragma unroll
                        for (int c = 0; c < 4; ++c) zr4[c] = zv[c] - zero_int<BITS, BF>(zv[c]);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float sc, zr = 0.0f;
                    if constexpr (SLIM) {
                        sc = s4[c];
                        if constexpr (FRAC) zr = zr4[c];
                    } else {
                        sc = __uint_as_float(lds32_u32(rc + c * CS8));
                        if constexpr (FRAC) zr = __uint_as_float(lds32_u32(rc + c * CS8 + 4));
                    }
                    const int T = c >> 1, half = c & 1;
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float d = FRAC ? dsum[T][n][2 * half + e] - zr * xs_sum[n][e]
                                                 : dsum[T][n][2 * half + e];
                            acc[c][n][e] = fmaf(sc, d, acc[c][n][e]);
                        }
                }
#pragma unroll
                for (int T = 0; T < 2; ++T)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) dsum[T][n][e] = 0.0f;
                if constexpr (FRAC) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) xs_sum[n][0] = xs_sum[n][1] = 0.0f;
                }
                if (left == 0) {
                    left = p.qpg;
                    rc += COLS * RS;
                    sz_row += 2 * COLS;
                    if (i + 1 < nq) load_creg();
                }
            }
        };

        for (int kst = 0; kst < nst_w; ++kst) {
            const bool good = mbar_wait_bounded(&bar[kst & (nst - 1)], (kst / nst) & 1, WAIT_NS);
            if (!good) atomicOr(&g_gemv_status, 1u);
            if (!__all_sync(0xffffffffu, good)) break;  // give up this warp's range
            const uint32_t stage = st0 + (kst & (nst - 1)) * SB;
            const int i0 = kst * SQ;
            if (i0 + SQ <= nq) {
#pragma unroll
                for (int iq = 0; iq < SQ; ++iq) quad(stage, iq, i0 + iq);
            } else {
#pragma unroll
                for (int iq = 0; iq < SQ; ++iq)
                    if (i0 + iq < nq) quad(stage, iq, i0 + iq);
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) xaddr[n] += QK * 2 * SQ;
            if constexpr (FRAC) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) xqaddr[n][e] += 4 * SQ;
            }
            // every lane has used this stage's words: refill its slot with stage kst + nst
            __syncwarp();
            if (lane == 0 && kst + nst < nst_w) {
                fence_proxy_async_smem();
                issue(kst + nst);
            }
        }
    };
    if (frac)
        main_loop(std::true_type{});
    else
        main_loop(std::false_type{});

    // ---- reduce over the warps of the CTA, then write y (with late_wait, only
    // once the previous kernel on the stream has completed)
    float* red = reinterpret_cast<float*>(smem + p.off_red);  // [WK][M][COLS]
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int m = tok[n][e];
                if (m < p.M) red[(warp * p.M + m) * COLS + 4 * cg + c] = acc[c][n][e];
            }
    __syncthreads();
    float* part = reinterpret_cast<float*>(smem + p.off_part);  // [M][COLS]
    if (p.CS > 1) {
        for (int i = threadIdx.x; i < p.M * COLS; i += blockDim.x) {
            part[i] = sum_warps(red, p.WK, p.M * COLS, i);
        }
        // reduce over the CTAs of the cluster through distributed shared memory
        cluster_sync();
        if (p.late_wait) grid_dependency_wait();
        const uint32_t part_addr = smem_u32(part);
        for (int i = rank + p.CS * (int)threadIdx.x; i < p.M * COLS; i += p.CS * blockDim.x) {
            float sacc = 0.0f;
            for (int r = 0; r < p.CS; ++r) sacc += ld_shared_cluster_f32(map_shared_rank(part_addr + 4u * i, r));
            const int m = i / COLS, col = col0 + i % COLS;
            if (col < p.N && check(m < p.M, &g_gemv_status)) {
                const float b = p.bias ? T16::load(p.bias[col]) : 0.0f;
                p.y[(size_t)m * p.N + col] = T16::store(sacc + b);
            }
        }
        cluster_sync();  // peers keep their shared memory until every read is done
    } else {
        if (p.late_wait) grid_dependency_wait();
        for (int i = threadIdx.x; i < p.M * COLS; i += blockDim.x) {
            const float sacc = sum_warps(red, p.WK, p.M * COLS, i);
            const int m = i / COLS, col = col0 + i % COLS;
            if (col < p.N && check(m < p.M, &g_gemv_status)) {
                const float b = p.bias ? T16::load(p.bias[col]) : 0.0f;
                p.y[(size_t)m * p.N + col] = T16::store(sacc + b);
            }
        }
    }
}

// ------------------------------------------------------------------- host
int ilog2(int v) {
    int r = 0;
    while ((1 << (r + 1)) <= v) ++r;
    return r;
}

static_assert(4 * sizeof(CUtensorMap) + sizeof(Params) <= sizeof(Prepared::args), "prepared launch arguments");

template <int BITS, int NT, bool BF>
wq_status run(const Problem& pb, cudaStream_t stream, Prepared* prep) {
    using F = Fmt<BITS>;
    constexpr int EPS = F::EPS;
    constexpr int QK = 4 * EPS;
    auto kern = gemv_kernel<BITS, NT, BF>;
    static std::atomic<uint64_t> attr_ctx[MAX_DEVICES];  // context the smem limit was raised in
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (const wq_status st = ensure_smem_attr((const void*)kern, 227 * 1024, attr_ctx, dev); st != WQ_OK) return st;
    Params prm{};
    prm.x = pb.x; prm.w_q = pb.w_q; prm.w_lo = pb.w_lo; prm.s = pb.scales; prm.z = pb.zeros;
    prm.bias = pb.bias;
    prm.y = pb.y; prm.M = pb.M; prm.K = pb.K; prm.N = pb.N; prm.G = pb.G;
    prm.late_wait = (pb.flags & WQ_FLAG_PDL_INPUTS_READY) ? 1 : 0;
    prm.Kw = pb.K / EPS;
    prm.Q = (prm.Kw + 3) / 4;
    prm.qpg = (pb.G == pb.K) ? (1 << 29) : pb.G / QK;
    prm.qpg_shift = (prm.qpg & (prm.qpg - 1)) == 0 ? ilog2(prm.qpg) : -1;
    prm.n_groups = (pb.K + pb.G - 1) / pb.G;
    const int colblocks = (pb.N + COLS - 1) / COLS;

    // The plan depends on the shape and flags only: computed once per device and
    // kept (its occupancy queries would otherwise cost more than the launch).
    // One map per instantiation (bit width, tokens per MMA, element type).
    struct Plan {
        Params q;
        size_t smem;
    };
    static std::mutex plan_mu;
    static std::map<std::array<int, 6>, Plan> plans;
    const std::array<int, 6> key{dev, pb.M, pb.K, pb.N, pb.G, prm.late_wait};
    bool found = false;
    Params best{};
    size_t best_smem = 0;
    {
        std::lock_guard<std::mutex> lk(plan_mu);
        const auto it = plans.find(key);
        if (it != plans.end()) {
            best = it->second.q;
            best_smem = it->second.smem;
            found = true;
        }
    }
    if (!found) {
        const int sms = sm_count();

        auto layout = [&](int WK, int CS, int QW, Params& q, bool one_slot = false) -> size_t {
            q.WK = WK; q.CS = CS; q.QW = QW;
            const int rows_cta = WK * QW * 4;
            const int quads_cta = WK * QW;
            const int ch = EPS >= 8 ? EPS : 8;
            q.cpt_shift = ilog2(rows_cta * EPS / ch);
            q.qc_shift = ilog2(quads_cta);
            q.groups_cta = std::min((quads_cta * QK + pb.G - 1) / pb.G + 1, (pb.K + pb.G - 1) / pb.G);
            q.xs_tok_stride = rows_cta * EPS * 2 + 16;
            q.nst = (QW > SQ && !one_slot) ? 2 : 1;
            size_t off = (size_t)WK * q.nst * stage_bytes<BITS>();
            q.off_bar = (uint32_t)off;
            off += (size_t)WK * MAXST * 8 + 8;  // per-warp stage barriers, then the s/z barrier
            off = (off + 127) & ~(size_t)127;
            q.sz_box = std::min(q.groups_cta, 256);
            q.sz_rows = (q.groups_cta + q.sz_box - 1) / q.sz_box * q.sz_box;
            q.off_sz = (uint32_t)off;
            q.sz_stride = (uint32_t)(((size_t)q.sz_rows * COLS * 2 + 127) & ~(size_t)127);
            off += (size_t)2 * q.sz_stride;
            q.off_x = (uint32_t)off;
            off += (size_t)pb.M * q.xs_tok_stride;
            off = (off + 15) & ~(size_t)15;
            q.off_xq = (uint32_t)off;
            off += (size_t)pb.M * quads_cta * 4;
            off = (off + 15) & ~(size_t)15;
            q.off_tab = (uint32_t)off;
            off += (size_t)q.groups_cta * COLS * sizeof(Rec<BITS, BF>);
            q.off_red = (uint32_t)off;
            off += (size_t)WK * pb.M * COLS * 4;
            q.off_part = (uint32_t)off;
            off += (size_t)pb.M * COLS * 4;
            return off + 1024;  // slack for aligning the base to 1024 bytes
        };

        long best_score = 0;
        // Products that overlap the previous one (WQ_FLAG_PDL_INPUTS_READY) gain
        // most from small CTAs: 8 warps and one stage slot per warp keep shared
        // memory low enough for three or more CTAs per SM, so several launches
        // stream at once.  Used when there are enough column blocks to fill the SMs.
        if (prm.late_wait && colblocks >= sms / 2) {
            int QW = 1;
            while (QW * 8 < prm.Q) QW <<= 1;
            Params q = prm;
            const size_t sm = layout(8, 1, QW, q, true);
            int occ = 0;
            if (sm <= 227 * 1024) {
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 8 * 32, sm);
                cudaGetLastError();
            }
            if (occ >= 3) {
                found = true;
                best = q;
                best_smem = sm;
            }
        }
        // Otherwise, among (warps per CTA, cluster size), pick the plan with the
        // fewest waves x quads per warp; ties go to no cluster and larger CTAs.
        for (int WK : {16, 8, 4}) {
            if (found && best_score == 0) break;
            for (int CS : {1, 2, 4, 8}) {
                if (CS > 1 && WK * CS > prm.Q) continue;
                int QW = 1;
                while (QW * WK * CS < prm.Q) QW <<= 1;
                Params q = prm;
                const size_t sm = layout(WK, CS, QW, q);
                if (sm > 227 * 1024) continue;
                int occ = 0;
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, WK * 32, sm);
                cudaGetLastError();
                if (occ <= 0) continue;
                const long ctas = (long)colblocks * CS;
                const long waves = (ctas + (long)occ * sms - 1) / ((long)occ * sms);
                // per-warp serial work (quads, at least a full ring of them) x waves,
                // plus a penalty for the cluster reduction
                const long score = waves * std::max(QW, SQ) * 64 + (CS > 1 ? 96 : 0) + (16 / WK);
                if (!found || score < best_score) {
                    found = true;
                    best = q;
                    best_smem = sm;
                    best_score = score;
                }
            }
        }
        if (!found) return WQ_ERR_INVALID_ARG;  // shape too large for the shared-memory plan
        std::lock_guard<std::mutex> lk(plan_mu);
        plans.emplace(key, Plan{best, best_smem});
    }
    // this call's arrays
    best.x = pb.x; best.w_q = pb.w_q; best.w_lo = pb.w_lo; best.s = pb.scales; best.z = pb.zeros;
    best.bias = pb.bias; best.y = pb.y;

    CUtensorMap mw, ml, ms, mz;
    bool ok = make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_q, pb.N, prm.Kw, (uint64_t)pb.N * 4, COLS, 4 * SQ,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.scales, pb.N, prm.n_groups, (uint64_t)pb.N * 2, COLS,
                        best.sz_box, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_map(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.zeros, pb.N, prm.n_groups, (uint64_t)pb.N * 2, COLS,
                        best.sz_box, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (BITS == 3)
        ok = ok && make_map(&ml, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_lo, pb.N, pb.K / 32, (uint64_t)pb.N * 4, COLS,
                            2 * SQ, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ml = mw;
    if (!ok) return WQ_ERR_CUDA;

    if (prep) {  // record the launch instead of making it
        Prepared& r = *prep;
        r.kern = (const void*)kern;
        r.grid = dim3(colblocks, best.CS, 1);
        r.block = dim3(best.WK * 32, 1, 1);
        r.smem = best_smem;
        r.cluster_y = best.CS > 1 ? (unsigned)best.CS : 1u;
        r.pdl = (pb.flags & (WQ_FLAG_PDL | WQ_FLAG_PDL_INPUTS_READY)) != 0;
        r.nargs = 5;
        const size_t mo = sizeof(CUtensorMap);
        const CUtensorMap* maps[4] = {&mw, &ml, &ms, &mz};
        for (int i = 0; i < 4; ++i) {
            std::memcpy(r.args + i * mo, maps[i], mo);
            r.arg_off[i] = i * mo;
        }
        std::memcpy(r.args + 4 * mo, &best, sizeof(best));
        r.arg_off[4] = 4 * mo;
        r.x_off = 4 * mo + offsetof(Params, x);
        r.y_off = 4 * mo + offsetof(Params, y);
        return WQ_OK;
    }

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(colblocks, best.CS, 1);
    cfg.blockDim = dim3(best.WK * 32, 1, 1);
    cfg.dynamicSmemBytes = best_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (best.CS > 1) {  // a cluster of one CTA is no cluster: launch without the attribute
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = best.CS;
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
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, mw, ml, ms, mz, best));
}

}  // namespace

wq_status gemv_device_status(int reset) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_gemv_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_gemv_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return (v & 1u) ? WQ_ERR_TIMEOUT : (v & 2u) ? WQ_ERR_CHECK : WQ_OK;
}

namespace {

template <bool BF>
wq_status launch_typed(const Problem& p, cudaStream_t s, Prepared* prep) {
    const bool two = p.M > 8;
    switch (p.bits) {
        case 1: return two ? run<1, 2, BF>(p, s, prep) : run<1, 1, BF>(p, s, prep);
        case 2: return two ? run<2, 2, BF>(p, s, prep) : run<2, 1, BF>(p, s, prep);
        case 3: return two ? run<3, 2, BF>(p, s, prep) : run<3, 1, BF>(p, s, prep);
        case 4: return two ? run<4, 2, BF>(p, s, prep) : run<4, 1, BF>(p, s, prep);
        case 8: return two ? run<8, 2, BF>(p, s, prep) : run<8, 1, BF>(p, s, prep);
        default: return WQ_ERR_UNSUPPORTED;
    }
}

}  // namespace

namespace {
wq_status gemv_route(const Problem& p, cudaStream_t s, Prepared* prep) {
    if (gemv_lean_takes(p)) {
        const wq_status st = launch_gemv_lean(p, s, prep);
        if (st != WQ_ERR_UNSUPPORTED) return st;  // else: its x stage does not fit; the kernel below takes it
    }
    return (p.flags & WQ_FLAG_BF16) ? launch_typed<true>(p, s, prep) : launch_typed<false>(p, s, prep);
}
}  // namespace

wq_status launch_gemv(const Problem& p, cudaStream_t s) { return gemv_route(p, s, nullptr); }

wq_status prepare_gemv(const Problem& p, Prepared& pr) { return gemv_route(p, nullptr, &pr); }

}  // namespace wq
