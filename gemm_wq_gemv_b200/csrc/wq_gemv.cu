// wq_gemv.cu -- decode-time product y (M x N) = x (M x K) @ dequant(W_q), 1 <= M <= 16.
//
// What is computed: dashq_kernel.py `_dashq_gemv_kernel` (one token there; up to
// 16 here): each output column n is sum_k x[k] * (q[k][n] - z[g][n]) * s[g][n],
// g = k / G, with fp32 accumulation and one fp16 rounding at the end.
//
// How (sm_100a):
//  * Work split.  A CTA owns 32 output columns and a contiguous range of K; the
//    CTAs of one thread-block cluster split K further and reduce their fp32
//    partial sums through distributed shared memory (one launch, no workspace,
//    no atomics).  Inside a CTA, 8 warps split K again; lanes never need a
//    shuffle because the reduction over k happens inside the MMA.
//  * Loads.  Lane (g, t) of a warp (g = lane / 4, t = lane % 4) reads one
//    128-bit vector = 4 adjacent columns of one packed word row; the 8 lanes
//    with the same t read 128 contiguous bytes.  Loads bypass L1 and are marked
//    evict-first in L2; each warp keeps PD quads (4 word rows) in flight.
//  * Dequant.  A code pair (code j, code j + eps/2), which sits in the two
//    16-bit halves of a word at the same offset, is ORed into the mantissa of
//    the fp16 constant 1024 (0x6400) with one LOP3, then one exact fp16x2 FMA
//    scales it down and subtracts 1024 and the integer part of the zero point:
//    the result q - round(z) is exact in fp16.
//  * Dot product.  The exact (q - round(z)) values are the A operand of a warp
//    MMA m16n8k16 (fp16 in, fp32 accumulate) with x as the B operand: rows of
//    A are 16 output columns, the 16 k-slots are 4 word rows x 4 codes.  The
//    k-slots are a permutation of k; x is staged in shared memory in the same
//    permuted order, once per CTA.
//  * Per group, the fp32 MMA sum is scaled: acc += s * (D - (z - round(z)) * X),
//    X = sum of the x values of that group slice, so fractional zero points are
//    exact too and q == z gives exactly 0.
#include <algorithm>

#include "wq_dequant.cuh"
#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {
namespace {

constexpr int COLS = 32;    // output columns per CTA
constexpr int MAXW = 8;     // warps per CTA (split along K)
// quads (4 word rows) each warp keeps in flight
template <int BITS, int NT> constexpr int pd_for() { return (BITS == 3 || (BITS == 1 && NT == 2)) ? 4 : 8; }

// ------------------------------------------------------------------ kernel
struct Params {
    const uint16_t* x;
    const uint32_t* w_q;
    const uint32_t* w_lo;
    const uint16_t* s;
    const uint16_t* z;
    uint16_t* y;
    int M, K, N, G;
    int Kw;        // word rows of the main plane
    int Q;         // quads = ceil(Kw / 4)
    int QW;        // quads per warp
    int WK;        // warps per CTA
    int CS;        // CTAs per cluster (along K)
    int rows_cta;  // word rows staged per CTA = WK * QW * 4
    int groups_cta;
    int qpg;       // quads per group (a large number when one group spans K)
    int cpt_shift; // log2(x chunks per token staged by a CTA)
    int qc_shift;  // log2(quads per CTA)
    int xs_tok_stride;  // bytes between tokens in the x stage (padded)
    uint32_t off_xq, off_tab, off_red, off_part;  // smem byte offsets
};

template <int BITS, int NT>
__global__ void __launch_bounds__(MAXW * 32, 2)
gemv_kernel(const Params p) {
    using F = Fmt<BITS>;
    constexpr int EPS = F::EPS;
    constexpr int NC = F::NC;
    constexpr int QK = 4 * EPS;  // k values per quad
    constexpr int MMAS = EPS / 4;
    constexpr int PD = pd_for<BITS, NT>();
    extern __shared__ __align__(16) uint8_t smem[];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int rank = (int)blockIdx.y;  // cluster spans the whole grid y extent
    const int col0 = blockIdx.x * COLS;
    const int mycol = col0 + 4 * g;
    const bool col_ok = mycol < p.N;

    // quad range of the CTA and of this warp
    const int cta_q0 = rank * p.WK * p.QW;
    const int q_begin = cta_q0 + warp * p.QW;
    const int q_end = min(p.Q, q_begin + p.QW);
    const int nq = max(0, q_end - q_begin);

    const uint64_t pol = policy_evict_first();

    // ---- (1) W: issue the first PD quads before anything else (weights need no dependency wait)
    uint4 buf[PD];
    uint4 bufl[PD];
    auto load_quad = [&](int q, uint4& hv, uint4& lv) {
        const int r = 4 * q + t;
        if (col_ok && r < p.Kw) {
            hv = ld_stream_v4(p.w_q + (size_t)r * p.N + mycol, pol);
            if constexpr (BITS == 3)
                lv = ld_stream_v4(p.w_lo + (size_t)(r >> 1) * p.N + mycol, pol);
        } else {
            hv = make_uint4(0, 0, 0, 0);
            lv = make_uint4(0, 0, 0, 0);
        }
    };
#pragma unroll
    for (int j = 0; j < PD; ++j) {
        if (j < nq) load_quad(q_begin + j, buf[j], bufl[j]);
    }

    // ---- (2) s, z of the CTA's (group, column) records: first round of loads now
    const int k_cta0 = cta_q0 * QK;
    const int g_cta0 = min(k_cta0, p.K - 1) / p.G;
    const int n_groups = (p.K + p.G - 1) / p.G;
    const int nrec = p.groups_cta * COLS;
    Rec<BITS>* tab = reinterpret_cast<Rec<BITS>*>(smem + p.off_tab);
    constexpr int TB = 4;
    bool any_frac = false;
    auto tab_load = [&](int base, uint32_t (&v)[TB]) {
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const int i = base + u * (int)blockDim.x + (int)threadIdx.x;
            const int gg = g_cta0 + i / COLS, col = col0 + i % COLS;
            v[u] = 0u;
            if (i < nrec && col < p.N && gg < n_groups) {
                const size_t o = (size_t)gg * p.N + col;
                v[u] = (uint32_t)p.s[o] | ((uint32_t)p.z[o] << 16);
            }
        }
    };
    auto tab_store = [&](int base, const uint32_t (&v)[TB]) {
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const int i = base + u * (int)blockDim.x + (int)threadIdx.x;
            if (i < nrec) {
                // a column or group outside the matrix gets s = 0 and z = 0
                const float s = __half2float(__ushort_as_half((uint16_t)(v[u] & 0xffffu)));
                const float z = __half2float(__ushort_as_half((uint16_t)(v[u] >> 16)));
                const float zi = fminf(fmaxf(rintf(z), -256.0f), 256.0f);
                Rec<BITS> rec;
                rec.s = s;
                rec.zr = z - zi;
                any_frac |= (rec.zr != 0.0f);
#pragma unroll
                for (int ci = 0; ci < NC; ++ci) rec.c[ci] = dup_half(-(bias_magnitude<BITS>(ci) + zi));
                tab[i] = rec;
            }
        }
    };
    uint32_t tv[TB];
    tab_load(0, tv);

    // ---- (3) x may come from the previous kernel on the stream: wait, then load it
    grid_dependency_wait();

    // x is staged per token in k-slot order: word row r holds the pairs
    // (x[r*EPS + j], x[r*EPS + j + EPS/2]), j < EPS/2.  A chunk is one word row
    // (two for 8-bit), read as 16-byte vectors.
    constexpr int CH = EPS >= 8 ? EPS : 8;        // halves per chunk
    constexpr int UPC = CH / 8;                   // 16-byte vectors per chunk
    constexpr int XB = UPC >= 4 ? 1 : (UPC == 2 ? 2 : 4);  // chunks per thread per round
    const int row_cta0 = cta_q0 * 4;
    const int cpt = 1 << p.cpt_shift;             // chunks per token (rows_cta * EPS / CH)
    const int nchunk = p.M * cpt;
    auto x_load = [&](int base, uint4 (&v)[XB][UPC]) {
#pragma unroll
        for (int u = 0; u < XB; ++u) {
            const int c = base + u * (int)blockDim.x + (int)threadIdx.x;
            const int m = c >> p.cpt_shift, ci = c & (cpt - 1);
            const int k0 = (row_cta0 + ci * (CH / EPS)) * EPS;
            const uint16_t* src = p.x + (size_t)m * p.K + k0;
#pragma unroll
            for (int w = 0; w < UPC; ++w) v[u][w] = make_uint4(0, 0, 0, 0);
            if (c < nchunk) {
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
                uint8_t* dst = smem + m * p.xs_tok_stride + (size_t)ci * CH * 2;
#pragma unroll
                for (int w = 0; w < UPC; ++w)
                    *reinterpret_cast<uint4*>(dst + 16 * w) = make_uint4(P[4 * w], P[4 * w + 1], P[4 * w + 2], P[4 * w + 3]);
            }
        }
    };
    {
        uint4 xv[XB][UPC];
        x_load(0, xv);
        tab_store(0, tv);
        for (int base = TB * (int)blockDim.x; base < nrec; base += TB * (int)blockDim.x) {
            tab_load(base, tv);
            tab_store(base, tv);
        }
        x_store(0, xv);
        for (int base = XB * (int)blockDim.x; base < nchunk; base += XB * (int)blockDim.x) {
            x_load(base, xv);
            x_store(base, xv);
        }
    }
    // fractional zero points anywhere in this CTA's records?  (CTA-uniform)
    const bool frac = __syncthreads_or(any_frac) != 0;

    // ---- (4) per-quad x sums (fp32) from the staged x, for the fractional zero-point term
    const int quads_cta = 1 << p.qc_shift;
    if (frac) {
        float* xqw = reinterpret_cast<float*>(smem + p.off_xq);
        for (int i = threadIdx.x; i < p.M * quads_cta; i += blockDim.x) {
            const int m = i >> p.qc_shift, ql = i & (quads_cta - 1);
            const uint4* src = reinterpret_cast<const uint4*>(smem + m * p.xs_tok_stride + (size_t)ql * QK * 2);
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int w = 0; w < QK / 8; ++w) {
                const uint4 u = src[w];
                const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&e[h]));
                    a0 += f.x;
                    a1 += f.y;
                }
            }
            xqw[i] = a0 + a1;
        }
        __syncthreads();
    }
    grid_launch_dependents();

    const float* xq = reinterpret_cast<const float*>(smem + p.off_xq);

    float acc[4][NT][2];
    float dsum[2][NT][4];
    float xs_sum[NT][2];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[c][n][0] = acc[c][n][1] = 0.0f;
#pragma unroll
    for (int T = 0; T < 2; ++T)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) dsum[T][n][i] = 0.0f;
#pragma unroll
    for (int n = 0; n < NT; ++n) xs_sum[n][0] = xs_sum[n][1] = 0.0f;

    // token rows feeding the B operand of this lane (duplicates beyond M are harmless)
    const uint8_t* xb[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) xb[n] = smem + min(g + 8 * n, p.M - 1) * p.xs_tok_stride;
    int tok[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        tok[n][0] = 2 * t + 8 * n;
        tok[n][1] = 2 * t + 1 + 8 * n;
    }
    // group bookkeeping without divisions in the loop
    int gl = (q_begin * QK) / p.G - g_cta0;
    int left = p.qpg - ((q_begin * QK) % p.G) / QK;  // quads left in the current group
    // bias constants of the lane's 4 columns, held in registers for narrow records
    constexpr bool CREG = NC <= 2;
    uint32_t creg[4][CREG ? NC : 1];
    auto load_creg = [&](int gidx) {
        if constexpr (CREG) {
            const Rec<BITS>* r = tab + gidx * COLS + 4 * g;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int ci = 0; ci < NC; ++ci) creg[c][ci] = r[c].c[ci];
        }
    };
    if (nq > 0) load_creg(gl);
    const uint32_t lo_sel = (t & 1) ? 0x7372u : 0x7170u;  // 3-bit: which half of the lo word

    for (int base = 0; base < nq; base += PD) {
#pragma unroll
        for (int jj = 0; jj < PD; ++jj) {
            const int i = base + jj;
            if (i < nq) {
                const int q = q_begin + i;
                const uint4 hv = buf[jj];
                const uint4 lv = bufl[jj];
                if (i + PD < nq) load_quad(q + PD, buf[jj], bufl[jj]);

                const int ql = q - cta_q0;
                const Rec<BITS>* rc = tab + gl * COLS + 4 * g;

                // B fragments: this lane's word row of the quad, all MMAS pairs
                const int rl = 4 * ql + t;
                uint32_t bx[NT][EPS / 2];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
#pragma unroll
                    for (int v = 0; v < EPS / 8; ++v) {
                        const uint4 u = *reinterpret_cast<const uint4*>(xb[n] + (size_t)rl * EPS * 2 + 16 * v);
                        bx[n][4 * v + 0] = u.x;
                        bx[n][4 * v + 1] = u.y;
                        bx[n][4 * v + 2] = u.z;
                        bx[n][4 * v + 3] = u.w;
                    }
                    if constexpr (EPS / 8 == 0) {
                        const uint2 u = *reinterpret_cast<const uint2*>(xb[n] + (size_t)rl * EPS * 2);
                        bx[n][0] = u.x;
                        bx[n][1] = u.y;
                    }
                }
                // x sums of this quad for the tokens this lane accumulates
                if (frac) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        xs_sum[n][0] += (tok[n][0] < p.M) ? xq[tok[n][0] * quads_cta + ql] : 0.0f;
                        xs_sum[n][1] += (tok[n][1] < p.M) ? xq[tok[n][1] * quads_cta + ql] : 0.0f;
                    }
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
                            cA[ci] = rc[ca].c[ci];
                            cB[ci] = rc[cb].c[ci];
                        }
                    }
                    uint32_t wA = wv[ca], wB = wv[cb], wAh, wBh, lA = 0, lB = 0;
                    if constexpr (BITS == 4) { wAh = wA >> 8; wBh = wB >> 8; }
                    else if constexpr (BITS == 2 || BITS == 1) { wAh = wA >> 10; wBh = wB >> 10; }
                    else if constexpr (BITS == 3) {
                        wAh = wA >> 7; wBh = wB >> 7;
                        wA <<= 1; wB <<= 1;
                        lA = prmt(lw[ca], 0u, lo_sel) << 1;
                        lB = prmt(lw[cb], 0u, lo_sel) << 1;
                    } else { wAh = wA; wBh = wB; }
#pragma unroll
                    for (int h = 0; h < MMAS; ++h) {
                        uint32_t a[4];
                        a[0] = pair_q<BITS>(wA, wAh, lA, cA, 2 * h);
                        a[1] = pair_q<BITS>(wB, wBh, lB, cB, 2 * h);
                        a[2] = pair_q<BITS>(wA, wAh, lA, cA, 2 * h + 1);
                        a[3] = pair_q<BITS>(wB, wBh, lB, cB, 2 * h + 1);
#pragma unroll
                        for (int n = 0; n < NT; ++n) mma_16816(dsum[T][n], a, bx[n][2 * h], bx[n][2 * h + 1]);
                    }
                }

                // end of a group (or of this warp's range): scale and fold into acc
                --left;
                const bool last = (i == nq - 1) || left == 0;
                if (last) {
#pragma unroll
                    for (int T = 0; T < 2; ++T) {
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const int c = 2 * T + half;
                            const float s = rc[c].s;
                            const float zr = frac ? rc[c].zr : 0.0f;
#pragma unroll
                            for (int n = 0; n < NT; ++n) {
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const float d = frac ? dsum[T][n][2 * half + e] - zr * xs_sum[n][e]
                                                         : dsum[T][n][2 * half + e];
                                    acc[c][n][e] = fmaf(s, d, acc[c][n][e]);
                                }
                            }
                        }
#pragma unroll
                        for (int n = 0; n < NT; ++n)
#pragma unroll
                            for (int e = 0; e < 4; ++e) dsum[T][n][e] = 0.0f;
                    }
#pragma unroll
                    for (int n = 0; n < NT; ++n) xs_sum[n][0] = xs_sum[n][1] = 0.0f;
                    if (left == 0) {
                        ++gl;
                        left = p.qpg;
                        if (i + 1 < nq) load_creg(gl);
                    }
                }
            }
        }
    }

    // ---- reduce over the warps of the CTA
    float* red = reinterpret_cast<float*>(smem + p.off_red);  // [WK][M][COLS]
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int m = tok[n][e];
                if (m < p.M) red[(warp * p.M + m) * COLS + 4 * g + c] = acc[c][n][e];
            }
    __syncthreads();
    float* part = reinterpret_cast<float*>(smem + p.off_part);  // [M][COLS]
    for (int i = threadIdx.x; i < p.M * COLS; i += blockDim.x) {
        float sacc = 0.0f;
        for (int w = 0; w < p.WK; ++w) sacc += red[w * p.M * COLS + i];
        part[i] = sacc;
    }

    // ---- reduce over the CTAs of the cluster through distributed shared memory
    if (p.CS > 1) {
        cluster_sync();
        const uint32_t part_addr = smem_u32(part);
        for (int i = rank + p.CS * (int)threadIdx.x; i < p.M * COLS; i += p.CS * blockDim.x) {
            float sacc = 0.0f;
            for (int r = 0; r < p.CS; ++r) sacc += ld_shared_cluster_f32(map_shared_rank(part_addr + 4u * i, r));
            const int m = i / COLS, col = col0 + i % COLS;
            if (col < p.N) p.y[(size_t)m * p.N + col] = __half_as_ushort(__float2half_rn(sacc));
        }
        cluster_sync();  // peers keep their shared memory until every read is done
    } else {
        __syncthreads();
        for (int i = threadIdx.x; i < p.M * COLS; i += blockDim.x) {
            const int m = i / COLS, col = col0 + i % COLS;
            if (col < p.N) p.y[(size_t)m * p.N + col] = __half_as_ushort(__float2half_rn(part[i]));
        }
    }
}

// ------------------------------------------------------------------- host
int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int BITS>
size_t rec_bytes() { return sizeof(Rec<BITS>); }

int ilog2(int v) {
    int r = 0;
    while ((1 << (r + 1)) <= v) ++r;
    return r;
}

template <int BITS, int NT>
wq_status run(const Problem& pb, cudaStream_t stream) {
    using F = Fmt<BITS>;
    constexpr int EPS = F::EPS;
    constexpr int QK = 4 * EPS;
    auto kern = gemv_kernel<BITS, NT>;
    static unsigned long long attr_done = 0;  // one bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (dev < 64 && !(attr_done & (1ull << dev))) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess)
            return WQ_ERR_CUDA;
        attr_done |= 1ull << dev;
    }
    Params prm{};
    prm.x = pb.x; prm.w_q = pb.w_q; prm.w_lo = pb.w_lo; prm.s = pb.scales; prm.z = pb.zeros;
    prm.y = pb.y; prm.M = pb.M; prm.K = pb.K; prm.N = pb.N; prm.G = pb.G;
    prm.Kw = pb.K / EPS;
    prm.Q = (prm.Kw + 3) / 4;
    prm.qpg = (pb.G == pb.K) ? (1 << 29) : pb.G / QK;
    const int colblocks = (pb.N + COLS - 1) / COLS;
    const int WK = std::min(MAXW, std::max(1, prm.Q >= 8 ? 8 : (prm.Q >= 4 ? 4 : (prm.Q >= 2 ? 2 : 1))));
    const int sms = sm_count();

    auto smem_for = [&](int CS, int QW, Params& q) -> size_t {
        q.WK = WK; q.CS = CS; q.QW = QW;
        q.rows_cta = WK * QW * 4;
        const int quads_cta = WK * QW;
        const int ch = EPS >= 8 ? EPS : 8;
        q.cpt_shift = ilog2(q.rows_cta * EPS / ch);
        q.qc_shift = ilog2(quads_cta);
        const int k0 = 0, k1 = quads_cta * QK;  // span of one CTA
        q.groups_cta = std::min((k1 - k0 + pb.G - 1) / pb.G + 1, (pb.K + pb.G - 1) / pb.G);
        q.xs_tok_stride = q.rows_cta * EPS * 2 + 16;
        size_t off = (size_t)pb.M * q.xs_tok_stride;
        off = (off + 15) & ~(size_t)15;
        q.off_xq = (uint32_t)off;
        off += (size_t)pb.M * quads_cta * 4;
        off = (off + 15) & ~(size_t)15;
        q.off_tab = (uint32_t)off;
        off += (size_t)q.groups_cta * COLS * rec_bytes<BITS>();
        q.off_red = (uint32_t)off;
        off += (size_t)WK * pb.M * COLS * 4;
        q.off_part = (uint32_t)off;
        off += (size_t)pb.M * COLS * 4;
        return off;
    };

    // Pick the widest cluster split whose grid is resident in one wave.
    int best_cs = 1;
    Params chosen{};
    size_t chosen_smem = 0;
    bool found = false;
    for (int CS = 8; CS >= 1; CS >>= 1) {
        if (WK * CS > prm.Q && CS > 1) continue;
        int QW = 1;
        while (QW * WK * CS < prm.Q) QW <<= 1;
        Params q = prm;
        const size_t sm = smem_for(CS, QW, q);
        if (sm > 227 * 1024) continue;
        int occ = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, WK * 32, sm);
        cudaGetLastError();
        if (occ <= 0) continue;
        if ((long)colblocks * CS <= (long)occ * sms || CS == 1) {
            best_cs = CS;
            chosen = q;
            chosen_smem = sm;
            found = true;
            break;
        }
    }
    if (!found) return WQ_ERR_INVALID_ARG;  // shape too large for the shared-memory plan
    (void)best_cs;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(colblocks, chosen.CS, 1);
    cfg.blockDim = dim3(WK * 32, 1, 1);
    cfg.dynamicSmemBytes = chosen_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = 1;
    attrs[na].val.clusterDim.y = chosen.CS;
    attrs[na].val.clusterDim.z = 1;
    ++na;
    if (pb.flags & WQ_FLAG_PDL) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, chosen));
}

}  // namespace

wq_status launch_gemv(const Problem& p, cudaStream_t s) {
    const bool two = p.M > 8;
    switch (p.bits) {
        case 1: return two ? run<1, 2>(p, s) : run<1, 1>(p, s);
        case 2: return two ? run<2, 2>(p, s) : run<2, 1>(p, s);
        case 3: return two ? run<3, 2>(p, s) : run<3, 1>(p, s);
        case 4: return two ? run<4, 2>(p, s) : run<4, 1>(p, s);
        case 8: return two ? run<8, 2>(p, s) : run<8, 1>(p, s);
        default: return WQ_ERR_UNSUPPORTED;
    }
}

}  // namespace wq
