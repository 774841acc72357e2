// wq_gptq.cu -- GPTQ block quantisation of a weight matrix, fp32.
//
// What is computed: the "benchmark GPTQ implementations" page
// (`_prepare_weight_and_hessian`, `quantize_weight_eager` with the GROUP
// strategy, and the fake quantisation of `_quantize_block_triton_kernel`).
// W is (R, C) fp32, one row per output channel, H is (C, C).  Dead columns
// (H[c][c] == 0) get H[c][c] = 1 and W[:, c] = 0, and
// damp = percdamp * mean(diag H) is added to the diagonal.  The columns are
// then fake-quantised from left to right with their group's (s, z):
// q = clamp(rint(w / s) + z, -2^(b-1), 2^(b-1) - 1), w_hat = (q - z) s, where
// w is the column's current value; the error is spread over the later columns
// through the upper Cholesky factor U of H^-1 (the page's Hinv):
// w_j -= (w_i - w_hat_i) / U_ii * U_ij.  The loss is half the sum of
// ((w_i - w_hat_i) / U_ii)^2.
//
// How (sm_100a).  The page forms U with three dense factorisations (Cholesky
// factor of H, the inverse from it, Cholesky factor of the inverse).  One is
// enough here.  With J the order reversal, the lower Cholesky factor L of
// J H J gives H = V V^T with V = J L J upper triangular, and U = V^-1.  Let
// d_k = w_k - w_hat_k, with w_k the column's ORIGINAL value.  The column loop's
// errors satisfy E = D V (from W - W_hat = E U), and the current value of
// column j when it is quantised is
//     w_j + sum_{k<j} d_k V_kj / V_jj,
// so the loop needs V' = V diag(V)^-1 and no inverse; the loss term of column
// j is ((w_j' - w_hat_j) V_jj)^2 with w_j' that current value.
//
// Kernels.  The flipped, damped Hessian is factored in place by a blocked
// right-looking Cholesky (64-wide panels: the diagonal block and its inverse
// in one CTA, the panel as a product with that inverse, then the trailing
// lower triangle).  V' goes into the strictly upper triangle of the same
// array (its entry (k, j) comes from the factor's entry (C-1-k, C-1-j), so no
// entry is written that is still to be read).  Then, block by block of
// `blocksize` columns: one thread per row runs the column loop with the
// block's V' in shared memory, and an fp32 tile product adds the block's
// d V' to the running update of every later column (the page's
// W[:, i2:] -= Err1 Hinv[i1:i2, i2:]).  W, the running update and the block's
// d are kept K-major (C, R), so the row threads' per-column accesses are
// coalesced.  Everything is fp32 on the CUDA cores: the page fixes fp32, and
// TF32 tensor-core products would round the operands.
//
// Failure: a pivot that is not positive (H + damp not positive definite) sets
// bit 4 of the device status word (wq_device_status reports
// WQ_ERR_NOT_POSITIVE_DEFINITE); the factor then holds NaN and so do the
// outputs.  No kernel waits on anything.
#include <cuda_runtime.h>

#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {

__device__ unsigned int g_gptq_status = 0;

namespace {

constexpr int NB = 64;        // Cholesky panel width
constexpr int NBP = NB + 1;   // padded shared-memory row
constexpr int BMAX = 128;     // largest column block of the quantisation loop
constexpr int RT = 64;        // rows (threads) per CTA of the column loop
constexpr int RTP = RT + 1;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
    size_t p, wt, acc, dblk, vd, linv, damp, total;
};

Layout layout(int R, int C) {
    Layout l{};
    size_t o = 0;
    l.p = o;    o = align256(o + sizeof(float) * (size_t)C * C);
    l.wt = o;   o = align256(o + sizeof(float) * (size_t)C * R);
    l.acc = o;  o = align256(o + sizeof(float) * (size_t)C * R);
    l.dblk = o; o = align256(o + sizeof(float) * (size_t)BMAX * R);
    l.vd = o;   o = align256(o + sizeof(float) * (size_t)C);
    l.linv = o; o = align256(o + sizeof(float) * NB * NB);
    l.damp = o; o = align256(o + sizeof(float));
    l.total = o;
    return l;
}

// ---- set-up --------------------------------------------------------------

// damp = percdamp * mean(diag H), dead diagonal entries counted as 1.
__global__ void __launch_bounds__(1024) gptq_damp_kernel(const float* __restrict__ H, int C, float percdamp,
                                                         float* __restrict__ damp) {
    __shared__ float part[32];
    float s = 0.0f;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        const float h = H[(size_t)c * C + c];
        s += (h == 0.0f) ? 1.0f : h;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) *damp = percdamp * __fdiv_rn(s, (float)C);
    }
}

// P = J (H with dead diagonal entries 1, plus damp on the diagonal) J, lower triangle.
__global__ void gptq_flip_kernel(const float* __restrict__ H, int C, const float* __restrict__ damp,
                                 float* __restrict__ P) {
    const int j = blockIdx.x * 32 + threadIdx.x;
    const int i = blockIdx.y * 8 + threadIdx.y;
    if (i >= C || j > i) return;
    const int a = C - 1 - i, b = C - 1 - j;
    float h = H[(size_t)a * C + b];
    if (i == j) h = ((h == 0.0f) ? 1.0f : h) + *damp;
    P[(size_t)i * C + j] = h;
}

// Wt (C, R) = W^T, dead columns (H[c][c] == 0) zeroed; Acc = 0.
__global__ void gptq_transpose_kernel(const float* __restrict__ W, const float* __restrict__ H, int R, int C,
                                      float* __restrict__ Wt, float* __restrict__ Acc) {
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = r0 + y, c = c0 + threadIdx.x;
        tile[y][threadIdx.x] = (r < R && c < C) ? W[(size_t)r * C + c] : 0.0f;
    }
    __syncthreads();
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int c = c0 + y, r = r0 + threadIdx.x;
        if (c < C && r < R) {
            const bool dead = H[(size_t)c * C + c] == 0.0f;
            Wt[(size_t)c * R + r] = dead ? 0.0f : tile[threadIdx.x][y];
            Acc[(size_t)c * R + r] = 0.0f;
        }
    }
}

// ---- blocked Cholesky of P (lower, in place) -------------------------------

// The diagonal block at k0 (nb <= 64 wide, already updated by the earlier
// panels): factored in shared memory and its lower triangular inverse written
// to Linv (nb x nb, zeros above the diagonal).  Thread t owns row t.  The
// factorisation eliminates without square roots (after step j, the entries
// right of column j hold the Schur complement of the leading j + 1 columns),
// then scales column c by 1 / sqrt(pivot c); the inverse is formed row by row
// before the division by its diagonal.  One barrier per column; each thread's
// row updates issue their shared-memory loads eight at a time.
__global__ void __launch_bounds__(NB) chol_diag_kernel(float* __restrict__ P, int C, int k0, int nb,
                                                       float* __restrict__ Linv) {
    __shared__ float A[NB][NBP];
    __shared__ float Y[NB][NBP];
    __shared__ float sq[NB];
    const int t = threadIdx.x;
    for (int i0 = 0; i0 < NB; i0 += 16) {  // thread t reads column t of 16 rows: 16 loads in flight
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = i0 + u;
            v[u] = (i < nb && t <= i) ? P[(size_t)(k0 + i) * C + k0 + t] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            A[i0 + u][t] = v[u];
            Y[i0 + u][t] = (i0 + u == t) ? 1.0f : 0.0f;
        }
    }
    __syncthreads();
    const bool own = t < nb;
    for (int j = 0; j < nb; ++j) {
        if (own && t > j) {
            const float f = __fdiv_rn(A[t][j], A[j][j]);
            int c = j + 1;
            for (; c + 7 <= t; c += 8) {
                float a[8], r[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    a[u] = A[c + u][j];
                    r[u] = A[t][c + u];
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) A[t][c + u] = fmaf(-f, a[u], r[u]);
            }
            for (; c <= t; ++c) A[t][c] = fmaf(-f, A[c][j], A[t][c]);
        }
        __syncthreads();
    }
    if (own) {
        const float piv = A[t][t];
        if (!(piv > 0.0f)) atomicOr(&g_gptq_status, 4u);
        sq[t] = __fsqrt_rn(piv);  // NaN for a negative pivot
    }
    __syncthreads();
    if (own) {
        for (int c = 0; c < t; ++c) A[t][c] = __fdiv_rn(A[t][c], sq[c]);
        A[t][t] = sq[t];
    }
    __syncthreads();
    // rows of A^-1 before their division by the diagonal: Y_t -= (L_tk / L_kk) Y_k
    for (int k = 0; k < nb; ++k) {
        if (own && t > k) {
            const float f = __fdiv_rn(A[t][k], A[k][k]);
            int c = 0;
            for (; c + 7 <= k; c += 8) {
                float yk[8], yt[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    yk[u] = Y[k][c + u];
                    yt[u] = Y[t][c + u];
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) Y[t][c + u] = fmaf(-f, yk[u], yt[u]);
            }
            for (; c <= k; ++c) Y[t][c] = fmaf(-f, Y[k][c], Y[t][c]);
        }
        __syncthreads();
    }
    if (own)
        for (int c = 0; c <= t; ++c) Y[t][c] = __fdiv_rn(Y[t][c], A[t][t]);
    __syncthreads();
    for (int idx = t; idx < NB * NB; idx += NB) {
        const int i = idx / NB, c = idx % NB;
        if (i < nb && c <= i) P[(size_t)(k0 + i) * C + k0 + c] = A[i][c];
        if (i < nb && c < nb) Linv[i * NB + c] = (c <= i) ? Y[i][c] : 0.0f;
    }
}

// 64 x 64 tile product with both operands row-major along k (C = A B^T), k = nb <= 64.
//   panel:    P[i0.., k0..] = P[i0.., k0..] Linv^T          (the panel below the diagonal block)
//   trailing: P[i0.., m0..] -= P[i0.., k0..] P[m0.., k0..]^T (lower tiles of the trailing matrix)
// Each of the 256 threads computes a 4 x 4 patch.
template <bool PANEL>
__global__ void __launch_bounds__(256) chol_tile_kernel(float* __restrict__ P, int C, int k0, int nb,
                                                        const float* __restrict__ Linv) {
    __shared__ float As[NB][NBP];
    __shared__ float Bs[NB][NBP];
    const int tid = threadIdx.x;
    const int base = k0 + nb;  // first row after the panel's diagonal block
    int ti, tj;
    if (PANEL) {
        ti = blockIdx.x;
        tj = 0;
    } else {  // blockIdx.x -> (ti, tj), tj <= ti, row-major over the lower triangle of tiles
        ti = (int)((sqrtf(8.0f * (float)blockIdx.x + 1.0f) - 1.0f) * 0.5f);
        while ((ti + 1) * (ti + 2) / 2 <= (int)blockIdx.x) ++ti;
        while (ti * (ti + 1) / 2 > (int)blockIdx.x) --ti;
        tj = (int)blockIdx.x - ti * (ti + 1) / 2;
    }
    const int i0 = base + NB * ti, m0 = base + NB * tj;
    {  // 16 rows per thread, both operands: 32 loads in flight before the stores
        const int k = tid % NB, r0 = tid / NB;  // 256 threads: 4 rows per pass
        const bool kin = k < nb;
        float va[16], vb[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int r = r0 + 4 * u;
            va[u] = (kin && i0 + r < C) ? P[(size_t)(i0 + r) * C + k0 + k] : 0.0f;
            if (PANEL)
                vb[u] = (kin && r < nb) ? Linv[r * NB + k] : 0.0f;
            else
                vb[u] = (kin && m0 + r < C) ? P[(size_t)(m0 + r) * C + k0 + k] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            As[r0 + 4 * u][k] = va[u];
            Bs[r0 + 4 * u][k] = vb[u];
        }
    }
    __syncthreads();
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
#pragma unroll 8
    for (int k = 0; k < NB; ++k) {
        float a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            a[u] = As[ty * 4 + u][k];
            b[u] = Bs[tx + 16 * u][k];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= C) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int c = tx + 16 * v;
            if (PANEL) {
                if (c < nb) P[(size_t)i * C + k0 + c] = acc[u][v];
            } else {
                const int m = m0 + c;
                if (m < C && m <= i) P[(size_t)i * C + m] -= acc[u][v];
            }
        }
    }
}

// V' into the strictly upper triangle: P[k][j] = L[C-1-k][C-1-j] / L[C-1-j][C-1-j]
// for k < j; vd[j] = L[C-1-j][C-1-j] (= V_jj).
__global__ void gptq_vprime_kernel(float* __restrict__ P, int C, float* __restrict__ vd) {
    const int j = blockIdx.x * 32 + threadIdx.x;
    const int k = blockIdx.y * 8 + threadIdx.y;
    if (j >= C || k > j) return;
    const int b = C - 1 - j;
    const float djj = P[(size_t)b * C + b];
    if (k == j)
        vd[j] = djj;
    else
        P[(size_t)k * C + j] = __fdiv_rn(P[(size_t)(C - 1 - k) * C + b], djj);
}

// ---- the column loop --------------------------------------------------------

struct BlockParams {
    const float* P;       // V' in the strictly upper triangle
    const float* vd;      // V_jj
    const float* Wt;      // (C, R) original W, dead columns zeroed
    const float* Acc;     // (C, R) running update from the earlier blocks
    const float* scale;   // (R, NG)
    const float* zero;    // (R, NG)
    float* D;             // (cnt, R) d = w - w_hat of this block
    float* Q;             // (R, C) fake-quantised W, or null
    uint8_t* codes;       // (C, R) q + 2^(b-1), or null
    float* losses;        // (R,)
    int R, C, G, NG, i1, cnt;
    float qmin, qmax, half;
};

// One thread per row, RT rows per CTA.  Shared memory: the block's V'
// (cnt x cnt), the current values w' of the block's columns (column-major by
// thread, padded) and the original values, which are replaced by w_hat for the
// coalesced store of Q at the end.  The loop takes the block in sub-blocks of
// 32 columns held in registers.
__global__ void __launch_bounds__(RT) gptq_block_kernel(const BlockParams p) {
    extern __shared__ float sm[];
    const int cnt = p.cnt;
    float* Vs = sm;                        // cnt * cnt
    float* la = Vs + cnt * cnt;            // cnt * RTP: w' of column j for thread t at j * RTP + t
    float* wo = la + cnt * RTP;            // cnt * RTP: original w, then w_hat
    float* vds = wo + cnt * RTP;           // cnt: V_jj of the block's columns
    const int t = threadIdx.x;
    const int r0 = blockIdx.x * RT, r = r0 + t;
    const bool live = r < p.R;
    {  // V' of the block: each warp 4 rows per pass, each lane 4 columns: 16 loads in flight
        const int lane = t & 31, w = t >> 5;
        for (int ib = w * 4; ib < cnt; ib += 4 * (RT / 32)) {
            float v[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int i = ib + a, j = lane + 32 * b;
                    v[a][b] = (i < cnt && j < cnt && j > i) ? p.P[(size_t)(p.i1 + i) * p.C + p.i1 + j] : 0.0f;
                }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int i = ib + a, j = lane + 32 * b;
                    if (i < cnt && j < cnt) Vs[i * cnt + j] = v[a][b];
                }
        }
    }
    for (int j = t; j < cnt; j += RT) vds[j] = p.vd[p.i1 + j];
    for (int j0 = 0; j0 < cnt; j0 += 8) {  // the row's values: 16 loads in flight
        float w[8], a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const size_t g = (size_t)(p.i1 + j0 + u) * p.R + r;
            const bool in = live && j0 + u < cnt;
            w[u] = in ? p.Wt[g] : 0.0f;
            a[u] = in ? p.Acc[g] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (j0 + u < cnt) {
                la[(j0 + u) * RTP + t] = w[u] + a[u];
                wo[(j0 + u) * RTP + t] = w[u];
            }
        }
    }
    __syncthreads();
    float lsum = 0.0f, s = 1.0f, z = 0.0f;
    int gcur = -1;
    // sub-blocks of SB columns: their current values and errors in registers,
    // their errors then applied to the block's later columns as SB-term sums
    constexpr int SB = 32;
    for (int s0 = 0; s0 < cnt; s0 += SB) {
        float cur[SB], dl[SB];
#pragma unroll
        for (int u = 0; u < SB; ++u) cur[u] = (s0 + u < cnt) ? la[(s0 + u) * RTP + t] : 0.0f;
#pragma unroll
        for (int u = 0; u < SB; ++u) {
            dl[u] = 0.0f;
            const int i = s0 + u;
            if (i < cnt) {
                const int c = p.i1 + i;
                const int g = c / p.G;
                if (g != gcur) {
                    gcur = g;
                    s = live ? p.scale[(size_t)r * p.NG + g] : 1.0f;
                    z = live ? p.zero[(size_t)r * p.NG + g] : 0.0f;
                }
                const float wt = cur[u];
                float q = __fadd_rn(rintf(__fdiv_rn(wt, s)), z);  // nearbyint(w / s) + zp
                q = fminf(fmaxf(q, p.qmin), p.qmax);
                const float wh = __fmul_rn(__fsub_rn(q, z), s);
                const float e = __fmul_rn(__fsub_rn(wt, wh), vds[i]);  // (w - w_hat) / U_cc
                lsum = fmaf(e, e, lsum);
                dl[u] = __fsub_rn(wo[i * RTP + t], wh);
                wo[i * RTP + t] = wh;
                if (live) {
                    p.D[(size_t)i * p.R + r] = dl[u];
                    if (p.codes) p.codes[(size_t)c * p.R + r] = (uint8_t)(int)(q + p.half);
                }
                const float* vrow = Vs + i * cnt + s0;  // V'[i][s0 + v]
#pragma unroll
                for (int v = u + 1; v < SB; ++v) cur[v] = fmaf(dl[u], vrow[v < cnt - s0 ? v : 0], cur[v]);
            }
        }
        // the block's later columns: la[j] += sum_u dl[u] V'[s0 + u][j], four columns at a time
        for (int j = s0 + SB; j < cnt; j += 4) {
            float acc4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc4[k] = (j + k < cnt) ? la[(j + k) * RTP + t] : 0.0f;
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const float* vrow = Vs + (s0 + u) * cnt + j;
#pragma unroll
                for (int k = 0; k < 4; ++k) acc4[k] = fmaf(dl[u], (j + k < cnt) ? vrow[k] : 0.0f, acc4[k]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (j + k < cnt) la[(j + k) * RTP + t] = acc4[k];
        }
    }
    if (live) p.losses[r] += 0.5f * lsum;
    __syncthreads();
    if (p.Q) {
        for (int idx = t; idx < RT * cnt; idx += RT) {
            const int row = idx / cnt, col = idx % cnt;
            if (r0 + row < p.R) p.Q[(size_t)(r0 + row) * p.C + p.i1 + col] = wo[col * RTP + row];
        }
    }
}

// ---- the block update: Acc[j][r] += sum_k V'[i1+k][j] D[k][r], j >= i2 -----

constexpr int UT = 128;  // output tile (j and r)
constexpr int UK = 8;    // k chunk

// 256 threads, 8 x 8 outputs each.  The next k chunk is read into registers
// while the current one is multiplied from shared memory (two buffers, one
// barrier per chunk).  VEC: C, R and i2 multiples of 4, so every global access
// is a 16-byte vector.
template <bool VEC>
__global__ void __launch_bounds__(256) gptq_update_kernel(const float* __restrict__ P, const float* __restrict__ D,
                                                          float* __restrict__ Acc, int R, int C, int i1, int cnt,
                                                          int i2) {
    __shared__ __align__(16) float As[2][UK][UT];
    __shared__ __align__(16) float Bs[2][UK][UT];
    const int tid = threadIdx.x;
    const int j0 = i2 + blockIdx.x * UT, rb = blockIdx.y * UT;
    const int ty = tid / 16, tx = tid % 16;
    const int lk = tid / 32, lc = (tid % 32) * 4;  // loader: one k row, four columns
    float acc[8][8] = {};
    float pa[4], pb[4];
    auto fetch = [&](int k0) {
        const int k = k0 + lk;
        const int j = j0 + lc, rr = rb + lc;
        if (VEC) {
            const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 a4 = (k < cnt && j < C) ? *reinterpret_cast<const float4*>(P + (size_t)(i1 + k) * C + j) : z4;
            const float4 b4 = (k < cnt && rr < R) ? *reinterpret_cast<const float4*>(D + (size_t)k * R + rr) : z4;
            pa[0] = a4.x; pa[1] = a4.y; pa[2] = a4.z; pa[3] = a4.w;
            pb[0] = b4.x; pb[1] = b4.y; pb[2] = b4.z; pb[3] = b4.w;
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                pa[u] = (k < cnt && j + u < C) ? P[(size_t)(i1 + k) * C + j + u] : 0.0f;
                pb[u] = (k < cnt && rr + u < R) ? D[(size_t)k * R + rr + u] : 0.0f;
            }
        }
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            As[buf][lk][lc + u] = pa[u];
            Bs[buf][lk][lc + u] = pb[u];
        }
    };
    const int nchunk = (cnt + UK - 1) / UK;
    fetch(0);
    stash(0);
    __syncthreads();
    for (int kc = 0; kc < nchunk; ++kc) {
        const int buf = kc & 1;
        if (kc + 1 < nchunk) fetch((kc + 1) * UK);
#pragma unroll
        for (int kk = 0; kk < UK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        if (kc + 1 < nchunk) stash(buf ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int j = j0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
        if (j >= C) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r4 = rb + h * 64 + tx * 4;
            float* dst = Acc + (size_t)j * R + r4;
            if (VEC) {
                if (r4 < R) {
                    float4 o = *reinterpret_cast<float4*>(dst);
                    o.x += acc[u][4 * h + 0];
                    o.y += acc[u][4 * h + 1];
                    o.z += acc[u][4 * h + 2];
                    o.w += acc[u][4 * h + 3];
                    *reinterpret_cast<float4*>(dst) = o;
                }
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    if (r4 + v < R) dst[v] += acc[u][4 * h + v];
            }
        }
    }
}

}  // namespace

size_t gptq_workspace_bytes(int R, int C) { return layout(R, C).total; }

wq_status launch_gptq(const float* W, const float* H, const float* scale, const float* zero, int R, int C, int G,
                      int bits, int blocksize, float percdamp, float* Q, uint8_t* codes, float* losses,
                      void* workspace, cudaStream_t s) {
    const Layout l = layout(R, C);
    char* ws = static_cast<char*>(workspace);
    float* P = reinterpret_cast<float*>(ws + l.p);
    float* Wt = reinterpret_cast<float*>(ws + l.wt);
    float* Acc = reinterpret_cast<float*>(ws + l.acc);
    float* D = reinterpret_cast<float*>(ws + l.dblk);
    float* vd = reinterpret_cast<float*>(ws + l.vd);
    float* Linv = reinterpret_cast<float*>(ws + l.linv);
    float* damp = reinterpret_cast<float*>(ws + l.damp);

    if (cudaMemsetAsync(losses, 0, sizeof(float) * (size_t)R, s) != cudaSuccess) return WQ_ERR_CUDA;
    gptq_damp_kernel<<<1, 1024, 0, s>>>(H, C, percdamp, damp);
    gptq_flip_kernel<<<dim3((C + 31) / 32, (C + 7) / 8), dim3(32, 8), 0, s>>>(H, C, damp, P);
    gptq_transpose_kernel<<<dim3((C + 31) / 32, (R + 31) / 32), dim3(32, 8), 0, s>>>(W, H, R, C, Wt, Acc);
    for (int k0 = 0; k0 < C; k0 += NB) {
        const int nb = C - k0 < NB ? C - k0 : NB;
        chol_diag_kernel<<<1, NB, 0, s>>>(P, C, k0, nb, Linv);
        const int rest = C - k0 - nb;
        if (rest > 0) {
            const int T = (rest + NB - 1) / NB;
            chol_tile_kernel<true><<<T, 256, 0, s>>>(P, C, k0, nb, Linv);
            chol_tile_kernel<false><<<T * (T + 1) / 2, 256, 0, s>>>(P, C, k0, nb, Linv);
        }
    }
    gptq_vprime_kernel<<<dim3((C + 31) / 32, (C + 7) / 8), dim3(32, 8), 0, s>>>(P, C, vd);
    if (cudaGetLastError() != cudaSuccess) return WQ_ERR_CUDA;

    const int NG = (C + G - 1) / G;
    const size_t smem_max = sizeof(float) * ((size_t)BMAX * BMAX + 2 * (size_t)BMAX * RTP + BMAX);
    static std::atomic<uint64_t> attr_ctx[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (const wq_status st = ensure_smem_attr((const void*)gptq_block_kernel, (int)smem_max, attr_ctx, dev);
        st != WQ_OK)
        return st;
    BlockParams bp{P, vd, Wt, Acc, scale, zero, D, Q, codes, losses, R, C, G, NG, 0, 0,
                   (float)(-(1 << (bits - 1))), (float)((1 << (bits - 1)) - 1), (float)(1 << (bits - 1))};
    for (int i1 = 0; i1 < C; i1 += blocksize) {
        const int cnt = C - i1 < blocksize ? C - i1 : blocksize;
        bp.i1 = i1;
        bp.cnt = cnt;
        const size_t smem = sizeof(float) * ((size_t)cnt * cnt + 2 * (size_t)cnt * RTP + cnt);
        gptq_block_kernel<<<(R + RT - 1) / RT, RT, smem, s>>>(bp);
        const int i2 = i1 + cnt;
        if (i2 < C) {
            const dim3 grid((C - i2 + UT - 1) / UT, (R + UT - 1) / UT);
            if ((C % 4) == 0 && (R % 4) == 0 && (i2 % 4) == 0)
                gptq_update_kernel<true><<<grid, 256, 0, s>>>(P, D, Acc, R, C, i1, cnt, i2);
            else
                gptq_update_kernel<false><<<grid, 256, 0, s>>>(P, D, Acc, R, C, i1, cnt, i2);
        }
    }
    return cudaGetLastError() == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status gptq_device_status(int reset) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_gptq_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
    if (reset && v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_gptq_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return (v & 4u) ? WQ_ERR_NOT_POSITIVE_DEFINITE : WQ_OK;
}

}  // namespace wq
