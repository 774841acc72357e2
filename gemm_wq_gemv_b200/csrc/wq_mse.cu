// wq_mse.cu -- MSE-observer search of per-group scales and zero points.
//
// What is computed: the "Benchmark for MSE observer grid search" page
// (`grid_search_eager`, `grid_search_eager_no_patience`, and the fake
// quantisation of `_fused_grid_search_kernel`).  W is (rows, cols) fp32, groups
// are `G` consecutive values of a row.  For every group, with mn, mx its
// minimum and maximum, candidate i < steps shrinks the range by
// p_i = 1 - i / grid (lo = mn p_i, hi = mx p_i), derives (s, z) from it, fake
// quantises the group (q = clamp(rint(w / s + z)), w_hat = (q - z) s) and
// scores err_i = sum |w_hat - w|^norm.  The first candidate with the smallest
// error wins (a later one replaces it only when strictly smaller).  With
// patience the search stops after `patience` candidates in a row in which no
// group of the whole tensor improved; the winner is then the best candidate
// evaluated before the stop.
//
// Parameter rules (the page imports them without printing them):
//   affine (unsigned codes [0, 2^b - 1]): the range widened to contain 0,
//     s = (hi - lo) / (2^b - 1), z = clamp(-rint(lo / s)) (Jacob et al. 2018,
//     section 2.1);
//   symmetric (signed codes [-2^(b-1), 2^(b-1) - 1]): s = max(|lo|, |hi|) /
//     ((2^b - 1) / 2), z = 0.
//   A zero scale becomes 2^-23.
//
// How (sm_100a).  One thread per group: its G values stay in registers while
// all candidates are scored, so W is read once.  Every step up to w_hat uses
// the IEEE fp32 operations the fp32 definition names (correctly rounded
// division, rint, no contraction), so the parameters of a candidate are the
// same bits on any IEEE fp32 implementation; the error terms are summed in
// fp32 in ascending k.  The kernel is bound by arithmetic (a division and, for
// a general norm, a power per value and candidate), not by memory.
//
// Patience: the first pass records, per group, a bit mask of the candidates
// that strictly improved its running best (steps <= 32), and ORs the masks of
// all groups into one word.  The second pass finds the stop from that word,
// takes each group's last improvement before the stop -- its best evaluated
// candidate, since improvements are strict -- and writes its parameters.
#include <cuda_runtime.h>

#include "wq_internal.h"

namespace wq {
namespace {

constexpr float EPS32 = 1.1920928955078125e-07f;  // 2^-23

struct MseParams {
    const float* w;
    int rows, cols, G, gpr;  // gpr = cols / G
    long long ngroups;
    int steps, grid;
    float norm;
    int patience;            // 0: every candidate is evaluated
    int symmetric;
    float qmin, qmax, half;  // code range; half = (qmax - qmin) / 2
    float* scale;
    float* zero;
    int32_t* step;           // the winner (also the improvement mask between the passes)
    float* err;
    uint32_t* any_mask;      // OR of every group's improvement mask (patience only)
};

__device__ __forceinline__ float cand(int i, int grid) {
    return (float)(1.0 - (double)i / (double)grid);  // one rounding of the exact 1 - i / grid
}

__device__ __forceinline__ void qparams(const MseParams& p, float lo, float hi, float& s, float& z) {
    if (p.symmetric) {
        const float a = fmaxf(fabsf(lo), fabsf(hi));
        s = __fdiv_rn(a, p.half);
        if (s == 0.0f) s = EPS32;
        z = 0.0f;
    } else {
        lo = fminf(lo, 0.0f);
        hi = fmaxf(hi, 0.0f);
        s = __fdiv_rn(__fsub_rn(hi, lo), __fsub_rn(p.qmax, p.qmin));
        if (s == 0.0f) s = EPS32;
        z = __fsub_rn(p.qmin, rintf(__fdiv_rn(lo, s)));
        z = fminf(fmaxf(z, p.qmin), p.qmax);
    }
}

__device__ __forceinline__ float term(float d, float norm) {
    if (norm == 2.0f) return __fmul_rn(d, d);
    if (norm == 1.0f) return d;
    return d == 0.0f ? 0.0f : powf(d, norm);
}

__device__ __forceinline__ float value_err(const MseParams& p, float w, float s, float z) {
    const float t = __fadd_rn(__fdiv_rn(w, s), z);
    const float q = fminf(fmaxf(rintf(t), p.qmin), p.qmax);
    const float w_hat = __fmul_rn(__fsub_rn(q, z), s);
    return term(fabsf(__fsub_rn(w_hat, w)), p.norm);
}

// A group's values: GC > 0 holds them in registers (GC == G); GC == 0 reads
// them from memory at every candidate (any G; they stay in the L1 cache).
template <int GC>
struct Group {
    float v[GC > 0 ? GC : 1];
    const float* src;
    float mn, mx;

    __device__ __forceinline__ bool load(const MseParams& p, long long gi) {
        if (gi >= p.ngroups) return false;
        const long long row = gi / p.gpr;
        src = p.w + row * (long long)p.cols + (gi - row * p.gpr) * (long long)p.G;
        mn = INFINITY;
        mx = -INFINITY;
        if constexpr (GC > 0) {
#pragma unroll
            for (int k = 0; k < GC; ++k) {
                v[k] = __ldg(src + k);
                mn = fminf(mn, v[k]);
                mx = fmaxf(mx, v[k]);
            }
        } else {
            for (int k = 0; k < p.G; ++k) {
                const float x = __ldg(src + k);
                mn = fminf(mn, x);
                mx = fmaxf(mx, x);
            }
        }
        return true;
    }

    // sum |w_hat - w|^norm of candidate (s, z), in fp32, ascending k
    __device__ __forceinline__ float err(const MseParams& p, float s, float z) const {
        float e = 0.0f;
        if constexpr (GC > 0) {
#pragma unroll
            for (int k = 0; k < GC; ++k) e = __fadd_rn(e, value_err(p, v[k], s, z));
        } else {
            for (int k = 0; k < p.G; ++k) e = __fadd_rn(e, value_err(p, __ldg(src + k), s, z));
        }
        return e;
    }
};

template <int GC>
__global__ void __launch_bounds__(256) mse_search_kernel(const MseParams p) {
    const long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    Group<GC> grp;
    const bool on = grp.load(p, gi);
    uint32_t mask = 0;
    float best = INFINITY, bs = 0.0f, bz = 0.0f;
    int bi = 0;
    if (on) {
        for (int i = 0; i < p.steps; ++i) {
            const float pi = cand(i, p.grid);
            float s, z;
            qparams(p, __fmul_rn(grp.mn, pi), __fmul_rn(grp.mx, pi), s, z);
            const float e = grp.err(p, s, z);
            if (e < best) {
                best = e;
                bi = i;
                bs = s;
                bz = z;
                mask |= 1u << i;
            }
        }
        if (!p.patience) {
            p.step[gi] = bi;
            p.err[gi] = best;
            p.scale[gi] = bs;
            p.zero[gi] = bz;
        } else {
            p.step[gi] = (int32_t)mask;
        }
    }
    if (p.patience) {  // one OR per warp into the word every group's mask meets
        const uint32_t wm = __reduce_or_sync(0xffffffffu, mask);
        if ((threadIdx.x & 31) == 0 && wm) atomicOr(p.any_mask, wm);
    }
}

// Second pass of the patience search: the stop, then each group's winner.
template <int GC>
__global__ void __launch_bounds__(256) mse_finish_kernel(const MseParams p) {
    const long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    Group<GC> grp;
    if (!grp.load(p, gi)) return;
    // candidates evaluated: the search stops once `patience` candidates in a
    // row improved no group anywhere
    const uint32_t any = *p.any_mask;
    int evaluated = p.steps, stale = 0;
    for (int i = 0; i < p.steps; ++i) {
        stale = ((any >> i) & 1u) ? 0 : stale + 1;
        if (stale >= p.patience) {
            evaluated = i + 1;
            break;
        }
    }
    const uint32_t mine = (uint32_t)p.step[gi] & (evaluated >= 32 ? 0xffffffffu : ((1u << evaluated) - 1u));
    const int bi = mine ? 31 - __clz(mine) : 0;  // the last strict improvement
    const float pi = cand(bi, p.grid);
    float s, z;
    qparams(p, __fmul_rn(grp.mn, pi), __fmul_rn(grp.mx, pi), s, z);
    p.step[gi] = bi;
    p.scale[gi] = s;
    p.zero[gi] = z;
    p.err[gi] = mine ? grp.err(p, s, z) : INFINITY;
}

template <int GC>
wq_status run_mse(const MseParams& p, cudaStream_t stream) {
    const int threads = 256;
    const long long blocks = (p.ngroups + threads - 1) / threads;
    if (blocks > 0x7fffffffll) return WQ_ERR_INVALID_ARG;
    if (p.patience && cudaMemsetAsync(p.any_mask, 0, sizeof(uint32_t), stream) != cudaSuccess) return WQ_ERR_CUDA;
    mse_search_kernel<GC><<<(unsigned)blocks, threads, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return WQ_ERR_CUDA;
    if (p.patience) {
        mse_finish_kernel<GC><<<(unsigned)blocks, threads, 0, stream>>>(p);
        if (cudaGetLastError() != cudaSuccess) return WQ_ERR_CUDA;
    }
    return WQ_OK;
}

}  // namespace

wq_status launch_mse_search(const float* w, int rows, int cols, int group_size, int bits, int symmetric,
                            int steps, int grid, float norm, int patience, float* scale, float* zero,
                            int32_t* step, float* err, uint32_t* any_mask, cudaStream_t stream) {
    MseParams p{};
    p.w = w;
    p.rows = rows;
    p.cols = cols;
    p.G = group_size;
    p.gpr = cols / group_size;
    p.ngroups = (long long)rows * p.gpr;
    p.steps = steps;
    p.grid = grid;
    p.norm = norm;
    p.patience = patience;
    p.symmetric = symmetric;
    if (symmetric) {
        p.qmin = -(float)(1 << (bits - 1));
        p.qmax = (float)((1 << (bits - 1)) - 1);
    } else {
        p.qmin = 0.0f;
        p.qmax = (float)((1 << bits) - 1);
    }
    p.half = (p.qmax - p.qmin) / 2.0f;  // exact: (2^b - 1) / 2
    p.scale = scale;
    p.zero = zero;
    p.step = step;
    p.err = err;
    p.any_mask = any_mask;
    switch (group_size) {
        case 8: return run_mse<8>(p, stream);
        case 16: return run_mse<16>(p, stream);
        case 32: return run_mse<32>(p, stream);
        default: return run_mse<0>(p, stream);  // any other G, values read from memory
    }
}

}  // namespace wq
