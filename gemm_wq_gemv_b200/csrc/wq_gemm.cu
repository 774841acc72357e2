// wq_gemm.cu -- batched product y (M x N) = x (M x K) @ dequant(W_q) on the tcgen05 tensor cores.
//
// What is computed: "GPTQModel-Compatible Triton Kernel" README
// (`gptqmodel_quantized_matmul`: output = x @ dequantize(qweight)) and the batched
// branch of dashq_kernel.py `forward` (x @ dequantize_weight()), with fp32
// accumulation and one fp16 rounding at the end.
//
// How (sm_100a), per CTA = one tile of 128 weight columns x TN tokens x a K range:
//  * The product is computed transposed (D = W^T x^T), so the 128 weight columns
//    fill the MMA's M = 128 and the tokens are its N (16..256).  D lives in
//    tensor memory: lane = weight column, column = token, fp32.
//  * Warp 0 (one lane) streams each 64-deep k block with TMA into a ring of
//    shared-memory stages: the x tile (TN x 64 fp16, 128-byte swizzle, which is
//    the MMA's K-major layout), the packed word tile (64 / eps rows x 128 columns),
//    the 3-bit lo-plane tile and the s, z rows of the block's group(s).
//  * Warps 2-5 (one thread per weight column) turn that column's words into 64
//    fp16 values (q - z) * s -- code pairs become exact q - round(z) with one
//    LOP3 + one FMA, are put in k order with PRMT and scaled with one more FMA --
//    and store them into the A tile in the same swizzled K-major layout.
//  * Warp 1 (one lane) issues four tcgen05.mma (K = 16 each) per stage and
//    frees the stage with tcgen05.commit when they have read it.
//  * K is split over the CTAs of a thread-block cluster; after the main loop the
//    fp32 tiles are summed through distributed shared memory (one launch, no
//    workspace), converted to fp16 and stored by warps 2-5.
// Every wait on an mbarrier is bounded; on time-out the kernel records
// WQ_ERR_TIMEOUT in a device status word, skips its remaining work, still
// frees its tensor memory and returns.

#include <algorithm>

#include "wq_dequant.cuh"
#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {

// Device status of the GEMM: 0, or 1 once a bounded wait ran out.
__device__ unsigned int g_gemm_status = 0;

namespace {

constexpr int BMW = 128;    // weight columns per tile (MMA M)
constexpr int BK = 64;      // k per stage
constexpr int NWARPS = 6;   // 0 TMA, 1 MMA + TMEM, 2-5 dequant + epilogue
constexpr uint64_t WAIT_NS = 2000000000ull;

struct GemmParams {
    uint16_t* y;
    int M, K, N, G;
    int TN;              // tokens per tile (MMA N)
    int CS;              // CTAs per cluster along K
    int kb_cta;          // k blocks per CTA
    int GPB;             // s/z rows per stage
    int stages;
    uint32_t stage_bytes, off_a, off_w, off_lo, off_s, off_z;
    uint32_t tx_bytes;
    uint32_t tmem_cols;
    uint32_t bar_off;    // offset of the barrier block from the aligned base
    int njl;             // token chunks (32) owned per CTA in the split-K reduction
};

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

template <int BITS>
__global__ void __launch_bounds__(NWARPS * 32, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_lo, const __grid_constant__ CUtensorMap tm_s,
            const __grid_constant__ CUtensorMap tm_z, const GemmParams p) {
    using F = Fmt<BITS>;
    constexpr int EPS = F::EPS;          // codes per word of the main plane
    constexpr int NC = F::NC;
    constexpr int RW = BK / EPS;         // word rows per stage

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint64_t* full_tma = reinterpret_cast<uint64_t*>(base + p.bar_off);
    uint64_t* full_a = full_tma + p.stages;
    uint64_t* empty = full_a + p.stages;
    uint64_t* accum = empty + p.stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BMW;
    const int m0 = blockIdx.y * p.TN;
    const int rank = (int)blockIdx.z;  // cluster spans grid z
    const int kb0 = rank * p.kb_cta;   // first k block of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&full_a[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    auto fail = [&]() {
        *abort_flag = 1;
        atomicExch(&g_gemm_status, 1u);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            prefetch_tmap(&tm_s);
            prefetch_tmap(&tm_z);
            if constexpr (BITS == 3) prefetch_tmap(&tm_lo);
            const uint64_t pol_w = policy_evict_first();
            grid_dependency_wait();
            for (int kb = 0; kb < p.kb_cta; ++kb) {
                const int s = kb % p.stages, r = kb / p.stages;
                if (r > 0 && !mbar_wait_bounded(&empty[s], (r - 1) & 1, WAIT_NS)) { fail(); break; }
                if (*abort_flag) break;
                uint8_t* st = base + (size_t)s * p.stage_bytes;
                const int kg = (kb0 + kb) * BK;
                mbar_arrive_expect_tx(&full_tma[s], p.tx_bytes);
                tma_load_2d(st, &tm_x, &full_tma[s], kg, m0);
                tma_load_2d_hint(st + p.off_w, &tm_w, &full_tma[s], n0, kg / EPS, pol_w);
                if constexpr (BITS == 3) tma_load_2d_hint(st + p.off_lo, &tm_lo, &full_tma[s], n0, kg / 32, pol_w);
                const int grow = kg / p.G;
                tma_load_2d(st + p.off_s, &tm_s, &full_tma[s], n0, grow);
                tma_load_2d(st + p.off_z, &tm_z, &full_tma[s], n0, grow);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | ((uint32_t)(p.TN >> 3) << 17) | (8u << 24);
            for (int kb = 0; kb < p.kb_cta; ++kb) {
                const int s = kb % p.stages, r = kb / p.stages;
                if (!mbar_wait_bounded(&full_tma[s], r & 1, WAIT_NS)) { fail(); break; }
                if (!mbar_wait_bounded(&full_a[s], r & 1, WAIT_NS)) { fail(); break; }
                if (*abort_flag) break;
                tc_fence_after();
                const uint32_t st = smem_u32(base + (size_t)s * p.stage_bytes);
                const uint64_t bdesc = sw128_desc(st);
                const uint64_t adesc = sw128_desc(st + p.off_a);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma_f16(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(accum);
        }
    } else {
        // ------------------------------------------- dequantisation (one column each)
        const int qd = warp & 3;                 // TMEM lane quadrant this warp may read
        const int nl = 32 * qd + lane;           // weight column within the tile
        const uint32_t lo_sel0 = 0x7170u, lo_sel1 = 0x7372u;
        for (int kb = 0; kb < p.kb_cta; ++kb) {
            const int s = kb % p.stages, r = kb / p.stages;
            if (!mbar_wait_bounded(&full_tma[s], r & 1, WAIT_NS)) { fail(); break; }
            if (*abort_flag) break;
            uint8_t* st = base + (size_t)s * p.stage_bytes;
            const uint32_t* wt = reinterpret_cast<const uint32_t*>(st + p.off_w);
            const uint32_t* lt = reinterpret_cast<const uint32_t*>(st + p.off_lo);
            const uint16_t* sr = reinterpret_cast<const uint16_t*>(st + p.off_s);
            const uint16_t* zr_ = reinterpret_cast<const uint16_t*>(st + p.off_z);
            uint8_t* arow = st + p.off_a + nl * 128;
            const int sw = nl & 7;

            int cur_g = -1;
            uint32_t c[NC];
            uint32_t s2 = 0, zs2 = 0;
#pragma unroll
            for (int rw = 0; rw < RW; ++rw) {
                // group row of this word within the stage's s/z rows
                const int gi = (p.GPB == 1) ? 0 : (rw * EPS) / p.G;
                if (gi != cur_g) {
                    cur_g = gi;
                    const float sv = __half2float(__ushort_as_half(sr[gi * BMW + nl]));
                    const float zv = __half2float(__ushort_as_half(zr_[gi * BMW + nl]));
                    const float zi = fminf(fmaxf(rintf(zv), -256.0f), 256.0f);
#pragma unroll
                    for (int ci = 0; ci < NC; ++ci) c[ci] = dup_half(-(bias_magnitude<BITS>(ci) + zi));
                    s2 = dup_half(sv);
                    zs2 = dup_half(-(zv - zi) * sv);
                }
                uint32_t w = wt[rw * BMW + nl], wh = 0, ls = 0;
                uint32_t lw = 0;
                if constexpr (BITS == 3) lw = lt[(rw >> 1) * BMW + nl];
                prep_word<BITS>(w, wh, ls, lw, (rw & 1) ? lo_sel1 : lo_sel0);
                uint32_t P[EPS / 2];
#pragma unroll
                for (int j = 0; j < EPS / 2; ++j) P[j] = pair_q<BITS>(w, wh, ls, c, j);
                uint32_t Nh[EPS / 2];
#pragma unroll
                for (int i = 0; i < EPS / 4; ++i) {
                    Nh[i] = prmt(P[2 * i], P[2 * i + 1], 0x5410u);
                    Nh[i + EPS / 4] = prmt(P[2 * i], P[2 * i + 1], 0x7632u);
                }
#pragma unroll
                for (int i = 0; i < EPS / 2; ++i) Nh[i] = hfma2_u32(Nh[i], s2, zs2);
                // k = rw * EPS .. + EPS - 1 -> 16-byte chunks of 8 halves, swizzled
                if constexpr (EPS >= 8) {
#pragma unroll
                    for (int v = 0; v < EPS / 8; ++v) {
                        const int chunk = rw * (EPS / 8) + v;
                        *reinterpret_cast<uint4*>(arow + ((chunk ^ sw) << 4)) =
                            make_uint4(Nh[4 * v], Nh[4 * v + 1], Nh[4 * v + 2], Nh[4 * v + 3]);
                    }
                } else {
                    const int chunk = rw >> 1;
                    *reinterpret_cast<uint2*>(arow + ((chunk ^ sw) << 4) + 8 * (rw & 1)) = make_uint2(Nh[0], Nh[1]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[s]);
        }
    }

    __syncwarp();  // warps 0 and 1: lanes 1-31 wait for lane 0 before the aligned barriers below

    // ------------------------------------------------------------------ epilogue
    grid_launch_dependents();
    const bool split = p.CS > 1;
    const int nchunks = p.TN / 32;
    uint8_t* recv = base;  // reuses the stage ring once every CTA of the cluster is done
    if (warp >= 2) {
        if (!*abort_flag) {
            if (!mbar_wait_bounded(accum, 0, WAIT_NS)) fail();
        }
        tc_fence_after();
    }
    if (split) cluster_sync();  // every CTA of the cluster has finished its main loop

    const int qd = warp & 3;
    const int nl = 32 * qd + lane;
    const int ncol = n0 + nl;
    if (warp >= 2 && !*abort_flag) {
        if (split) {
            for (int j = 0; j < nchunks; ++j) {
                const int owner = j % p.CS;
                if (owner == rank) continue;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(32 * qd) << 16) + 32 * j, v);
                tmem_ld_wait();
                const int jl = j / p.CS;
                const uint32_t dst = smem_u32(recv) + (uint32_t)((((rank * p.njl + jl) * 32) * BMW + nl) * 4);
                const uint32_t rdst = map_shared_rank(dst, owner);
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) st_shared_cluster_f32(rdst + cc * BMW * 4, __uint_as_float(v[cc]));
            }
        }
    }
    if (split) cluster_sync();  // all partial tiles have landed in their owners
    if (warp >= 2 && !*abort_flag) {
        for (int j = 0; j < nchunks; ++j) {
            if (split && (j % p.CS) != rank) continue;
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(32 * qd) << 16) + 32 * j, v);
            tmem_ld_wait();
            float acc[32];
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) acc[cc] = __uint_as_float(v[cc]);
            if (split) {
                const int jl = j / p.CS;
                for (int src = 0; src < p.CS; ++src) {
                    if (src == rank) continue;
                    const float* rb = reinterpret_cast<const float*>(recv) + ((src * p.njl + jl) * 32) * BMW + nl;
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) acc[cc] += rb[cc * BMW];
                }
            }
            if (ncol < p.N) {
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) {
                    const int m = m0 + 32 * j + cc;
                    if (m < p.M) p.y[(size_t)m * p.N + ncol] = __half_as_ushort(__float2half_rn(acc[cc]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, p.tmem_cols);
    }
}

// ------------------------------------------------------------------------ host
template <int BITS>
wq_status run(const Problem& pb, cudaStream_t stream) {
    constexpr int EPS = Fmt<BITS>::EPS;
    constexpr int RW = BK / EPS;
    constexpr int RL = (BITS == 3) ? BK / 32 : 0;
    auto kern = gemm_kernel<BITS>;

    GemmParams p{};
    p.y = pb.y;
    p.M = pb.M; p.K = pb.K; p.N = pb.N; p.G = pb.G;
    // s/z rows per 64-deep block: 1 if a group covers whole blocks, else 64 / G
    if (pb.G % BK == 0) p.GPB = 1;
    else if (BK % pb.G == 0) p.GPB = BK / pb.G;
    else return WQ_ERR_UNSUPPORTED;

    // token tile: balanced tiles of at most 256 tokens, multiple of 16
    const int mt = (pb.M + 255) / 256;
    int TN = (pb.M + mt - 1) / mt;
    TN = std::max(32, (TN + 31) / 32 * 32);  // the epilogue reads tensor memory 32 columns at a time
    p.TN = TN;
    const int ntiles = (pb.N + BMW - 1) / BMW;
    const int tiles = ntiles * mt;
    const int KB = pb.K / BK;
    const int sms = sm_count();
    int CS = 1;
    for (int c = 8; c >= 2; c >>= 1) {
        if (KB % c == 0 && KB / c >= 2 && tiles * c <= sms) { CS = c; break; }
    }
    p.CS = CS;
    p.kb_cta = KB / CS;
    p.tmem_cols = 32;
    while ((int)p.tmem_cols < TN) p.tmem_cols <<= 1;

    // stage layout: x tile | A tile | words | lo words | s rows | z rows (1024-aligned stage)
    const uint32_t xb = (uint32_t)TN * 128u;
    p.off_a = (xb + 1023u) & ~1023u;
    p.off_w = p.off_a + BMW * 128u;
    p.off_lo = p.off_w + RW * BMW * 4u;
    p.off_s = p.off_lo + RL * BMW * 4u;
    p.off_z = p.off_s + p.GPB * BMW * 2u;
    const uint32_t end = p.off_z + p.GPB * BMW * 2u;
    p.stage_bytes = (end + 1023u) & ~1023u;
    p.tx_bytes = xb + RW * BMW * 4u + RL * BMW * 4u + 2u * p.GPB * BMW * 2u;
    const size_t limit = 227 * 1024;
    const size_t bar_bytes = 256;
    int stages = (int)((limit - 1024 - bar_bytes) / p.stage_bytes);
    stages = std::min(stages, 6);
    stages = std::min(stages, std::max(2, p.kb_cta));
    if (stages < 2) return WQ_ERR_UNSUPPORTED;
    p.stages = stages;
    p.njl = (TN / 32 + CS - 1) / CS;
    const size_t recv_bytes = (size_t)CS * p.njl * 32 * BMW * 4;
    size_t ring = (size_t)stages * p.stage_bytes;
    if (CS > 1 && recv_bytes > ring) ring = (recv_bytes + 1023) & ~(size_t)1023;
    p.bar_off = (uint32_t)ring;
    // At least 80 KB so that no more than two CTAs share an SM: two tensor-memory
    // allocations of at most 256 columns always fit in the SM's 512 columns, so
    // tcgen05.alloc never waits on a CTA of another cluster.
    const size_t smem = std::max<size_t>(1024 + ring + bar_bytes, 80 * 1024);
    if (smem > limit) return WQ_ERR_UNSUPPORTED;

    CUtensorMap mx, mw, ml, ms, mz;
    const int groups = (pb.K + pb.G - 1) / pb.G;
    bool ok = make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, pb.x, pb.K, pb.M, (uint64_t)pb.K * 2, BK, TN,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_q, pb.N, pb.K / EPS, (uint64_t)pb.N * 4, BMW, RW,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (BITS == 3)
        ok = ok && make_map(&ml, CU_TENSOR_MAP_DATA_TYPE_UINT32, pb.w_lo, pb.N, pb.K / 32, (uint64_t)pb.N * 4, BMW,
                            RL, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        ml = mw;
    ok = ok && make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.scales, pb.N, groups, (uint64_t)pb.N * 2, BMW, p.GPB,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_map(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, pb.zeros, pb.N, groups, (uint64_t)pb.N * 2, BMW, p.GPB,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return WQ_ERR_CUDA;

    static unsigned long long attr_done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (dev < 64 && !(attr_done & (1ull << dev))) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)limit) != cudaSuccess)
            return WQ_ERR_CUDA;
        attr_done |= 1ull << dev;
    }

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ntiles, mt, CS);
    cfg.blockDim = dim3(NWARPS * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = 1;
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = CS;
    ++na;
    if (pb.flags & WQ_FLAG_PDL) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, mx, mw, ml, ms, mz, p));
}

}  // namespace

wq_status launch_gemm(const Problem& p, cudaStream_t s) {
    switch (p.bits) {
        case 1: return run<1>(p, s);
        case 2: return run<2>(p, s);
        case 3: return run<3>(p, s);
        case 4: return run<4>(p, s);
        case 8: return run<8>(p, s);
        default: return WQ_ERR_UNSUPPORTED;
    }
}

wq_status gemm_device_status(int reset) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return v ? WQ_ERR_TIMEOUT : WQ_OK;
}

}  // namespace wq
