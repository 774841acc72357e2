// wq_gemm.cu -- batched product y (M x N) = x (M x K) @ dequant(W_q) on the tcgen05 tensor cores.
//
// What is computed: "GPTQModel-Compatible Triton Kernel" README
// (`gptqmodel_quantized_matmul`: output = x @ dequantize(qweight)) and the batched
// branch of dashq_kernel.py `forward` (x @ dequantize_weight()), with fp32
// accumulation and one rounding at the end.  x, s, z, the bias and y are all
// fp16 or all bf16 (the module's `out_dtype`; the MMA takes both operands in it).
//
// How (sm_100a), per CTA = one tile of 128 weight columns x TN tokens x a K range:
//  * The product is computed transposed (D = W^T x^T), so the 128 weight columns
//    fill the MMA's M = 128 and the tokens are its N (16..256).  D lives in
//    tensor memory: lane = weight column, column = token, fp32.
//  * Warp 0 (one lane) streams each 64-deep k block with TMA into a ring of
//    shared-memory stages: the x tile (TN x 64 16-bit values, 128-byte swizzle, which is
//    the MMA's K-major layout), the packed word tile (64 / eps rows x 128 columns),
//    the 3-bit lo-plane tile and the s, z rows of the block's group(s).
//  * Warps 2-9 (two threads per weight column, each taking half of the stage's
//    word rows) turn that column's words into 32 values (q - z) * s each --
//    code pairs become exact q - round(z) with one LOP3 + one FMA (bf16: see
//    wq_dequant.cuh), are put in k order with PRMT and scaled with one more
//    fp16x2 / bf16x2 FMA -- and store them with
//    tcgen05.st into tensor memory, where the MMA reads its A operand.
//  * Warp 1 (one lane) issues four tcgen05.mma (K = 16 each) per stage and
//    frees the stage with tcgen05.commit when they have read it.
//  * K may be split over the CTAs of a thread-block cluster; after the main loop
//    each CTA writes the 32-token slices of its fp32 tile that another rank owns
//    into a caller-provided global workspace (it stays in L2), one cluster
//    barrier (release / acquire) orders those writes, and each owner adds its
//    peers' slices to its own before converting to fp16 and storing y.
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
constexpr int NWARPS = 10;  // 0 TMA, 1 MMA + TMEM, 2-9 dequant + epilogue (two per TMEM lane quadrant)
constexpr int NDQ = NWARPS - 2;
constexpr size_t CHUNK_BYTES = 128 * 32 * 4;  // one 32-token fp32 slice of the tile
constexpr uint64_t WAIT_NS = 2000000000ull;

struct GemmParams {
    uint16_t* y;
    const uint16_t* bias;  // (N,) fp16 / bf16 or null
    int M, K, N, G;
    int TN;              // tokens per tile (MMA N)
    int CS;              // CTAs per cluster along K
    int kb_cta;          // k blocks per CTA
    int GPB;             // s/z rows per stage
    int gmode;           // 0: G a multiple of 64; 1: G a power of two below 64; 2: any other G
    int g_shift;         // log2(G) when G < 64
    int stages;
    uint32_t stage_bytes, off_w, off_lo, off_s, off_z;
    uint32_t a_col;      // first tensor-memory column of the A stages (32 columns per stage)
    uint32_t tx_bytes;
    uint32_t tmem_cols;
    uint32_t bar_off;    // offset of the barrier block from the aligned base
    uint4* ws;           // split-K slices: [tile][rank][32-token chunk][16-byte piece][128 columns]
    size_t ws_u4;        // 16-byte units of the caller's workspace (checked build)
    int late_wait;       // wait for the previous kernel only before writing the workspace / y
};

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// GW: every group covers whole 64-deep k blocks (G a multiple of 64, or G = K),
// the common case, compiled without the per-row group logic of the others.
template <int BITS, bool BF, bool GW>
__global__ void __launch_bounds__(NWARPS * 32, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_lo, const __grid_constant__ CUtensorMap tm_s,
            const __grid_constant__ CUtensorMap tm_z, const GemmParams p) {
    using F = Fmt<BITS>;
    using T16 = Dt<BF>;
    constexpr int EPS = F::EPS;          // codes per word of the main plane
    constexpr int NC = ncons<BITS, BF>();
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
            mbar_init(&full_a[s], NDQ / 2);  // the four warps of the half that dequantises stage s
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
        atomicOr(&g_gemm_status, 1u);
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
            if (!p.late_wait) grid_dependency_wait();
            // stage slot, its use parity and the s/z row, advanced without divisions
            int s = 0;
            uint32_t ph = 0;
            int kg = kb0 * BK;
            int grow = kg / p.G, gnext = (grow + 1) * p.G;
            for (int kb = 0; kb < p.kb_cta; ++kb) {
                if (kb >= p.stages && !mbar_wait_bounded(&empty[s], ph ^ 1u, WAIT_NS)) { fail(); break; }
                if (*abort_flag) break;
                uint8_t* st = base + (size_t)s * p.stage_bytes;
                mbar_arrive_expect_tx(&full_tma[s], p.tx_bytes);
                tma_load_2d(st, &tm_x, &full_tma[s], kg, m0);
                tma_load_2d_hint(st + p.off_w, &tm_w, &full_tma[s], n0, kg / EPS, pol_w);
                if constexpr (BITS == 3) tma_load_2d_hint(st + p.off_lo, &tm_lo, &full_tma[s], n0, kg / 32, pol_w);
                tma_load_2d(st + p.off_s, &tm_s, &full_tma[s], n0, grow);
                tma_load_2d(st + p.off_z, &tm_z, &full_tma[s], n0, grow);
                kg += BK;
                if (GW) {                   // a group spans whole k blocks: next row once kg reaches it
                    if (kg >= gnext) { ++grow; gnext += p.G; }
                } else if (p.gmode == 1) {  // 64 / G rows per k block
                    grow += p.GPB;
                } else {                    // the group of the block's first k, then GPB rows
                    grow = kg / p.G;
                }
                if (++s == p.stages) { s = 0; ph ^= 1u; }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // D fp32 (bit 4), A and B both fp16 (format 0) or both bf16 (format 1,
            // bits 7 and 10), N = TN (bits 17-22, N / 8), M = 128 (bits 24-28, M / 16)
            constexpr uint32_t ab_fmt = BF ? ((1u << 7) | (1u << 10)) : 0u;
            const uint32_t idesc = (1u << 4) | ab_fmt | ((uint32_t)(p.TN >> 3) << 17) | (8u << 24);
            int s = 0;
            uint32_t ph = 0;
            const uint64_t bdesc0 = sw128_desc(smem_u32(base));
            const uint64_t bstep = (uint64_t)(p.stage_bytes >> 4);  // descriptor address units
            for (int kb = 0; kb < p.kb_cta; ++kb) {
                // the dequantising warps arrive on full_a only after they saw full_tma complete
                if (!mbar_wait_bounded(&full_a[s], ph, WAIT_NS)) { fail(); break; }
                if (!mbar_wait_bounded(&full_tma[s], ph, WAIT_NS)) { fail(); break; }
                tc_fence_after();
                const uint64_t bdesc = bdesc0 + bstep * (uint64_t)s;
                const uint32_t a_tm = tmem_d + p.a_col + 32u * s;  // lane 0, this stage's A columns
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma_f16_ts(tmem_d, a_tm + 8 * kk, bdesc + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
                if (++s == p.stages) { s = 0; ph ^= 1u; }
            }
            tc_commit(accum);
        }
    } else {
        // ----------------------- dequantisation: a column per thread; the two warps of a
        // TMEM lane quadrant take alternate stages, all of a stage's word rows each
        const int qd = warp & 3;                 // TMEM lane quadrant this warp may read
        const int hf = (warp - 2) >> 2;          // this warp takes the k blocks with kb % 2 == hf
        const int nl = 32 * qd + lane;           // weight column within the tile
        const uint32_t lo_sel0 = 0x7170u, lo_sel1 = 0x7372u;

        // (q - z) * s for word row rw of this column, in k order, into out[0 .. EPS/2)
        auto word = [&](const uint8_t* st, int rw, const uint32_t (&c)[NC], uint32_t s2, uint32_t zs2,
                        uint32_t* out) {
            const uint32_t* wt = reinterpret_cast<const uint32_t*>(st + p.off_w);
            uint32_t lw = 0;
            if constexpr (BITS == 3) lw = reinterpret_cast<const uint32_t*>(st + p.off_lo)[(rw >> 1) * BMW + nl];
            Word<BITS, BF> wd;
            wd.prep(wt[rw * BMW + nl], lw, (rw & 1) ? lo_sel1 : lo_sel0);
            uint32_t P[EPS / 2];
#pragma unroll
            for (int j = 0; j < EPS / 2; ++j) P[j] = wd.pair(c, j);
#pragma unroll
            for (int i = 0; i < EPS / 4; ++i) {
                out[i] = fma2_u32<BF>(prmt(P[2 * i], P[2 * i + 1], 0x5410u), s2, zs2);
                out[i + EPS / 4] = fma2_u32<BF>(prmt(P[2 * i], P[2 * i + 1], 0x7632u), s2, zs2);
            }
        };
        // per-(group, column) constants from the stage's s, z rows
        auto consts = [&](const uint8_t* st, int gi, uint32_t (&c)[NC], uint32_t& s2, uint32_t& zs2) {
            const float sv = T16::load(reinterpret_cast<const uint16_t*>(st + p.off_s)[gi * BMW + nl]);
            const float zv = T16::load(reinterpret_cast<const uint16_t*>(st + p.off_z)[gi * BMW + nl]);
            const float zi = zero_int<BITS, BF>(zv);
#pragma unroll
            for (int ci = 0; ci < NC; ++ci) c[ci] = pair_const<BITS, BF>(ci, zi);
            s2 = dup_t<BF>(sv);
            zs2 = dup_t<BF>(-(zv - zi) * sv);
        };

        int s = 0;
        uint32_t ph = 0;
        for (int kb = 0; kb < p.kb_cta; ++kb) {
            if ((kb & 1) == hf) {
                if (!mbar_wait_bounded(&full_tma[s], ph, WAIT_NS)) { fail(); break; }
                if (*abort_flag) break;
                const uint8_t* st = base + (size_t)s * p.stage_bytes;
                uint32_t c[NC], s2, zs2;
                uint32_t a32[32];  // this thread's 64 k values (32 pairs) of the stage's A row
                if constexpr (GW) {  // one group covers the whole k block
                    consts(st, 0, c, s2, zs2);
#pragma unroll
                    for (int rw = 0; rw < RW; ++rw) word(st, rw, c, s2, zs2, a32 + rw * (EPS / 2));
                } else if (p.gmode == 2) {
                    // Group boundaries anywhere in the block (G a multiple of the
                    // codes per word, so never inside a word row): row gi of the
                    // stage's s, z tile is group (block start) / G + gi.
                    const int kbase = (kb0 + kb) * BK;
                    int gi = 0;
                    int next = (kbase / p.G + 1) * p.G - kbase;  // block offset of the next group start
                    consts(st, 0, c, s2, zs2);
#pragma unroll
                    for (int rw = 0; rw < RW; ++rw) {
                        if (rw * EPS >= next) {
                            ++gi;
                            next += p.G;
                            consts(st, gi, c, s2, zs2);
                        }
                        word(st, rw, c, s2, zs2, a32 + rw * (EPS / 2));
                    }
                } else {
                    int cur = -1;
#pragma unroll
                    for (int rw = 0; rw < RW; ++rw) {
                        const int gi = (rw * EPS) >> p.g_shift;  // G divides 64: a power of two
                        if (gi != cur) {
                            cur = gi;
                            consts(st, gi, c, s2, zs2);
                        }
                        word(st, rw, c, s2, zs2, a32 + rw * (EPS / 2));
                    }
                }
                // A row of weight column nl = tensor-memory lane nl; k pairs along the columns
                tmem_st_32x32b_x32(tmem_d + ((uint32_t)(32 * qd) << 16) + p.a_col + 32u * s, a32);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_a[s]);
            }
            if (++s == p.stages) { s = 0; ph ^= 1u; }
        }
    }

    __syncwarp();  // warps 0 and 1: lanes 1-31 wait for lane 0 before the aligned barriers below

    // ------------------------------------------------------------------ epilogue
    grid_launch_dependents();
    const bool split = p.CS > 1;
    const int nchunks = p.TN / 32;
    if (warp >= 2) {
        if (!*abort_flag) {
            if (!mbar_wait_bounded(accum, 0, WAIT_NS)) fail();
        }
        tc_fence_after();
    }

    const int qd = warp & 3;
    const int hf = (warp - 2) >> 2;   // epilogue warps of a quadrant take alternate 32-token chunks
    const int nl = 32 * qd + lane;
    const int ncol = n0 + nl;
    const uint32_t tm_row = tmem_d + ((uint32_t)(32 * qd) << 16);
    if (p.late_wait) grid_dependency_wait();  // the workspace and y may still be in use before this
    // Split-K exchange.  Chunk j (32 tokens) of the tile is owned by rank j % CS.
    // A slice in the workspace is 8 pieces x 128 columns x 16 bytes, so the 32
    // threads of a warp write (and later read) 512 contiguous bytes per piece.
    constexpr size_t CHUNK_U4 = CHUNK_BYTES / 16;
    const size_t tile_slot = (size_t)(blockIdx.y * gridDim.x + blockIdx.x) * (size_t)p.CS;
    if (split && warp >= 2 && !*abort_flag) {
        uint4* mine = p.ws + (tile_slot + rank) * nchunks * CHUNK_U4;
        // this CTA's non-owned chunks, alternately to the two warps of the quadrant
        for (int j = 0, sidx = 0; j < nchunks; ++j) {
            if (j % p.CS == rank) continue;
            if ((sidx++ & 1) != hf) continue;
            uint32_t v[32];
            tmem_ld_32x32b_x32(tm_row + 32 * j, v);
            tmem_ld_wait();
            uint4* dst = mine + (size_t)j * CHUNK_U4 + nl;
            if (!check((size_t)(dst + 7 * 128 - p.ws) < p.ws_u4, &g_gemm_status)) continue;
#pragma unroll
            for (int pc = 0; pc < 8; ++pc)
                __stcg(dst + pc * 128, make_uint4(v[4 * pc], v[4 * pc + 1], v[4 * pc + 2], v[4 * pc + 3]));
        }
    }
    if (split) cluster_sync();  // release / acquire: the slices above are visible to the owners
    if (warp >= 2 && !*abort_flag) {
        // owned chunks j = rank + CS i (every chunk without a split), alternately per warp half
        for (int j = (split ? rank : 0) + hf * p.CS; j < nchunks; j += 2 * p.CS) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tm_row + 32 * j, v);
            tmem_ld_wait();
            float acc[32];
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) acc[cc] = __uint_as_float(v[cc]);
            if (split) {
                for (int src = 0; src < p.CS; ++src) {
                    if (src == rank) continue;
                    const uint4* sp = p.ws + ((tile_slot + src) * nchunks + j) * CHUNK_U4 + nl;
                    if (!check((size_t)(sp + 7 * 128 - p.ws) < p.ws_u4, &g_gemm_status)) continue;
                    uint4 u[8];
#pragma unroll
                    for (int pc = 0; pc < 8; ++pc) u[pc] = __ldcg(sp + pc * 128);
#pragma unroll
                    for (int pc = 0; pc < 8; ++pc) {
                        acc[4 * pc] += __uint_as_float(u[pc].x);
                        acc[4 * pc + 1] += __uint_as_float(u[pc].y);
                        acc[4 * pc + 2] += __uint_as_float(u[pc].z);
                        acc[4 * pc + 3] += __uint_as_float(u[pc].w);
                    }
                }
            }
            if (ncol < p.N) {
                const float bv = p.bias ? T16::load(p.bias[ncol]) : 0.0f;
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) {
                    const int m = m0 + 32 * j + cc;
                    if (m < p.M) p.y[(size_t)m * p.N + ncol] = T16::store(acc[cc] + bv);
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
// Tile plan shared by the launcher and the workspace query.
struct Tiling {
    int TN;      // tokens per tile, a multiple of 32, at most 256
    int mt;      // token tiles
    int ntiles;  // weight-column tiles
    int CS;      // CTAs per cluster along K (1: no split)
};

size_t split_bytes(const Tiling& t, int CS) {
    return (size_t)t.ntiles * t.mt * CS * (t.TN / 32) * CHUNK_BYTES;
}

// Splits K over up to 8 CTAs while the grid still fits the SMs once and each CTA
// keeps at least two k blocks, as far as ws_bytes of workspace allows.
Tiling plan(int M, int K, int N, size_t ws_bytes) {
    Tiling t{};
    t.mt = (M + 255) / 256;
    const int tn = (M + t.mt - 1) / t.mt;
    t.TN = std::max(32, (tn + 31) / 32 * 32);  // the epilogue reads tensor memory 32 columns at a time
    t.ntiles = (N + BMW - 1) / BMW;
    const int tiles = t.ntiles * t.mt;
    const int KB = (K + BK - 1) / BK;  // a ragged last block reads zeros past K
    const int sms = sm_count();
    t.CS = 1;
    for (int c = 8; c >= 2; c >>= 1) {
        if (KB % c == 0 && KB / c >= 2 && tiles * c <= sms && split_bytes(t, c) <= ws_bytes) {
            t.CS = c;
            break;
        }
    }
    return t;
}

template <int BITS, bool BF>
wq_status run(const Problem& pb, cudaStream_t stream) {
    constexpr int EPS = Fmt<BITS>::EPS;
    constexpr int RW = BK / EPS;
    constexpr int RL = (BITS == 3) ? BK / 32 : 0;

    GemmParams p{};
    p.y = pb.y;
    p.bias = pb.bias;
    p.M = pb.M; p.K = pb.K; p.N = pb.N; p.G = pb.G;
    // s/z rows per 64-deep block: 1 if a group covers whole blocks, else 64 / G
    if (pb.G % BK == 0) {
        p.GPB = 1;
        p.gmode = 0;
    } else if (BK % pb.G == 0) {
        p.GPB = BK / pb.G;
        p.gmode = 1;
    } else {  // a 64-deep block meets at most ceil(63 / G) + 1 groups
        p.GPB = (BK - 1 + pb.G - 1) / pb.G + 1;
        p.gmode = 2;
    }
    p.g_shift = 0;
    while ((1 << (p.g_shift + 1)) <= pb.G && p.g_shift < 6) ++p.g_shift;
    auto kern = p.gmode == 0 ? gemm_kernel<BITS, BF, true> : gemm_kernel<BITS, BF, false>;

    // token tiles of at most 256 (balanced), K split over a cluster where it pays
    const Tiling t = plan(pb.M, pb.K, pb.N, pb.ws ? pb.ws_bytes : 0);
    const int TN = t.TN, mt = t.mt, ntiles = t.ntiles, CS = t.CS;
    p.TN = TN;
    p.CS = CS;
    p.kb_cta = (pb.K + BK - 1) / BK / CS;
    p.ws = static_cast<uint4*>(pb.ws);
    p.ws_u4 = pb.ws_bytes / 16;
    p.late_wait = (pb.flags & WQ_FLAG_PDL_INPUTS_READY) ? 1 : 0;

    // stage layout: x tile | A tile | words | lo words | s rows | z rows (1024-aligned stage)
    const uint32_t xb = (uint32_t)TN * 128u;
    p.off_w = (xb + 1023u) & ~1023u;
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
    // tensor memory: the fp32 accumulator (TN columns), then 32 columns of 16-bit A pairs per stage
    p.a_col = (uint32_t)((TN + 31) / 32 * 32);
    if (p.a_col + 32u * (uint32_t)stages > 512u) stages = (int)((512u - p.a_col) / 32u);
    p.tmem_cols = 32;
    while (p.tmem_cols < p.a_col + 32u * (uint32_t)stages) p.tmem_cols <<= 1;
    if (stages < 2) return WQ_ERR_UNSUPPORTED;
    p.stages = stages;
    const size_t ring = (size_t)stages * p.stage_bytes;
    p.bar_off = (uint32_t)ring;
    // Enough shared memory that the CTAs resident on one SM never ask for more
    // than the SM's 512 tensor-memory columns together, so tcgen05.alloc never
    // waits on a CTA of another cluster: over 116 KB (one CTA per SM) when a CTA
    // takes more than 256 columns, else at least 80 KB (at most two per SM).
    const size_t smem_floor = p.tmem_cols > 256 ? 116 * 1024 : 80 * 1024;
    const size_t smem = std::max<size_t>(1024 + ring + bar_bytes, smem_floor);
    if (smem > limit) return WQ_ERR_UNSUPPORTED;

    CUtensorMap mx, mw, ml, ms, mz;
    const int groups = (pb.K + pb.G - 1) / pb.G;
    bool ok = make_map(&mx, BF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, pb.x, pb.K,
                       pb.M, (uint64_t)pb.K * 2, BK, TN, CU_TENSOR_MAP_SWIZZLE_128B);
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

    // context the smem limit was raised in, per kernel instantiation
    static std::atomic<uint64_t> attr_ctx_gw[MAX_DEVICES], attr_ctx_any[MAX_DEVICES];
    std::atomic<uint64_t>* attr_ctx = p.gmode == 0 ? attr_ctx_gw : attr_ctx_any;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
    if (const wq_status st = ensure_smem_attr((const void*)kern, (int)limit, attr_ctx, dev); st != WQ_OK) return st;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ntiles, mt, CS);
    cfg.blockDim = dim3(NWARPS * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (CS > 1) {  // a cluster of one CTA is no cluster: launch without the attribute
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = CS;
        ++na;
    }
    if (pb.flags & (WQ_FLAG_PDL | WQ_FLAG_PDL_INPUTS_READY)) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, mx, mw, ml, ms, mz, p));
}

template <bool BF>
wq_status launch_typed(const Problem& p, cudaStream_t s) {
    switch (p.bits) {
        case 1: return run<1, BF>(p, s);
        case 2: return run<2, BF>(p, s);
        case 3: return run<3, BF>(p, s);
        case 4: return run<4, BF>(p, s);
        case 8: return run<8, BF>(p, s);
        default: return WQ_ERR_UNSUPPORTED;
    }
}

}  // namespace

wq_status launch_gemm(const Problem& p, cudaStream_t s) {
    return (p.flags & WQ_FLAG_BF16) ? launch_typed<true>(p, s) : launch_typed<false>(p, s);
}

size_t gemm_workspace_bytes(int M, int K, int N, int bits, int G) {
    (void)bits;
    (void)G;
    const Tiling t = plan(M, K, N, ~(size_t)0);
    return t.CS > 1 ? split_bytes(t, t.CS) : 0;
}

wq_status gemm_device_status(int reset) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
    }
    return (v & 1u) ? WQ_ERR_TIMEOUT : (v & 2u) ? WQ_ERR_CHECK : WQ_OK;
}

}  // namespace wq
