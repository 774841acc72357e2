/*
 * wq.h -- C ABI of libwq.so: the weight-only quantized matrix product
 *         y = x @ dequant(W_q) on an sm_100a GPU.
 *
 * Data format (dashq_kernel.py, module docstring, `_pack_kmajor`,
 * `TritonQuantLinear.__init__`; "GPTQModel-Compatible Triton Kernel" README,
 * sections "Quantization Format" and "Group Quantization"):
 *
 *   codes   (K, N)  uint8, row-major: the b-bit code q[k][n] of input row k,
 *                   output column n, 0 <= q < 2^b.
 *   w_q     (K/eps, N) uint32 words, row-major (N contiguous), eps = 32 / b:
 *                   code q[k][n] sits in word w_q[k/eps][n] at bit b*(k%eps).
 *                   b = 1, 2, 4, 8.
 *   3-bit:  w_q (K/16, N) holds the 2-bit plane of q >> 1 (16 per word) and
 *           w_lo (K/32, N) the 1-bit plane of q & 1 (32 per word):
 *           q = (((w_q[k/16][n] >> 2*(k%16)) & 3) << 1) | ((w_lo[k/32][n] >> (k%32)) & 1).
 *   scales, zeros  (K/G, N) IEEE binary16 bit patterns, row-major; G is the
 *                   group size, group_size = -1 meaning G = K (one group per
 *                   output column).  Row k uses group k / G.
 *   dequant         w[k][n] = (q[k][n] - z[k/G][n]) * s[k/G][n]
 *   x  (M, K) binary16 row-major;  y (M, N) binary16 row-major:
 *                   y[m][n] = sum_k x[m][k] * w[k][n], accumulated in fp32
 *                   and rounded to nearest even once at the end.
 *
 * Words are uint32 bit patterns: a code in the top bits makes the int32 view
 * of a word negative, which changes nothing here.
 *
 * Conventions shared by every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates or frees device or host memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     enqueue work on it and return once the launch is accepted; results are
 *     ready when the stream reaches that point.
 *   - Arguments are validated before anything is launched; a rejected call
 *     launches nothing and returns the reason.
 *   - wq_gemv / wq_gemm array pointers must be 16-byte aligned, and packed
 *     word arrays 4-byte aligned everywhere (WQ_ERR_ALIGNMENT otherwise).
 *   - N must be a multiple of 8 for wq_gemv and wq_gemm (128-bit word loads
 *     and 16-byte aligned fp16 rows).
 *   - The device must be compute capability 10.0 (B200, sm_100a); the
 *     library holds sm_100a code only.
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WQ_ABI_VERSION 3

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,   /* a shape, size or pointer the operation cannot take */
    WQ_ERR_UNSUPPORTED = 2,   /* bits outside {1,2,3,4,8}, or a device other than sm_100 */
    WQ_ERR_ALIGNMENT = 3,     /* a pointer not 16-byte aligned, or N not a multiple of 8 */
    WQ_ERR_CODE_RANGE = 4,    /* a code >= 2^bits was found (reported by the bindings) */
    WQ_ERR_TIMEOUT = 5,       /* a kernel gave up a bounded wait (see wq_device_status) */
    WQ_ERR_CUDA = 6,          /* the CUDA runtime refused a launch or query */
    WQ_ERR_SCRATCH_LIMIT = 7, /* the shape needs more split-K scratch than wq_gemm_noalloc holds */
    WQ_ERR_CHECK = 8,         /* checked build only: a kernel's bounds check caught an access outside
                                 its array and skipped it (see wq_device_status) */
    WQ_ERR_NOT_POSITIVE_DEFINITE = 9 /* wq_gptq_quantize: the damped Hessian has a pivot <= 0
                                        (see wq_device_status) */
} wq_status;

/*
 * Launch flags for wq_gemv, wq_gemm, wq_matmul and wq_gemm_noalloc.
 * WQ_FLAG_PDL: launch as a programmatic dependent of the previous kernel on
 *   the stream.  The kernel may start while that kernel still runs: it streams
 *   w_q, w_lo, scales and zeros at once and reads x only after the previous
 *   kernel has completed.  So with this flag the previous kernel on the stream
 *   must not write w_q, w_lo, scales or zeros.  Decode loops over many layers
 *   use it to overlap one product's weight reads with the previous product.
 */
#define WQ_FLAG_PDL 1u
/*
 * WQ_FLAG_PDL_INPUTS_READY: like WQ_FLAG_PDL, but the kernel waits for the
 *   previous kernel on the stream only before it writes y (and, for wq_gemm,
 *   its workspace): it reads x as well as the weights at once.  So the previous
 *   kernel must write none of x, w_q, w_lo, scales and zeros.  Independent
 *   products that follow one another on a stream (projections of one
 *   activation, expert weights of one token) use it to overlap completely.
 */
#define WQ_FLAG_PDL_INPUTS_READY 2u
/*
 * WQ_FLAG_BF16: x, scales, zeros, bias and y hold bfloat16 instead of
 *   binary16 (dashq_kernel.py `TritonQuantLinear`: scale, zero and bias are
 *   stored in its `out_dtype`, and the product is computed in the dtype of x).
 *   The accumulation stays fp32 and y is rounded once to bfloat16 (nearest
 *   even).  wq_gemm dequantises each weight to bfloat16 for the tensor cores
 *   with one bf16 FMA, (q - zi) * s + bf16(-(z - zi) * s), zi = round(z)
 *   clamped to [0, 2^bits - 1] (the module's batched branch dequantises in
 *   the dtype of x); wq_gemv keeps q - zi exact and applies s and z - zi in
 *   fp32.  With either type the layouts, shapes and other rules are the same.
 */
#define WQ_FLAG_BF16 4u
/* Every flag bit the products accept; any other bit gives WQ_ERR_INVALID_ARG. */
#define WQ_FLAG_ALL (WQ_FLAG_PDL | WQ_FLAG_PDL_INPUTS_READY | WQ_FLAG_BF16)

/* Version of this ABI (WQ_ABI_VERSION). */
int wq_abi_version(void);

/* A static, human-readable name for a status code.  Never NULL. */
const char* wq_status_string(wq_status s);

/*
 * Pack codes into K-major words (dashq_kernel.py `_pack_kmajor`; 3-bit planes
 * as in `TritonQuantLinear.__init__`).
 *   codes_kn  (K, N) uint8 device array.
 *   w_q       (K/eps, N) uint32 output (3-bit: (K/16, N) hi plane).
 *   w_lo      3-bit: (K/32, N) uint32 output lo plane; must be NULL otherwise.
 *   bad_count optional uint32 device counter, may be NULL.  When given, the
 *             kernel adds the number of codes >= 2^bits to it (the caller sets
 *             it to zero first).  Such codes are always masked to `bits` bits,
 *             so they never spill into a neighbouring field.
 * Requires K % eps == 0 (3-bit: K % 32 == 0), K >= 1, N >= 1.
 */
wq_status wq_pack_kmajor(const uint8_t* codes_kn, int K, int N, int bits,
                         uint32_t* w_q, uint32_t* w_lo, uint32_t* bad_count, void* stream);

/*
 * Inverse of wq_pack_kmajor (dashq_kernel.py `_unpack_kmajor`; 3-bit
 * recombination as in `dequantize_weight`): writes codes_kn (K, N) uint8.
 * Same shape rules as packing; w_lo required iff bits == 3.
 */
wq_status wq_unpack_kmajor(const uint32_t* w_q, const uint32_t* w_lo, int K, int N, int bits,
                           uint8_t* codes_kn, void* stream);

/*
 * Decode-time product for a few rows of x: 1 <= M <= 16
 * (dashq_kernel.py `_dashq_gemv_kernel` and `forward` for one token; here any
 * M up to 16 reads W_q once).  x (M, K), y (M, N), binary16 (bfloat16 with
 * WQ_FLAG_BF16, which then also applies to scales, zeros and bias).
 * group_size: -1, or a positive divisor of K that is a multiple of 4 * eps
 * (1-bit: 128, 2-bit: 64, 3-bit: 64, 4-bit: 32, 8-bit: 16); other group sizes
 * give WQ_ERR_UNSUPPORTED here (wq_gemm takes them).  Requires K % eps == 0
 * (3-bit: K % 32 == 0) and N % 8 == 0.
 * One launch: the split-K partial sums are reduced on chip (thread-block
 * cluster shared memory); no workspace and no zero-initialised output needed.
 *   bias  optional (N,) device array of the same type as x, 2-byte aligned,
 *         or NULL: then y[m][n] = RN(sum_k x[m][k] w[k][n] + bias[n]), the sum in fp32
 *         (dashq_kernel.py `TritonQuantLinear.forward` adds its bias to the
 *         product's output).
 */
wq_status wq_gemv(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                  const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias,
                  uint16_t* y, int M, int K, int N, int bits, int group_size, unsigned flags,
                  void* stream);

/*
 * Batched product for any M >= 1 ("GPTQModel-Compatible Triton Kernel"
 * README, `gptqmodel_quantized_matmul`; dashq_kernel.py `forward`, batched
 * branch).  Same arguments as wq_gemv (bias included), plus a workspace.  group_size: -1, or a
 * positive divisor of K that is a multiple of eps (3-bit: of 32) and either a
 * multiple or a divisor of 64.  Requires K % 64 == 0 and N % 8 == 0.
 * Packed tiles are dequantised to fp16 (bf16 with WQ_FLAG_BF16) into tensor
 * memory and multiplied on the tensor cores (tcgen05, fp32 accumulators in
 * tensor memory).
 *   workspace        device scratch for splitting K over the CTAs of a cluster
 *                    (fp32 partial tiles, reduced through L2), owned by the
 *                    caller; it needs no initialisation and keeps no state
 *                    between calls.  Calls that may run at the same time on
 *                    the device must not share one.
 *   workspace_bytes  its size; with less than wq_gemm_workspace_size() (or
 *                    NULL) the product is computed without splitting K, which
 *                    is correct but uses fewer SMs for small M x N.
 */
wq_status wq_gemm(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                  const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias,
                  uint16_t* y, int M, int K, int N, int bits, int group_size, unsigned flags,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The product for any M, routed to wq_gemv or wq_gemm by a measured crossover
 * (the M-crossover of the "next" list; not in the pages): wq_gemv when
 * M <= 8, or M <= 16 with 4- or 8-bit words or with M * K < 65536 (x then
 * fits its on-chip staging), and the group size is one wq_gemv takes;
 * wq_gemm otherwise.  Same arguments
 * and rules as wq_gemm; the workspace is used only on the wq_gemm route
 * (wq_matmul_workspace_size() reports 0 on the other).
 */
wq_status wq_matmul(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                    const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias,
                    uint16_t* y, int M, int K, int N, int bits, int group_size, unsigned flags,
                    void* workspace, size_t workspace_bytes, void* stream);

/* 1 if wq_matmul takes the wq_gemv route for this shape, 0 if wq_gemm (host-only). */
int wq_matmul_uses_gemv(int M, int K, int N, int bits, int group_size);

/* Workspace bytes wq_matmul uses for this shape (host-only). */
size_t wq_matmul_workspace_size(int M, int K, int N, int bits, int group_size);

/* Workspace bytes wq_gemm uses for this shape (0 when it does not split K, or
 * when the arguments are invalid).  Host-only: it reads the current device's
 * SM count (148 when there is no device). */
size_t wq_gemm_workspace_size(int M, int K, int N, int bits, int group_size);

/*
 * wq_gemm without a caller workspace, for callers that cannot allocate device
 * memory when they call: a runtime that has handed all device memory to its
 * own pool, or a plug-in whose host forbids allocation after initialisation
 * (cudaMalloc also synchronises the device, which a per-token decode loop
 * cannot afford).  The pages have no counterpart: their kernels take no
 * workspace.
 *
 * Same arguments, rules and result as wq_gemm given a workspace of
 * wq_gemm_workspace_size() bytes.  The split-K scratch is a fixed array of
 * WQ_GEMM_NOALLOC_SCRATCH_BYTES in the library's device image, one per
 * device, so the call allocates nothing.  Nothing in it needs to start at zero
 * and no state is kept in it between calls.
 *   - The first call in each CUDA context looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and keeps it,
 *     keyed on the context's ID; make that first call before any stream
 *     capture.  A context created again after cudaDeviceReset has a new ID,
 *     so its first call looks the address up afresh (and should likewise come
 *     before any capture).
 *   - Calls that may run at the same time on one device (other streams, other
 *     host threads) share the array and race; calls in one stream do not,
 *     WQ_FLAG_PDL_INPUTS_READY included (it waits before the scratch is used).
 *   - A shape whose wq_gemm_workspace_size() exceeds the array is rejected
 *     with WQ_ERR_SCRATCH_LIMIT before anything is launched.  That size, and
 *     so which shapes fit, depends on the current device's SM count (the
 *     split-K plan fills the SMs once); on a 148-SM B200 every shape with
 *     M <= 256 and N <= 2048 fits, and M = 512, K = 4096, N = 2048 needs 16 MiB.
 */
#define WQ_GEMM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
wq_status wq_gemm_noalloc(const uint16_t* x, const uint32_t* w_q, const uint32_t* w_lo,
                          const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias,
                          uint16_t* y, int M, int K, int N, int bits, int group_size,
                          unsigned flags, void* stream);

/*
 * The GPTQModel packed format ("GPTQModel-Compatible Triton Kernel" README,
 * "API Reference": `gptqmodel_quantized_matmul(x, qweight, qzeros, scales,
 * bits, group_size)`; "Quantization Format": 2-bit 16, 3-bit 10 (with
 * padding), 4-bit 8, 8-bit 4 values per int32; "Dequantization Formula":
 * scales * (quantized_weight - quantized_zero)) converted to this library's
 * operands, so that wq_gemv / wq_gemm / wq_matmul compute that product.
 * Readings of what the README leaves open: code k of a column sits in word
 * k / V at bit bits * (k % V), lowest first (for 2, 4, 8 bits the K-major words
 * of this library unchanged); 3-bit words use bits 0-29; qzeros hold the zero
 * points of each group packed along N the same way, with no offset.
 *   qweight  (ceil(K / V), N) int32 device array.
 *   qzeros   (K / G, ceil(N / V)) int32 device array (G = K for group_size -1).
 *   w_q      3-bit: (K / 16, N) output hi plane; 2, 4, 8 bits: NULL (pass qweight
 *            itself to the products) or an output that receives a copy.
 *   w_lo     3-bit: (K / 32, N) output lo plane; NULL otherwise.
 *   zeros    (K / G, N) output, the zero points as binary16 (bfloat16 with
 *            WQ_FLAG_BF16, the only flag taken).
 * bits 2, 3, 4 or 8 (else WQ_ERR_UNSUPPORTED); K % 32 == 0 for 3 bits (the
 * two-plane format), K % (32 / bits) otherwise; the group size divides K.
 * Asynchronous on `stream`.
 */
wq_status wq_gptqmodel_convert(const uint32_t* qweight, const uint32_t* qzeros, int K, int N, int bits,
                               int group_size, uint32_t* w_q, uint32_t* w_lo, uint16_t* zeros,
                               unsigned flags, void* stream);

/*
 * MSE-observer search of per-group scales and zero points ("Benchmark for MSE
 * observer grid search" page: `grid_search_eager`,
 * `grid_search_eager_no_patience`, and the fake quantisation of
 * `_fused_grid_search_kernel`), the step upstream of this library's product
 * that chooses the s and z it consumes.
 *   w          (rows, cols) fp32 device array, row-major, 4-byte aligned;
 *              groups are group_size consecutive values of a row.
 *   bits       1..8.  symmetric = 0: unsigned codes [0, 2^bits - 1] with the
 *              affine rule -- the range widened to contain 0,
 *              s = (hi - lo) / (2^bits - 1), z = clamp(-rint(lo / s)).
 *              symmetric = 1: signed codes [-2^(bits-1), 2^(bits-1) - 1],
 *              s = max(|lo|, |hi|) / ((2^bits - 1) / 2), z = 0 (stored in
 *              this library's unsigned format as q + 2^(bits-1) with zero
 *              point 2^(bits-1)).  A zero scale becomes 2^-23.
 *   steps      candidates, 1..32: candidate i shrinks the group's [min, max]
 *              by p_i = 1 - i / grid (the page evaluates int(maxshrink * grid)).
 *   grid       >= 1.   norm: the error exponent, finite and > 0.
 *   patience   0: every candidate is evaluated; else the search stops after
 *              `patience` candidates in a row in which no group of the whole
 *              tensor improved, as the page's eager search does.
 *   scale, zero, err  (rows, cols / group_size) fp32 outputs: the winning
 *              candidate's parameters and its error sum |w_hat - w|^norm.
 *   step       (rows, cols / group_size) int32 output: the winning candidate.
 *   workspace  4 bytes of device memory (any contents) when patience > 0, else
 *              may be NULL; calls that may run at the same time must not share it.
 * Every step up to w_hat is done in IEEE fp32 (correctly rounded division,
 * round to nearest even), so a candidate's parameters are bit-exact; the error
 * is summed in fp32.  Requires rows, cols >= 1, cols % group_size == 0, and
 * 4-byte aligned arrays.  Asynchronous on `stream`.
 */
wq_status wq_mse_search(const float* w, int rows, int cols, int group_size, int bits, int symmetric,
                        int steps, int grid, float norm, int patience, float* scale, float* zero,
                        int32_t* step, float* err, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * GPTQ block quantisation ("benchmark GPTQ implementations" page:
 * _prepare_weight_and_hessian, quantize_weight_eager with the GROUP strategy,
 * and the fake quantisation of _quantize_block_triton_kernel), in fp32 as the
 * page fixes it.  The producer of the codes that wq_pack_kmajor packs.
 *
 * W (rows x cols, row-major, one row per output channel) and the Hessian H
 * (cols x cols, symmetric, row-major).  Columns c with H[c][c] == 0 are dead:
 * H[c][c] = 1 and W[:, c] = 0.  damp = percdamp * mean(diag H) is added to the
 * diagonal.  Column c takes group g = c / group_size and the fp32 parameters
 * scale[r][g], zero[r][g] (rows x ceil(cols / group_size), row-major; zero
 * points on the page's signed scale, 0 for symmetric arguments).  Columns are
 * quantised from left to right in blocks of `blocksize`:
 *   q = clamp(rint(w / s) + z, -2^(bits-1), 2^(bits-1) - 1), w_hat = (q - z) s,
 * with w the column's current value, and the error is spread over the later
 * columns through the upper Cholesky factor of the inverse damped Hessian.
 *
 * Outputs (device, written on `stream`):
 *   Q      rows x cols fp32, row-major: the fake-quantised W (the page's result),
 *          or null;
 *   codes  cols x rows uint8, K-major (the layout wq_pack_kmajor takes with
 *          K = cols, N = rows): q + 2^(bits-1), so that the product's zero point
 *          is z + 2^(bits-1); or null;
 *   losses rows fp32: half the sum of each row's loss terms (the page's
 *          `losses`; its `loss` is their sum).
 * workspace: wq_gptq_workspace_size(rows, cols) bytes of device memory, 256-byte
 *   aligned, owned by the caller, not read before written; it must not be used
 *   by anything else until the call's work on `stream` is done.
 *
 * Arguments: rows, cols >= 1 (cols <= 65536), 1 <= group_size, bits 1..8,
 * 1 <= blocksize <= 128 (the page's benchmark uses 128; in exact arithmetic
 * the result does not depend on it), 0 <= percdamp < 1e30 (else
 * WQ_ERR_INVALID_ARG / WQ_ERR_UNSUPPORTED for bits).  Float arrays 4-byte
 * aligned (else WQ_ERR_ALIGNMENT).  Scales must be nonzero.
 *
 * A damped Hessian that is not positive definite sets the device status read
 * by wq_device_status (WQ_ERR_NOT_POSITIVE_DEFINITE); the outputs are then
 * NaN.  Asynchronous on `stream`; H and W are only read.
 */
size_t wq_gptq_workspace_size(int rows, int cols);
wq_status wq_gptq_quantize(const float* W, const float* H, const float* scale, const float* zero, int rows,
                           int cols, int group_size, int bits, int blocksize, float percdamp, float* Q,
                           uint8_t* codes, float* losses, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * A decode product prepared once (the weights bound, x and y per call).  The
 * dashq_kernel.py page's TritonQuantLinear holds the packed weights, scales
 * and zero points as a layer and applies them to each new x; this is that
 * layer at the C level: the plan keeps the kernel choice, its launch shape and
 * the TMA descriptors of w_q, w_lo, scales and zeros, so a run is one launch.
 *
 * wq_gemv_plan_create: the arguments of wq_gemv without x, y and the stream,
 *   checked by the same rules (x and y are checked at each run), on the current
 *   device.  *plan receives a handle (null on error).  The plan refers to the
 *   weight, s, z and bias arrays by address: they must stay allocated and may
 *   not move while the plan is used (their contents may change).  Host-only
 *   work plus device attribute queries; nothing is launched.
 * wq_gemv_plan_run: y (M x N) = x (M x K) @ dequant(W_q) on `stream`, the same
 *   result, bits and launch flags as wq_gemv with the plan's arguments.  x, y:
 *   device pointers, 16-byte aligned (else WQ_ERR_ALIGNMENT).  The current
 *   device must be the plan's (else WQ_ERR_INVALID_ARG, nothing launched).
 *   Safe to call from several host threads on one plan (the plan is read only).
 * wq_gemv_plan_destroy: frees the handle (null is allowed).  The plan is valid
 *   in the CUDA context it was created in.
 */
typedef struct wq_gemv_plan wq_gemv_plan;
wq_status wq_gemv_plan_create(const uint32_t* w_q, const uint32_t* w_lo, const uint16_t* scales,
                              const uint16_t* zeros, const uint16_t* bias, int M, int K, int N, int bits,
                              int group_size, unsigned flags, wq_gemv_plan** plan);
wq_status wq_gemv_plan_run(const wq_gemv_plan* plan, const uint16_t* x, uint16_t* y, void* stream);
void wq_gemv_plan_destroy(wq_gemv_plan* plan);

/*
 * Device-side status of the current device: WQ_OK, or WQ_ERR_TIMEOUT when a
 * kernel on this device gave up a bounded wait since the last reset (its
 * output is then incomplete), or WQ_ERR_CHECK when a bounds check of the
 * checked build fired, or WQ_ERR_NOT_POSITIVE_DEFINITE when a factorisation
 * of wq_gptq_quantize met a pivot <= 0 (reported in that order).  Synchronises the device.  reset != 0 clears it.
 */
wq_status wq_device_status(int reset);

/*
 * 1 if this library is the checked build (compiled with WQ_CHECKS, as
 * libwq_checked.so), else 0.  Host-only.  In the checked build every kernel of
 * the products (wq_gemv, wq_gemm and their plans) checks the index of each
 * global and shared-memory access it computes itself
 * (x, y, the split-K workspace, the s/z rows and the staging buffers; the TMA
 * copies are bounded by their descriptors) against the array it belongs to;
 * an access that fails is skipped and recorded, and wq_device_status then
 * returns WQ_ERR_CHECK (after WQ_ERR_TIMEOUT, which it reports first).  It is
 * the stand-in for a memory checker: slower, for tests.
 */
int wq_checked_build(void);

/*
 * Failure-detection self-test (the pages have no counterpart).  Every mbarrier
 * wait in the products is bounded: on time-out the kernel records it in a
 * device status word (read with wq_device_status as WQ_ERR_TIMEOUT), skips its
 * remaining work and exits, so the context stays usable.  This call runs that
 * path on purpose, without any fault: one CTA waits, with the products' bounded
 * wait, on an mbarrier that nothing completes, gives up after limit_ns and
 * records the time-out in a status word of its own.  It synchronises `stream`.
 *   limit_ns  1e3 .. 1e9 (else WQ_ERR_INVALID_ARG, nothing launched)
 * Returns WQ_ERR_TIMEOUT when the wait ran out (the expected result), WQ_OK if
 * it did not, WQ_ERR_CUDA if the launch or the copies failed.  The products'
 * status words are not touched.
 */
wq_status wq_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
