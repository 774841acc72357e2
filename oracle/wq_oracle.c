/*
 * wq_oracle.c -- the CPU oracle for the weight-only quantized matrix product.
 *
 * TEST INFRASTRUCTURE.  This file is not part of the product.  Only the test
 * suite, the smoke check and the bench's CPU-baseline / reference arm may
 * build, load or call it.  It shares no code, header, table or helper with the
 * CUDA library; the only thing both sides share is the seeded input generator.
 *
 * What it computes is the plain definition of the method, written out loop by
 * loop in fp64, with no blocking, fusion or reordering:
 *
 *   q[k][n]  = the k-bit code of row k, column n, read from the K-major packed
 *              words            (dashq_kernel.py: module docstring, `_pack_kmajor`,
 *                                `_unpack_kmajor`; 3-bit two bit-planes:
 *                                `TritonQuantLinear.__init__`, `dequantize_weight`)
 *   g        = k / group_size, group_size = -1 meaning one group of K rows
 *                               ("GPTQModel-Compatible Triton Kernel" README,
 *                                section "Group Quantization")
 *   w[k][n]  = (q[k][n] - z[g][n]) * s[g][n]
 *                               (README section "Dequantization Formula";
 *                                dashq_kernel.py `dequantize_weight`)
 *   y[m][n]  = sum_k x[m][k] * w[k][n], k ascending
 *                               (README "API Reference": output = x @ dequantize(qweight);
 *                                dashq_kernel.py `forward`, batched branch)
 *   B[m][n]  = sum_k |x[m][k] * w[k][n]|   (the scale of the error bound)
 *
 * The floating-point inputs (x, s, z, bias) are all fp16 or all bf16 (the
 * module's `out_dtype`, dashq_kernel.py `TritonQuantLinear.__init__`), chosen
 * by the `dt` argument: ORC_FP16 (0) or ORC_BF16 (1).  Both are widened to
 * double exactly from their definitions: IEEE 754 binary16 (sign, 5-bit
 * exponent with bias 15, 10-bit fraction) and bfloat16 (sign, 8-bit exponent
 * with bias 127, 7-bit fraction: the upper half of a binary32).
 *
 * Words are handled as uint32 bit patterns with logical shifts; the pages'
 * torch code uses int32 with arithmetic shifts and a mask, which gives the same
 * bits for every code.
 *
 * Return values: 0 on success, a negative ORC_E* value otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EARG (-1)        /* a shape or group size the definition cannot take */
#define ORC_EBITS (-2)       /* a bit width outside {1, 2, 3, 4, 8} */
#define ORC_ERANGE (-3)      /* a code that does not fit in `bits` bits */
#define ORC_ENOMEM (-4)

#define ORC_FP16 0
#define ORC_BF16 1

int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the OpenMP loops use from now on (timing only; results do not depend on it). */
void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* IEEE 754 binary16 -> double, exact. */
double orc_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 -> double, exact. */
double orc_bf16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -133);              /* subnormal: f * 2^-126 * 2^-7 */
    } else if (e == 255) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(128 + f), e - 134);   /* (1 + f/128) * 2^(e-127) */
    }
    return sign ? -v : v;
}

/* One stored value of type dt widened to double. */
static double widen(uint16_t h, int dt) {
    return dt == ORC_BF16 ? orc_bf16_to_double(h) : orc_half_to_double(h);
}

static int supported_dt(int dt) { return dt == ORC_FP16 || dt == ORC_BF16; }

/* out[i] = the value of v[i] (type dt) as a double. */
int orc_widen(const uint16_t* v, int n, int dt, double* out) {
    if (n < 0 || !supported_dt(dt)) return ORC_EARG;
    for (int i = 0; i < n; ++i) out[i] = widen(v[i], dt);
    return ORC_OK;
}

static int supported_bits(int bits) {
    return bits == 1 || bits == 2 || bits == 3 || bits == 4 || bits == 8;
}

/* Rows of K one packed word holds: 32 / bits (dashq_kernel.py `_pack_kmajor`). */
static int elems_per_word(int bits) { return 32 / bits; }

/* Pack a single k-bit plane: word[k / eps][n] |= v[k][n] << (bits * (k % eps)). */
static void pack_plane(const uint8_t* v_kn, int K, int N, int bits, int shift_down,
                       uint8_t mask_after, uint32_t* words) {
    int eps = elems_per_word(bits);
    memset(words, 0, sizeof(uint32_t) * (size_t)(K / eps) * (size_t)N);
    for (int k = 0; k < K; ++k) {
        for (int n = 0; n < N; ++n) {
            uint32_t v = (uint32_t)((v_kn[(size_t)k * N + n] >> shift_down) & mask_after);
            words[(size_t)(k / eps) * N + n] |= v << (bits * (k % eps));
        }
    }
}

/*
 * codes_kn (K, N) uint8 -> wq (K / eps, N) words.  3-bit: wq is the 2-bit plane
 * of (q >> 1), shape (K / 16, N), and wlo the 1-bit plane of (q & 1), shape
 * (K / 32, N) (dashq_kernel.py `TritonQuantLinear.__init__`).
 */
int orc_pack_kmajor(const uint8_t* codes_kn, int K, int N, int bits, uint32_t* wq, uint32_t* wlo) {
    if (!supported_bits(bits)) return ORC_EBITS;
    if (K <= 0 || N <= 0) return ORC_EARG;
    int kdiv = bits == 3 ? 32 : elems_per_word(bits);
    if (K % kdiv != 0) return ORC_EARG;
    uint32_t qmax = (1u << bits) - 1u;
    for (size_t i = 0; i < (size_t)K * N; ++i)
        if (codes_kn[i] > qmax) return ORC_ERANGE;
    if (bits == 3) {
        pack_plane(codes_kn, K, N, 2, 1, 3, wq);
        pack_plane(codes_kn, K, N, 1, 0, 1, wlo);
    } else {
        pack_plane(codes_kn, K, N, bits, 0, (uint8_t)qmax, wq);
    }
    return ORC_OK;
}

/* The code of row k, column n (dashq_kernel.py `_unpack_kmajor`; 3-bit:
 * q = (((hi >> 2*(k % 16)) & 3) << 1) | ((lo >> (k % 32)) & 1)). */
static uint32_t code_at(const uint32_t* wq, const uint32_t* wlo, int N, int bits, int k, int n) {
    if (bits == 3) {
        uint32_t hi = (wq[(size_t)(k / 16) * N + n] >> (2 * (k % 16))) & 3u;
        uint32_t lo = (wlo[(size_t)(k / 32) * N + n] >> (k % 32)) & 1u;
        return (hi << 1) | lo;
    }
    int eps = elems_per_word(bits);
    return (wq[(size_t)(k / eps) * N + n] >> (bits * (k % eps))) & ((1u << bits) - 1u);
}

int orc_unpack_kmajor(const uint32_t* wq, const uint32_t* wlo, int K, int N, int bits, uint8_t* codes_kn) {
    if (!supported_bits(bits)) return ORC_EBITS;
    if (K <= 0 || N <= 0) return ORC_EARG;
    int kdiv = bits == 3 ? 32 : elems_per_word(bits);
    if (K % kdiv != 0) return ORC_EARG;
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n)
            codes_kn[(size_t)k * N + n] = (uint8_t)code_at(wq, wlo, N, bits, k, n);
    return ORC_OK;
}

static int resolve_group(int K, int group_size) {
    if (group_size == -1) return K;
    if (group_size <= 0 || K % group_size != 0) return -1;
    return group_size;
}

/* w_kn[k][n] = (q - z[g][n]) * s[g][n] in fp64, g = k / G. */
int orc_dequant(const uint32_t* wq, const uint32_t* wlo, const uint16_t* s, const uint16_t* z,
                int K, int N, int bits, int group_size, double* w_kn, int dt) {
    if (!supported_bits(bits)) return ORC_EBITS;
    int G = resolve_group(K, group_size);
    if (G < 0 || N <= 0 || !supported_dt(dt)) return ORC_EARG;
    int kdiv = bits == 3 ? 32 : elems_per_word(bits);
    if (K % kdiv != 0) return ORC_EARG;
    /* Rows are independent: each element is the same fp64 expression whichever
     * thread computes it. */
#pragma omp parallel for schedule(static)
    for (int k = 0; k < K; ++k) {
        int g = k / G;
        for (int n = 0; n < N; ++n) {
            double q = (double)code_at(wq, wlo, N, bits, k, n);
            double zz = widen(z[(size_t)g * N + n], dt);
            double ss = widen(s[(size_t)g * N + n], dt);
            w_kn[(size_t)k * N + n] = (q - zz) * ss;
        }
    }
    return ORC_OK;
}

/* y[m][n] = sum_k x[m][k] * w[k][n] (k ascending), bound[m][n] = sum_k |x w|. */
int orc_matmul(const uint16_t* x, const double* w_kn, int M, int K, int N, double* y, double* bound,
               int dt) {
    if (M <= 0 || K <= 0 || N <= 0 || !supported_dt(dt)) return ORC_EARG;
    double* xd = (double*)malloc(sizeof(double) * (size_t)M * K);
    if (!xd) return ORC_ENOMEM;
    for (size_t i = 0; i < (size_t)M * K; ++i) xd[i] = widen(x[i], dt);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int m = 0; m < M; ++m) {
            double acc = 0.0, b = 0.0;
            for (int k = 0; k < K; ++k) {
                double p = xd[(size_t)m * K + k] * w_kn[(size_t)k * N + n];
                acc += p;
                b += fabs(p);
            }
            y[(size_t)m * N + n] = acc;
            if (bound) bound[(size_t)m * N + n] = b;
        }
    }
    free(xd);
    return ORC_OK;
}

/* The whole product: unpack, dequantise, fp64 matmul. */
int orc_wq_matmul(const uint16_t* x, const uint32_t* wq, const uint32_t* wlo, const uint16_t* s,
                  const uint16_t* z, int M, int K, int N, int bits, int group_size,
                  double* y, double* bound, int dt) {
    if (M <= 0) return ORC_EARG;
    double* w = (double*)malloc(sizeof(double) * (size_t)K * N);
    if (!w) return ORC_ENOMEM;
    int rc = orc_dequant(wq, wlo, s, z, K, N, bits, group_size, w, dt);
    if (rc == ORC_OK) rc = orc_matmul(x, w, M, K, N, y, bound, dt);
    free(w);
    return rc;
}

/*
 * Fused bias ("dashq_kernel.py" `TritonQuantLinear.forward`: the output of
 * the product plus `bias`, one value per output column, of type dt):
 * y[m][n] += bias[n], and the bias is one more addend of the error bound,
 * bound[m][n] += |bias[n]|.
 */
int orc_add_bias(double* y, double* bound, const uint16_t* bias, int M, int N, int dt) {
    if (M <= 0 || N <= 0 || !bias || !supported_dt(dt)) return ORC_EARG;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double b = widen(bias[n], dt);
            y[(size_t)m * N + n] += b;
            if (bound) bound[(size_t)m * N + n] += fabs(b);
        }
    return ORC_OK;
}

/*
 * The same product for a list of single outputs (m_i, n_i), each computed on
 * its own straight from the packed words.  Used where the full product is too
 * large to hold in fp64 or to finish in seconds.
 */
int orc_wq_matmul_sampled(const uint16_t* x, const uint32_t* wq, const uint32_t* wlo,
                          const uint16_t* s, const uint16_t* z, int M, int K, int N, int bits,
                          int group_size, const int32_t* ms, const int32_t* ns, int count,
                          double* y, double* bound, int dt) {
    if (!supported_bits(bits)) return ORC_EBITS;
    int G = resolve_group(K, group_size);
    if (G < 0 || M <= 0 || N <= 0 || !supported_dt(dt)) return ORC_EARG;
    int kdiv = bits == 3 ? 32 : elems_per_word(bits);
    if (K % kdiv != 0) return ORC_EARG;
    for (int i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_EARG;
#pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < count; ++i) {
        int m = ms[i], n = ns[i];
        double acc = 0.0, b = 0.0;
        for (int k = 0; k < K; ++k) {
            int g = k / G;
            double q = (double)code_at(wq, wlo, N, bits, k, n);
            double w = (q - widen(z[(size_t)g * N + n], dt)) * widen(s[(size_t)g * N + n], dt);
            double p = widen(x[(size_t)m * K + k], dt) * w;
            acc += p;
            b += fabs(p);
        }
        y[i] = acc;
        if (bound) bound[i] = b;
    }
    return ORC_OK;
}
