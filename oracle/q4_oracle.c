/*
 * q4_oracle.c -- plain, slow, obviously-correct CPU oracle for blockwise
 * 4-bit weight quantization, dequantization and the skinny matmul
 * C[M,N] = A[M,K] . dequant(W)[N,K]^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no code, header, table or helper with
 * the CUDA library: every conversion below is written out here from the
 * IEEE-754 definitions.
 *
 * What it follows (bitsandbytes PR #1920, "[ROCm] Optimize
 * kgemm_4bit_inference_naive ...", sections "Technical details" and "Fused
 * path support for M > 1", plus the maintainer's reply describing the
 * replacement SIMT kernel):
 *   - the fused op dequantizes blockwise 4-bit weights and multiplies them by
 *     a small number of activation rows (M >= 1, not only the vector case);
 *   - weights are 4-bit indices into a 16-entry code table ("NF4/FP4 dtype
 *     LUT"), scaled per block, default blocksize 64 ("the kernels support the
 *     other blocksizes");
 *   - accumulation is in fp32 on the GPU; this oracle accumulates in fp64;
 *   - only the torch inference (TN) layout: W is stored [out, in] = [N, K].
 * The byte-level contract (two codes per byte, high nibble = even element,
 * one fp32 absmax per contiguous block of row-major W) is the plainest
 * reading the pages support; the pages print no byte layout.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - quantize: x = w / absmax as one correctly rounded fp32 divide; a block
 *     whose absmax is 0 maps every x to 0; idx = argmin_j |x - code[j]| with
 *     the fp32 difference, ties go to the LOWEST j;
 *   - dequantize: out = round_to_dtype(code[idx] *_fp32 absmax), i.e. one
 *     fp32 multiply, then one round-to-nearest-even into the output format;
 *   - GEMM: y = sum_k double(a) * double(w) in k order, w the fp32 product
 *     code[idx] * absmax (not rounded to 16 bits), then one RNE rounding of
 *     the fp64 sum into the activation dtype;
 *   - fp32 activations (the reply: the SIMT kernel takes fp32, fp16 and
 *     bf16 inputs, all with fp32 accumulation): the same sum with a taken as
 *     given, and an fp32 bias.
 *
 * Parity pins: every function here is pinned by the CPU tests (hand-worked
 * examples, brute force on tiny inputs, closed forms, invariants, library
 * conversions); no function is "parity unpinned".
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math:
 * the oracle relies on IEEE single and double arithmetic, subnormals kept).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BF16 0
#define OR_FP16 1
#define OR_FP32 2

#define OR_OK 0
#define OR_BAD 1

/* ------------------------------------------------------------------ */
/* IEEE binary formats: decoding and round-to-nearest-even encoding.   */
/* ------------------------------------------------------------------ */

/* Parameters of a binary floating-point format: p significant bits
 * (including the hidden bit), minimum normal exponent emin, maximum finite
 * value. */
typedef struct {
    int p;
    int emin;
    int emax;
} or_format;

static const or_format OR_FMT_BF16 = {8, -126, 127};
static const or_format OR_FMT_FP16 = {11, -14, 15};
static const or_format OR_FMT_FP32 = {24, -126, 127};

/* Largest finite value of the format: (2 - 2^(1-p)) * 2^emax. */
static double or_max_finite(or_format f) {
    return ldexp(2.0 - ldexp(1.0, 1 - f.p), f.emax);
}

/* Round x (any double) to the nearest value of format f, ties to even,
 * with gradual underflow and overflow to infinity.  The result is returned
 * as a double holding the exactly representable value. */
static double or_round_to_format(double x, or_format f) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    double ax = fabs(x);
    int e2;
    frexp(ax, &e2);             /* ax = m * 2^e2, m in [0.5, 1) */
    int E = e2 - 1;             /* exponent of the leading bit */
    if (E < f.emin) E = f.emin; /* subnormal range: fixed spacing */
    double ulp = ldexp(1.0, E - (f.p - 1));
    double q = ax / ulp;        /* exact: ulp is a power of two */
    double r = nearbyint(q);    /* default rounding mode: ties to even */
    double res = r * ulp;
    if (res > or_max_finite(f)) res = INFINITY;
    return copysign(res, x);
}

/* Spacing of format f at |y|: 2^(floor(log2|y|) - (p-1)) for normal |y|;
 * the subnormal spacing 2^(emin - (p-1)) for y = 0 and subnormal y. */
static double or_ulp(double y, or_format f) {
    double ay = fabs(y);
    int E = f.emin;
    if (ay != 0.0 && !isinf(ay)) {
        int e2;
        frexp(ay, &e2);
        if (e2 - 1 > E) E = e2 - 1;
    }
    return ldexp(1.0, E - (f.p - 1));
}

/* Encode a double that is exactly representable in bf16 into its 16 bits.
 * bf16 is the upper half of binary32, so the binary32 bits are shifted. */
static uint16_t or_bf16_bits_of_exact(double v) {
    float fv = (float)v; /* exact by precondition */
    uint32_t u;
    memcpy(&u, &fv, 4);
    return (uint16_t)(u >> 16);
}

/* Encode a double that is exactly representable in binary16. */
static uint16_t or_fp16_bits_of_exact(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double av = fabs(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(av)) return (uint16_t)(sign | 0x7C00u);
    if (av == 0.0) return sign;
    int e2;
    frexp(av, &e2);
    int E = e2 - 1;
    if (E < -14) {
        /* subnormal: value = mant * 2^-24 */
        double mant = ldexp(av, 24);
        return (uint16_t)(sign | (uint16_t)mant);
    }
    double frac = ldexp(av, -E) - 1.0; /* in [0, 1) */
    uint16_t mant = (uint16_t)ldexp(frac, 10);
    uint16_t bexp = (uint16_t)(E + 15);
    return (uint16_t)(sign | (uint16_t)(bexp << 10) | mant);
}

/* Decode a bf16 bit pattern to its exact binary32 value. */
static float or_bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Decode a binary16 bit pattern to its exact value (as float: every
 * binary16 value is exactly representable in binary32). */
static float or_fp16_to_float(uint16_t h) {
    int sign = (h >> 15) & 1;
    int bexp = (h >> 10) & 0x1F;
    int mant = h & 0x3FF;
    double v;
    if (bexp == 0) {
        v = ldexp((double)mant, -24);
    } else if (bexp == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + ldexp((double)mant, -10), bexp - 15);
    }
    return (float)(sign ? -v : v);
}

static uint16_t or_encode(double x, int dtype) {
    if (dtype == OR_BF16) return or_bf16_bits_of_exact(or_round_to_format(x, OR_FMT_BF16));
    return or_fp16_bits_of_exact(or_round_to_format(x, OR_FMT_FP16));
}

/* ------------------------------------------------------------------ */
/* Exported conversion helpers (pinned directly by the CPU tests).      */
/* ------------------------------------------------------------------ */

/* Round each x[i] (double) once, to nearest-even, into bf16 or fp16 bits. */
int oracle_round(const double* x, int64_t count, int dtype, uint16_t* out) {
    if (dtype != OR_BF16 && dtype != OR_FP16) return OR_BAD;
    for (int64_t i = 0; i < count; ++i) out[i] = or_encode(x[i], dtype);
    return OR_OK;
}

/* Decode bf16 or fp16 bits to doubles (exact). */
int oracle_decode(const uint16_t* bits, int64_t count, int dtype, double* out) {
    if (dtype != OR_BF16 && dtype != OR_FP16) return OR_BAD;
    for (int64_t i = 0; i < count; ++i)
        out[i] = (double)(dtype == OR_BF16 ? or_bf16_to_float(bits[i]) : or_fp16_to_float(bits[i]));
    return OR_OK;
}

/* Spacing (ulp) of the output dtype (bf16, fp16 or fp32) at each y[i]. */
int oracle_ulp(const double* y, int64_t count, int dtype, double* out) {
    if (dtype != OR_BF16 && dtype != OR_FP16 && dtype != OR_FP32) return OR_BAD;
    or_format f = dtype == OR_BF16 ? OR_FMT_BF16 : dtype == OR_FP16 ? OR_FMT_FP16 : OR_FMT_FP32;
    for (int64_t i = 0; i < count; ++i) out[i] = or_ulp(y[i], f);
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Blockwise quantization.                                              */
/* ------------------------------------------------------------------ */

/* Index of the code nearest to x: argmin_j |x - code[j]| using the binary32
 * difference; scanning j upward with a strict "<" keeps the lowest index
 * among equally near codes. */
static int or_nearest_code(float x, const float* code) {
    int best = 0;
    float bestd = fabsf(x - code[0]);
    for (int j = 1; j < 16; ++j) {
        float d = fabsf(x - code[j]);
        if (d < bestd) {
            bestd = d;
            best = j;
        }
    }
    return best;
}

/*
 * Quantize n binary32 values (row-major W flattened) in blocks of `bs`
 * consecutive elements; the last block may be shorter.
 *   absmax[b] = max |w| over block b          (exact)
 *   x         = w / absmax[b]                 (one binary32 division)
 *   idx       = nearest code, lowest index on ties
 *   packed[p] = idx[2p] << 4 | idx[2p+1]      (idx[n] = 0 pads odd n)
 * Returns OR_BAD for a non-finite input or bad arguments.
 */
int oracle_quantize(const float* w, int64_t n, int bs, const float* code, uint8_t* packed,
                    float* absmax) {
    if (n < 0 || bs <= 0) return OR_BAD;
    int64_t nblocks = (n + bs - 1) / bs;
    for (int64_t b = 0; b < nblocks; ++b) {
        int64_t lo = b * (int64_t)bs;
        int64_t hi = lo + bs < n ? lo + bs : n;
        float amax = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            if (!isfinite(w[i])) return OR_BAD;
            float a = fabsf(w[i]);
            if (a > amax) amax = a;
        }
        absmax[b] = amax;
        for (int64_t i = lo; i < hi; ++i) {
            float x = amax > 0.0f ? w[i] / amax : 0.0f;
            int idx = or_nearest_code(x, code);
            if ((i & 1) == 0)
                packed[i >> 1] = (uint8_t)(idx << 4);
            else
                packed[i >> 1] = (uint8_t)(packed[i >> 1] | idx);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Dequantization.                                                      */
/* ------------------------------------------------------------------ */

static int or_index_at(const uint8_t* packed, int64_t i) {
    uint8_t byte = packed[i >> 1];
    return (i & 1) ? (byte & 0x0F) : (byte >> 4);
}

/* The binary32 weight value: code[idx] * absmax, one rounding. */
static float or_weight_at(const uint8_t* packed, const float* absmax, const float* code, int64_t i,
                          int bs) {
    return code[or_index_at(packed, i)] * absmax[i / bs];
}

/*
 * out[i] = round_rne_to_dtype(code[idx_i] * absmax[i / bs]).
 * dtype OR_BF16 / OR_FP16 write uint16 bit patterns; OR_FP32 writes floats.
 */
int oracle_dequantize(const uint8_t* packed, const float* absmax, const float* code, int64_t n,
                      int bs, int dtype, void* out) {
    if (n < 0 || bs <= 0) return OR_BAD;
    for (int64_t i = 0; i < n; ++i) {
        float v = or_weight_at(packed, absmax, code, i, bs);
        if (dtype == OR_FP32)
            ((float*)out)[i] = v;
        else if (dtype == OR_BF16 || dtype == OR_FP16)
            ((uint16_t*)out)[i] = or_encode((double)v, dtype);
        else
            return OR_BAD;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Skinny matmul.                                                       */
/* ------------------------------------------------------------------ */

/*
 * y[m,n] = sum_{k=0}^{K-1} double(a[m,k]) * double(w[n,k])   (fp64, k order)
 * S[m,n] = sum_k |double(a[m,k]) * double(w[n,k])|
 * with w[n,k] = code[idx(n*K+k)] *_fp32 absmax[(n*K+k)/bs] and A given as
 * bf16 or fp16 bit patterns, row-major [M, K].  Either output may be NULL.
 * Any M, N, K >= 0 (K = 0 gives y = 0); blocks may straddle rows.
 */
int oracle_gemm(const uint16_t* A, int act_dtype, const uint8_t* packed, const float* absmax,
                const float* code, int M, int N, int K, int bs, double* y, double* S) {
    if (M < 0 || N < 0 || K < 0 || bs <= 0) return OR_BAD;
    if (act_dtype != OR_BF16 && act_dtype != OR_FP16) return OR_BAD;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, accabs = 0.0;
            for (int k = 0; k < K; ++k) {
                uint16_t abits = A[(int64_t)m * K + k];
                float a = act_dtype == OR_BF16 ? or_bf16_to_float(abits) : or_fp16_to_float(abits);
                float w = or_weight_at(packed, absmax, code, (int64_t)n * K + k, bs);
                double prod = (double)a * (double)w;
                acc += prod;
                accabs += fabs(prod);
            }
            if (y) y[(int64_t)m * N + n] = acc;
            if (S) S[(int64_t)m * N + n] = accabs;
        }
    }
    return OR_OK;
}

/*
 * The same layer with a bias, the epilogue of the planned gemm_4bit op
 * (bitsandbytes PR #1920, "Technical details"):
 *     y[m,n] = bias[n] + sum_k double(a[m,k]) * double(w[n,k])
 * with bias given as N bf16/fp16 bit patterns of the activation type.  The
 * bias enters the fp64 value once, after the k sum; S is the same as without
 * a bias (the bias is exact, it adds no rounding of its own).
 */
int oracle_gemm_bias(const uint16_t* A, int act_dtype, const uint8_t* packed, const float* absmax,
                     const float* code, const uint16_t* bias, int M, int N, int K, int bs, double* y, double* S) {
    if (!bias) return OR_BAD;
    int rc = oracle_gemm(A, act_dtype, packed, absmax, code, M, N, K, bs, y, S);
    if (rc != OR_OK || !y) return rc;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            float b = act_dtype == OR_BF16 ? or_bf16_to_float(bias[n]) : or_fp16_to_float(bias[n]);
            y[(int64_t)m * N + n] += (double)b;
        }
    return OR_OK;
}

/*
 * The skinny matmul with fp32 activations (the maintainer's reply in PR
 * #1920: the replacement SIMT kernel accepts fp32 as well as fp16/bf16
 * inputs):
 *     y[m,n] = [bias[n]] + sum_{k=0}^{K-1} double(a[m,k]) * double(w[n,k])
 *     S[m,n] = sum_k |double(a[m,k]) * double(w[n,k])|
 * in k order in fp64, w[n,k] = code[idx(n*K+k)] *_fp32 absmax[(n*K+k)/bs]
 * as in oracle_gemm, A given as binary32 values, row-major [M, K], and bias
 * (N binary32 values) optional (NULL: none).  Either output may be NULL.
 */
int oracle_gemm_f32(const float* A, const uint8_t* packed, const float* absmax, const float* code,
                    const float* bias, int M, int N, int K, int bs, double* y, double* S) {
    if (M < 0 || N < 0 || K < 0 || bs <= 0) return OR_BAD;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, accabs = 0.0;
            for (int k = 0; k < K; ++k) {
                float a = A[(int64_t)m * K + k];
                float w = or_weight_at(packed, absmax, code, (int64_t)n * K + k, bs);
                double prod = (double)a * (double)w;
                acc += prod;
                accabs += fabs(prod);
            }
            if (bias) acc += (double)bias[n];
            if (y) y[(int64_t)m * N + n] = acc;
            if (S) S[(int64_t)m * N + n] = accabs;
        }
    }
    return OR_OK;
}
