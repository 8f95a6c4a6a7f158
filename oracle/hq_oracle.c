/*
 * Plain CPU oracle for the Hadamard-rotated, tensor-wise-quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file:
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it follows (web pages on the subject):
 *  - "Training Transformers with 4-bit Integers" (paperlayer.ai summary), section 3.3
 *    "Hadamard Quantization": a block-diagonal transform built from Hadamard blocks H_k is
 *    applied to both matmul operands; the transform cancels in the product.
 *  - "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs" (atlas.scime.ai summary),
 *    "Approach": right-hand Hadamard on activations and weights in the forward pass, a
 *    left-hand Hadamard on output gradients in the backward pass (HALO-2), tensor-wise
 *    quantization; "Limitations": tensor-wise round-to-nearest quantization, FP8 as the
 *    hardware format below FP6.
 *  - Same 4-bit page, section 3.1 "Learned Step Size Quantization": symmetric integer range
 *    (QN = QP) and an INT32 product dequantized back to floating point.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - H_k is Sylvester's natural-order Hadamard matrix; the FWHT runs its stages with the
 *    pairing distance h = 1, 2, 4, ..., k/2 (index bit 0 first), every add/sub in fp32
 *    round-to-nearest-even, no fused multiply-add (build with -ffp-contract=off).
 *  - The rotation is orthonormal: y = fp32(t * c_k), c_k = fp32(1/sqrt(k)).
 *  - INT8: inv = fp32(127/a), q = clamp(rne(fp32(y*inv)), -127, 127), scale = fp32(a/127).
 *  - FP8 e4m3 (E4M3FN, bias 7, max 448, no infinities): inv = fp32(448/a),
 *    q = e4m3 nearest-even of fp32(y*inv) saturated to +-448, scale = fp32(a/448).
 *  - FP6 / FP4 (the formats HALO names below FP8; the pages give no bit layout): the
 *    minifloats e3m2 (bias 3, max 28), e2m3 (bias 1, max 7.5) and e2m1 (bias 1, max 6),
 *    sign-magnitude, subnormals, no infinities or NaN; inv = fp32(max/a), q = nearest-even
 *    of fp32(y*inv) saturated to +-max, scale = fp32(a/max); one code per byte, value in the
 *    low 6 (4) bits.
 *  - a = 0 gives scale 1 and all-zero codes; a non-finite a is an error.
 *  - Codes are stored with the rotated dimension innermost (K-major for the GEMM).
 *
 * Precision: the FWHT and quantizer are fp32 because the method fixes that precision for
 * its codes; the FP8 GEMM accumulates in fp64 (exact for e4m3 products at these K); the
 * INT8 GEMM accumulates in int32 (exact while 127*127*K < 2^31).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_SHAPE 2
#define ORC_ERR_NONFINITE 5

/* Threads the OpenMP loops below will use (reported with CPU timings). */
int hq_oracle_threads(void) { return omp_get_max_threads(); }

/* ---------------------------------------------------------------- bf16 <-> fp32 */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static float bf16_bits_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to a binary format with `p` significand bits (implicit bit included),
 * minimum normal exponent `emin` (value 2^emin), round-to-nearest, ties to even.
 * No overflow handling: callers stay in range.  Uses only exact power-of-two scaling
 * and rint() in the default (nearest-even) rounding mode. */
static double round_to_format(double v, int p, int emin) {
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);        /* a = f * 2^e, f in [0.5, 1) -> leading bit has weight 2^(e-1) */
    int lead = e - 1;
    if (lead < emin) lead = emin; /* subnormal: quantum fixed at 2^(emin-p+1) */
    double quantum = ldexp(1.0, lead - (p - 1));
    double r = rint(a / quantum) * quantum;
    return v < 0 ? -r : r;
}

/* double -> bf16 bits, one rounding to nearest even (bf16: 8 significand bits, emin -126). */
uint16_t hq_oracle_bf16_from_f64(double v) {
    double r = round_to_format(v, 8, -126);
    float f = (float)r; /* exact: r has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

uint16_t hq_oracle_bf16_from_f32(float v) { return hq_oracle_bf16_from_f64((double)v); }

/* ---------------------------------------------------------------- e4m3 */

/* E4M3FN decode from the bit definition: s eeee mmm, bias 7; e=0 subnormal m*2^-9;
 * 0x7F / 0xFF are NaN (there are no infinities). */
double hq_oracle_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* fp32 -> e4m3 code, nearest with ties to even, saturating to +-448 (never NaN for finite
 * input). */
uint8_t hq_oracle_e4m3_encode(float x) {
    double v = (double)x;
    uint8_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;                 /* saturate */
    double r = round_to_format(a, 4, -6);               /* 4 significand bits, emin -6 */
    if (r >= 448.0) return sign | 0x7E;
    if (r == 0.0) return sign;
    int e;
    frexp(r, &e);
    int lead = e - 1;
    if (lead < -6) {                                    /* subnormal: m * 2^-9 */
        int m = (int)ldexp(r, 9);
        return sign | (uint8_t)m;
    }
    int m = (int)((ldexp(r, -lead) - 1.0) * 8.0);
    return sign | (uint8_t)(((lead + 7) << 3) | m);
}

/* ---------------------------------------------------------------- FP6 / FP4 minifloats */

/* Format parameters by code: fmt 2 = e3m2, 3 = e2m3, 4 = e2m1 (exponent bits, mantissa bits,
 * bias).  Returns 0 for any other fmt. */
static int minifloat_params(int fmt, int* ebits, int* mbits, int* bias) {
    switch (fmt) {
        case 2: *ebits = 3; *mbits = 2; *bias = 3; return 1;
        case 3: *ebits = 2; *mbits = 3; *bias = 1; return 1;
        case 4: *ebits = 2; *mbits = 1; *bias = 1; return 1;
        default: return 0;
    }
}

/* Largest finite value: all exponent and mantissa bits set (there are no infinities). */
double hq_oracle_minifloat_max(int fmt) {
    int eb, mb, bias;
    if (!minifloat_params(fmt, &eb, &mb, &bias)) return NAN;
    return ldexp(2.0 - ldexp(1.0, -mb), (1 << eb) - 1 - bias);
}

/* Decode from the bit definition: s | e (eb bits) | m (mb bits); e = 0 is subnormal,
 * m * 2^(1 - bias - mb); otherwise (1 + m / 2^mb) * 2^(e - bias).  Bits above the sign are
 * ignored. */
double hq_oracle_minifloat_decode(int fmt, uint8_t c) {
    int eb, mb, bias;
    if (!minifloat_params(fmt, &eb, &mb, &bias)) return NAN;
    int s = (c >> (eb + mb)) & 1, e = (c >> mb) & ((1 << eb) - 1), m = c & ((1 << mb) - 1);
    double v = e == 0 ? ldexp((double)m, 1 - bias - mb) : ldexp(1.0 + ldexp((double)m, -mb), e - bias);
    return s ? -v : v;
}

/* fp32 -> code, nearest with ties to even, saturating to +-max; the sign of zero is kept. */
uint8_t hq_oracle_minifloat_encode(int fmt, float x) {
    int eb, mb, bias;
    if (!minifloat_params(fmt, &eb, &mb, &bias)) return 0;
    const uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? (uint8_t)(1u << (eb + mb)) : 0;
    const uint8_t maxcode = (uint8_t)((1u << (eb + mb)) - 1);
    const double mx = hq_oracle_minifloat_max(fmt), emin = 1 - bias;
    double a = fabs((double)x);
    if (a >= mx) return sign | maxcode;
    double r = round_to_format(a, mb + 1, (int)emin);
    if (r >= mx) return sign | maxcode;
    if (r == 0.0) return sign;
    int e;
    frexp(r, &e);
    int lead = e - 1;
    if (lead < emin) return sign | (uint8_t)(int)ldexp(r, bias - 1 + mb); /* subnormal */
    int m = (int)ldexp(ldexp(r, -lead) - 1.0, mb);
    return sign | (uint8_t)(((lead + bias) << mb) | m);
}

/* ---------------------------------------------------------------- Hadamard */

/* In-place Sylvester FWHT of one block of length k: for h = 1, 2, ..., k/2, every pair
 * (i, i+h) with bit h of i clear becomes (x_i + x_{i+h}, x_i - x_{i+h}).  Unnormalised. */
void hq_oracle_fwht_block(float* x, int k) {
    for (int h = 1; h < k; h <<= 1) {
        for (int i = 0; i < k; ++i) {
            if (i & h) continue;
            float u = x[i], v = x[i + h];
            x[i] = u + v;
            x[i + h] = u - v;
        }
    }
}

/* fp32(1/sqrt(k)), correctly rounded: computed in double then rounded once to fp32. */
float hq_oracle_norm_const(int k) { return (float)(1.0 / sqrt((double)k)); }

static int valid_k(int k) { return k == 16 || k == 32 || k == 64 || k == 128 || k == 256; }

static float load_elem(const void* src, int dtype, int64_t idx) {
    if (dtype == 0) return ((const float*)src)[idx];
    return bf16_bits_to_f32(((const uint16_t*)src)[idx]);
}

/* Randomized variant (a random sign diagonal D before the Hadamard blocks, t = H_k D x: the
 * "randomized Hadamard transform" of the neighbouring pages' incoherence processing, e.g. the
 * QuIP# abstract in the search listing).  neg[p] != 0 negates position p of the rotated
 * dimension (one flag per position, shared by every block row/column); NULL = no signs.
 * The negation is exact, so D only permutes signs before the same fp32 butterflies. */
int hq_oracle_rotate_signed(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                            const uint8_t* neg, float* y);

/* Rotate src[rows][cols] (dtype 0 = fp32, 1 = bf16) along `dim` in blocks of k and normalise.
 * dim = 1: along cols, y has shape [rows][cols].
 * dim = 0: along rows, y has shape [cols][rows] (the rotated dimension is made innermost).
 * Returns ORC_OK or an error code. */
int hq_oracle_rotate(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                     float* y) {
    return hq_oracle_rotate_signed(src, dtype, rows, cols, dim, k, NULL, y);
}

int hq_oracle_rotate_signed(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                            const uint8_t* neg, float* y) {
    if (!valid_k(k) || (dtype != 0 && dtype != 1) || (dim != 0 && dim != 1)) return ORC_ERR_ARG;
    if (rows < 0 || cols < 0) return ORC_ERR_ARG;
    int64_t rot = dim == 1 ? cols : rows, other = dim == 1 ? rows : cols;
    if (rot % k != 0) return ORC_ERR_SHAPE;
    float c = hq_oracle_norm_const(k);
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < other; ++o) {
        float buf[256];
        for (int64_t b = 0; b < rot; b += k) {
            for (int i = 0; i < k; ++i) {
                int64_t r = dim == 1 ? o : b + i, cc = dim == 1 ? b + i : o;
                float v = load_elem(src, dtype, r * cols + cc);
                buf[i] = (neg && neg[b + i]) ? -v : v;
            }
            hq_oracle_fwht_block(buf, k);
            for (int i = 0; i < k; ++i) y[o * rot + b + i] = buf[i] * c;
        }
    }
    return ORC_OK;
}

/* Tensor-wise absmax of n fp32 values; returns +INF if any value is not finite. */
static float absmax(const float* y, int64_t n) {
    float a = 0.0f;
    int bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(y[i]);
        if (!(v <= 3.4028234663852886e38f)) bad = 1;
        else if (v > a) a = v;
    }
    return bad ? INFINITY : a;
}

/* Quantize already-rotated values y[n] tensor-wise.  fmt 0 = INT8, 1 = FP8 e4m3,
 * 2 = FP6 e3m2, 3 = FP6 e2m3, 4 = FP4 e2m1.  Writes n one-byte codes and the fp32
 * dequantization scale. */
int hq_oracle_quantize_rotated_given(const float* y, int64_t n, int fmt, float a, uint8_t* codes, float* scale);

int hq_oracle_quantize_rotated(const float* y, int64_t n, int fmt, uint8_t* codes, float* scale) {
    if (fmt < 0 || fmt > 4) return ORC_ERR_ARG;
    return hq_oracle_quantize_rotated_given(y, n, fmt, absmax(y, n), codes, scale);
}

/* The same quantizer with the tensor-wise absmax a supplied: for a slice of a larger tensor,
 * a is the whole tensor's (sharded quantization). */
int hq_oracle_quantize_rotated_given(const float* y, int64_t n, int fmt, float a, uint8_t* codes, float* scale) {
    if (fmt < 0 || fmt > 4) return ORC_ERR_ARG;
    if (!isfinite(a)) {
        *scale = NAN;
        return ORC_ERR_NONFINITE;
    }
    if (a == 0.0f) {
        memset(codes, 0, (size_t)n);
        *scale = 1.0f;
        return ORC_OK;
    }
    float qmax = fmt == 0 ? 127.0f : fmt == 1 ? 448.0f : (float)hq_oracle_minifloat_max(fmt);
    float inv = qmax / a;
    *scale = a / qmax;
    for (int64_t i = 0; i < n; ++i) {
        float z = y[i] * inv;
        if (fmt == 0) {
            float r = rintf(z);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            codes[i] = (uint8_t)(int8_t)(int)r;
        } else if (fmt == 1) {
            codes[i] = hq_oracle_e4m3_encode(z);
        } else {
            codes[i] = hq_oracle_minifloat_encode(fmt, z);
        }
    }
    return ORC_OK;
}

/* max |y[i]| (exact; +inf if any element is not finite). */
float hq_oracle_absmax(const float* y, int64_t n) { return absmax(y, n); }

/* Rotate then quantize (hq_quantize's definition).  codes has the rotated dim innermost. */
int hq_oracle_quantize_signed(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                              const uint8_t* neg, int fmt, uint8_t* codes, float* scale);

int hq_oracle_quantize(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                       int fmt, uint8_t* codes, float* scale) {
    return hq_oracle_quantize_signed(src, dtype, rows, cols, dim, k, NULL, fmt, codes, scale);
}

/* Randomized variant: the sign flags neg (see hq_oracle_rotate_signed), then the same. */
int hq_oracle_quantize_signed(const void* src, int dtype, int64_t rows, int64_t cols, int dim, int k,
                              const uint8_t* neg, int fmt, uint8_t* codes, float* scale) {
    int64_t n = rows * cols;
    float* y = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!y) return ORC_ERR_ARG;
    int st = hq_oracle_rotate_signed(src, dtype, rows, cols, dim, k, neg, y);
    if (st == ORC_OK) st = hq_oracle_quantize_rotated(y, n, fmt, codes, scale);
    free(y);
    return st;
}

/* ---------------------------------------------------------------- GEMMs */

/* C[i][j] = sum_l A[i][l] * B[j][l], int8 codes, int32 accumulation, for the listed rows
 * of A (rows == NULL: all M rows, C is [M][N]; else C is [nrows][N]). */
void hq_oracle_gemm_i8(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K,
                       const int64_t* rows, int64_t nrows, int32_t* C) {
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const int8_t* a = A + (rows ? rows[r] : r) * K;
        for (int64_t j = 0; j < N; ++j) {
            const int8_t* b = B + j * K;
            int32_t s = 0;
            for (int64_t l = 0; l < K; ++l) s += (int32_t)a[l] * (int32_t)b[l];
            C[r * N + j] = s;
        }
    }
}

/* Same contraction for floating-point codes (fmt 1 = e4m3, 2..4 = FP6 / FP4), each decoded
 * exactly to double, fp64 accumulation (exact for these formats at the sizes tested). */
void hq_oracle_gemm_fp(int fmt, const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K,
                       const int64_t* rows, int64_t nrows, double* C) {
    double lut[256];
    for (int c = 0; c < 256; ++c)
        lut[c] = fmt == 1 ? hq_oracle_e4m3_decode((uint8_t)c) : hq_oracle_minifloat_decode(fmt, (uint8_t)c);
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const uint8_t* a = A + (rows ? rows[r] : r) * K;
        for (int64_t j = 0; j < N; ++j) {
            const uint8_t* b = B + j * K;
            double s = 0.0;
            for (int64_t l = 0; l < K; ++l) s += lut[a[l]] * lut[b[l]];
            C[r * N + j] = s;
        }
    }
}

void hq_oracle_gemm_f8(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K,
                       const int64_t* rows, int64_t nrows, double* C) {
    hq_oracle_gemm_fp(1, A, B, M, N, K, rows, nrows, C);
}

/* ---------------------------------------------------------------- dequantization epilogue */

/* Two evaluations of out = acc * s_a * s_b as bf16:
 *  ref  : the value fp64(acc) * s_a * s_b (two fp64 products, relative error below 2^-52)
 *         rounded to bf16: the reference the 1-ulp bound is measured against;
 *  fast : the device formula bf16(fp32(acc) * fp32(s_a * s_b)), every step fp32 RNE.
 * acc_kind 0 = int32 accumulators, 1 = double accumulators.  Either output may be NULL. */
void hq_oracle_epilogue(const void* acc, int acc_kind, int64_t n, float sa, float sb,
                        uint16_t* ref, uint16_t* fast) {
    float sab = sa * sb;
    for (int64_t i = 0; i < n; ++i) {
        double a = acc_kind == 0 ? (double)((const int32_t*)acc)[i] : ((const double*)acc)[i];
        if (ref) ref[i] = hq_oracle_bf16_from_f64(a * (double)sa * (double)sb);
        if (fast) {
            float af = acc_kind == 0 ? (float)((const int32_t*)acc)[i] : (float)a;
            float v = af * sab;
            fast[i] = hq_oracle_bf16_from_f32(v);
        }
    }
}

/* ---------------------------------------------------------------- rotated-output placement */

/* The accumulators scaled to fp32 without the bf16 rounding: z = fp32(acc) * fp32(s_a * s_b),
 * every step fp32 RNE (the "fast" epilogue formula above, stopped before bf16).  Used where
 * the GEMM's output is still rotated and is de-rotated in fp32 before it is rounded. */
void hq_oracle_dequant_f32(const void* acc, int acc_kind, int64_t n, float sa, float sb, float* z) {
    float sab = sa * sb;
    for (int64_t i = 0; i < n; ++i) {
        float af = acc_kind == 0 ? (float)((const int32_t*)acc)[i] : (float)((const double*)acc)[i];
        z[i] = af * sab;
    }
}

/* bf16 bit patterns of n fp32 values, each rounded to nearest even. */
void hq_oracle_f32_to_bf16(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = hq_oracle_bf16_from_f32(x[i]);
}
