/*
 * dq_oracle.c -- plain, slow, single-threaded CPU oracle for the int8
 * dynamic-quantization linear layer (dense and 64x64 block-sparse weight).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Every routine is the method's definition written out with scalar loops,
 * in the order the sources state it:
 *
 *  - Per-token ("per-row") dynamic absmax quantization of activations to
 *    int8 ("int8 dynamic quant + bsr support", pytorch/ao PR 821, title and
 *    description), with the absmax/127 symmetric scale that the Paddle
 *    "sparse_fc supported" PR (PaddlePaddle PR 41770, SpmmPluginDynamic
 *    constructor) computes for its int8 weight.  Scale and rounding are
 *    fixed as: s = fp32( max(absmax, 1e-8f) / 127 ), q = clamp(rint(x/s),
 *    -127, 127), round half to even, every operation one IEEE fp32 op.
 *  - The same formula per output channel for the weight (Paddle PR 41770,
 *    review of the plugin: a per-channel scale turns the GEMM alpha into a
 *    vector).
 *  - int8 x int8 -> int32 GEMM, exact integer accumulation (PR 821 review:
 *    the Triton dot product accumulates in int32, and its overflow bound of
 *    about 2^31 / 2^14 on K is worked out there).
 *  - The bf16 output epilogue out = bf16( acc * s_row * s_col + bias ),
 *    evaluated left to right in fp32 with round-to-nearest-even and no
 *    fused multiply-add; bf16 output is what keeps accuracy (PR 821,
 *    i8i8->bf16 eval vs i8i8->i8/32 eval).
 *  - The BSR (crow_indices / col_indices / values of 64x64 blocks) weight
 *    product (PR 821 description and the vit_h_14 --bsr 64 benchmark
 *    command), plus the pack / densify conversions between a dense int8
 *    weight and its BSR form.
 *  - Dynamic per-token FP8 (e4m3) quantization and the exact e4m3 product
 *    (vLLM csrc/quantization commits), and the weight-only int4 groupwise
 *    dequantization with its bf16 product ("Fused HQQ Quantization Gemm",
 *    pytorch/ao PR 153); their readings are stated beside each section.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fwrapv -fPIC
 * -shared (see oracle/build.py).  -ffp-contract=off forbids FMA contraction
 * so each fp32 multiply and add rounds on its own; -fwrapv makes an int32
 * overflow (which the int64 twin of the GEMM would expose) well defined.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is carried as its 16-bit pattern: the top half of an IEEE fp32. */
static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on the bit pattern.
 * NaN stays a (quiet) NaN; +-inf stays +-inf; an overflow rounds to inf. */
static uint16_t float_to_bf16_bits_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) {           /* inf or NaN */
        if (u & 0x007fffffu) return (uint16_t)((u >> 16) | 0x0040u);
        return (uint16_t)(u >> 16);
    }
    uint32_t keep_lsb = (u >> 16) & 1u;                /* ties go to even */
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

uint16_t oracle_float_to_bf16(float f) { return float_to_bf16_bits_rne(f); }
float oracle_bf16_to_float(uint16_t h) { return bf16_bits_to_float(h); }

/* ---- per-row symmetric absmax quantization (activations and weight) --- */

/* One row: absmax -> scale -> int8 codes.  `vals` already holds the row as
 * fp32 values (exact for bf16 input). */
static float quantize_one_row(const float* vals, int64_t K, int8_t* q) {
    float absmax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(vals[k]);
        if (a > absmax) absmax = a;
    }
    const float eps = 1e-8f;
    float clipped = absmax > eps ? absmax : eps;       /* max(absmax, 1e-8) */
    float scale = clipped / 127.0f;                    /* one IEEE division */
    for (int64_t k = 0; k < K; ++k) {
        float ratio = vals[k] / scale;                 /* true division, RN */
        float r = nearbyintf(ratio);                   /* ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[k] = (int8_t)r;
    }
    return scale;
}

/* x: bf16 bits [M, K], row stride ldx elements.  q: int8 [M, K], row
 * stride ldq.  scales: fp32 [M].  Returns 0, or -1 if a row is too long for
 * the scratch row (K > 1<<20). */
int oracle_quantize_rows_bf16(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                              int8_t* q, int64_t ldq, float* scales) {
    static float row[1 << 20];
    if (K > (1 << 20)) return -1;
    fesetround(FE_TONEAREST);
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t k = 0; k < K; ++k) row[k] = bf16_bits_to_float(x[i * ldx + k]);
        scales[i] = quantize_one_row(row, K, q + i * ldq);
    }
    return 0;
}

/* Weight preparation: fp32 [N, K] (nn.Linear layout, row n = output
 * channel n), per-output-channel symmetric int8.  Same formula per row. */
int oracle_quantize_rows_f32(const float* w, int64_t N, int64_t K, int64_t ldw,
                             int8_t* q, int64_t ldq, float* scales) {
    fesetround(FE_TONEAREST);
    for (int64_t n = 0; n < N; ++n)
        scales[n] = quantize_one_row(w + n * ldw, K, q + n * ldq);
    return 0;
}

/* ---- int8 GEMM, exact integer accumulation ----------------------------- */

/* acc[m, n] = sum_k A[m, k] * W[n, k]; A [M, K] ld lda, W [N, K] ld ldw,
 * acc int32 [M, N] row-major. */
void oracle_gemm_s32(const int8_t* A, int64_t M, int64_t K, int64_t lda,
                     const int8_t* W, int64_t N, int64_t ldw, int32_t* acc) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int32_t)A[m * lda + k] * (int32_t)W[n * ldw + k];
            acc[m * N + n] = s;
        }
}

/* Twin with int64 accumulation, for the brute-force overflow check. */
void oracle_gemm_s64(const int8_t* A, int64_t M, int64_t K, int64_t lda,
                     const int8_t* W, int64_t N, int64_t ldw, int64_t* acc) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)A[m * lda + k] * (int64_t)W[n * ldw + k];
            acc[m * N + n] = s;
        }
}

/* ---- epilogue: dequantize, bias, bf16 ----------------------------------- */

/* out[m, n] = bf16_rne( ((float)acc[m, n] * s_row[m]) * s_col[n] + bias[n] )
 * Left to right, each op one fp32 rounding.  bias == NULL means no addition
 * at all (not even +0.0). */
void oracle_epilogue_bf16(const int32_t* acc, int64_t M, int64_t N,
                          const float* s_row, const float* s_col,
                          const uint16_t* bias, uint16_t* out) {
    fesetround(FE_TONEAREST);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float f = (float)acc[m * N + n];
            f = f * s_row[m];
            f = f * s_col[n];
            if (bias) f = f + bf16_bits_to_float(bias[n]);
            out[m * N + n] = float_to_bf16_bits_rne(f);
        }
}

/* ---- block-sparse (BSR) weight ------------------------------------------ */

/* W in BSR form with bs x bs blocks over an [N, K] weight: block row b holds
 * output channels bs*b .. bs*b+bs-1; its blocks are p = crow[b] .. crow[b+1]-1,
 * block p sits at block column col[p] and its values are values[p][j][t]
 * (row j = channel, t = k offset, t contiguous).  Duplicate blocks add.
 * acc int32 [M, N] row-major. */
void oracle_bsr_gemm_s32(const int8_t* A, int64_t M, int64_t K, int64_t lda, int64_t N,
                         const int32_t* crow, const int32_t* col, const int8_t* values,
                         int64_t bs, int32_t* acc) {
    (void)K;
    memset(acc, 0, (size_t)(M * N) * sizeof(int32_t));
    const int64_t nbr = N / bs;
    for (int64_t b = 0; b < nbr; ++b)
        for (int64_t p = crow[b]; p < crow[b + 1]; ++p) {
            const int64_t c = col[p];
            const int8_t* blk = values + p * bs * bs;
            for (int64_t m = 0; m < M; ++m)
                for (int64_t j = 0; j < bs; ++j) {
                    int32_t s = 0;
                    for (int64_t t = 0; t < bs; ++t)
                        s += (int32_t)A[m * lda + c * bs + t] * (int32_t)blk[j * bs + t];
                    acc[m * N + b * bs + j] += s;
                }
        }
}

/* Dense int8 [N, K] -> BSR values for the given (crow, col) pattern:
 * values[p][j][t] = W[bs*b + j][bs*col[p] + t]. */
void oracle_bsr_pack(const int8_t* W, int64_t N, int64_t K, const int32_t* crow,
                     const int32_t* col, int64_t bs, int8_t* values) {
    const int64_t nbr = N / bs;
    for (int64_t b = 0; b < nbr; ++b)
        for (int64_t p = crow[b]; p < crow[b + 1]; ++p)
            for (int64_t j = 0; j < bs; ++j)
                for (int64_t t = 0; t < bs; ++t)
                    values[(p * bs + j) * bs + t] = W[(b * bs + j) * K + col[p] * bs + t];
}

/* BSR -> dense int32 [N, K] (int32 so that duplicate blocks can add
 * without wrapping); entries outside every block are 0. */
void oracle_bsr_densify(int64_t N, int64_t K, const int32_t* crow, const int32_t* col,
                        const int8_t* values, int64_t bs, int32_t* W) {
    memset(W, 0, (size_t)(N * K) * sizeof(int32_t));
    const int64_t nbr = N / bs;
    for (int64_t b = 0; b < nbr; ++b)
        for (int64_t p = crow[b]; p < crow[b + 1]; ++p)
            for (int64_t j = 0; j < bs; ++j)
                for (int64_t t = 0; t < bs; ++t)
                    W[(b * bs + j) * K + col[p] * bs + t] += values[(p * bs + j) * bs + t];
}

/* ---- dynamic FP8 (e4m3) per-token quantization and product ------------- */
/*
 * The sibling precision of the vLLM quantization commits (csrc/quantization
 * history: a vectorised FP8 quantize kernel; dynamic activation scales; the
 * scaled activations clamped to +-(largest e4m3 value) so that no NaN
 * appears), taken per token like the int8 path:
 *     s = fp32( max(absmax, 1e-8f) / 448 ),
 *     q = e4m3( clamp( fp32(x / s), -448, 448 ) ),
 * the conversion rounding to nearest, ties to even mantissa.  e4m3 ("fn"
 * variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal
 * values (1 + m/8) * 2^(e-7) for e = 1..15 except e = 15, m = 7 (NaN), so the
 * largest is 448 = 1.75 * 2^8; subnormals (m/8) * 2^-6; no infinities.
 */

/* e4m3 code -> its value (exact in double). NaN codes give NaN. */
double oracle_e4m3_to_double(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* finite fp32 -> e4m3, round to nearest, ties to even mantissa; magnitudes
 * at or above 448 give 448 (the clamp). */
uint8_t oracle_float_to_e4m3(float f) {
    const uint8_t sign = signbit(f) ? 0x80 : 0x00;
    const double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                       /* subnormal range: steps of 2^-9 */
        const double q = nearbyint(ldexp(a, 9));    /* 0 .. 8; 8 is the smallest normal */
        return sign | (uint8_t)q;
    }
    int e;
    (void)frexp(a, &e);                             /* a = fr * 2^e, fr in [0.5, 1) */
    int ex = e - 1;                                 /* a = (1 + f) * 2^ex, ex in -6 .. 8 */
    double mq = nearbyint((ldexp(a, -ex) - 1.0) * 8.0);   /* 0 .. 8, ties to even */
    if (mq == 8.0) { mq = 0.0; ex += 1; }
    int code = ((ex + 7) << 3) | (int)mq;
    if (code > 0x7E) code = 0x7E;
    return sign | (uint8_t)code;
}

static float quantize_one_row_fp8(const float* vals, int64_t K, uint8_t* q) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        const float a = fabsf(vals[k]);
        if (a > amax) amax = a;
    }
    const float s = fmaxf(amax, 1e-8f) / 448.0f;   /* one IEEE division */
    for (int64_t k = 0; k < K; ++k) {
        float v = vals[k] / s;                       /* one IEEE division */
        if (v > 448.0f) v = 448.0f;
        if (v < -448.0f) v = -448.0f;
        q[k] = oracle_float_to_e4m3(v);
    }
    return s;
}

int oracle_quantize_rows_bf16_fp8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scales) {
    fesetround(FE_TONEAREST);
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row) return -1;
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t k = 0; k < K; ++k) row[k] = bf16_bits_to_float(x[i * ldx + k]);
        scales[i] = quantize_one_row_fp8(row, K, q + i * ldq);
    }
    free(row);
    return 0;
}

int oracle_quantize_rows_f32_fp8(const float* w, int64_t N, int64_t K, int64_t ldw,
                                 uint8_t* q, int64_t ldq, float* scales) {
    fesetround(FE_TONEAREST);
    for (int64_t n = 0; n < N; ++n) scales[n] = quantize_one_row_fp8(w + n * ldw, K, q + n * ldq);
    return 0;
}

/* acc[m,n] = sum_k e4m3(A[m,k]) * e4m3(W[n,k]) in double.  Every product has
 * at most 8 significant bits and |products| lie in [2^-18, 2^17]; K <= 2^20
 * terms keep every partial sum within 53 bits, so the double sum is exact. */
void oracle_gemm_fp8_f64(const uint8_t* A, int64_t M, int64_t K, int64_t lda,
                         const uint8_t* W, int64_t N, int64_t ldw, double* acc) {
    double lut[256];
    for (int c = 0; c < 256; ++c) lut[c] = oracle_e4m3_to_double((uint8_t)c);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += lut[A[m * lda + k]] * lut[W[n * ldw + k]];
            acc[m * N + n] = s;
        }
}

/* ---- weight-only int4, asymmetric, groupwise (HQQ) ---------------------
 *
 * "Fused HQQ Quantization Gemm" (pytorch/ao PR 153), description and
 * implementation details: the weight of a linear layer is held as 4-bit
 * codes (u4: 0..15, or s4: -8..7), quantized along the in-features (K, axis 1
 * of the [N, K] weight) in groups of `group` consecutive values, each group
 * of each output channel with its own bf16 scale and zero point; the fused
 * kernel upcasts the codes to bf16, shifts them by the zero point and scales
 * them, then multiplies with the bf16 activations.  Two codes share one byte
 * (row interleave, no other preprocessing).
 *
 * Readings taken where the page is silent (each one stated here):
 *   - dequantized weight w = bf16( bf16(q - z) * s ): the zero point is
 *     subtracted first (the usual asymmetric definition, w = (q - z) * s) and
 *     each of the two operations rounds once to bf16, to nearest even, as a
 *     bf16 tensor expression does;
 *   - packing: byte j of row r holds code (r, 2j) in bits 0..3 and code
 *     (r, 2j + 1) in bits 4..7 (s4 codes as two's-complement nibbles), the
 *     packed rows stored [N, K/2] like the weight's own rows;
 *   - scales and zero points are [N, K/group] (channel, group), row-major;
 *   - the product is the plain bf16 matmul of activations and dequantized
 *     weight: out[m, n] = sum_k x[m, k] * w[n, k] (forward), and the
 *     transposed product out[m, k] = sum_n y[m, n] * w[n, k] used for the
 *     input gradient in the backward pass (the page's kernel serves both the
 *     forward and the backward orientation of the packed weight).
 */

/* Rounds a finite double to bf16 (8 significant bits), to nearest, ties to
 * even, in one step (no intermediate rounding to fp32); overflow gives inf. */
static uint16_t double_to_bf16_rne(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0x0000u;
    if (isnan(v)) return 0x7fc0u;
    if (isinf(v)) return v > 0 ? 0x7f80u : 0xff80u;
    int e = ilogb(v);                       /* |v| in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;                 /* subnormal bf16: fixed quantum 2^-133 */
    const double quantum = ldexp(1.0, e - 7);
    const double r = nearbyint(v / quantum) * quantum;   /* exact scaling by 2^k */
    if (fabs(r) >= ldexp(1.0, 128)) return v > 0 ? 0x7f80u : 0xff80u;
    const float f = (float)r;               /* r has <= 8 significant bits: exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

uint16_t oracle_double_to_bf16(double v) {
    fesetround(FE_TONEAREST);
    return double_to_bf16_rne(v);
}

/* codes [rows, cols] (cols even; u4 0..15 or s4 -8..7) -> packed [rows, cols/2]. */
void oracle_hqq_pack(const int8_t* codes, int64_t rows, int64_t cols, uint8_t* packed) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols / 2; ++j) {
            const uint8_t lo = (uint8_t)codes[r * cols + 2 * j] & 0x0fu;
            const uint8_t hi = (uint8_t)codes[r * cols + 2 * j + 1] & 0x0fu;
            packed[r * (cols / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
}

static int nibble_code(uint8_t nib, int is_signed) {
    return (is_signed && nib >= 8) ? (int)nib - 16 : (int)nib;
}

/* packed [rows, cols/2] -> codes [rows, cols]. */
void oracle_hqq_unpack(const uint8_t* packed, int64_t rows, int64_t cols, int is_signed, int8_t* codes) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < cols; ++k) {
            const uint8_t b = packed[r * (cols / 2) + k / 2];
            const uint8_t nib = (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0x0fu);
            codes[r * cols + k] = (int8_t)nibble_code(nib, is_signed);
        }
}

/* packed codes [N, K/2], scale / zero bf16 [N, K/group] -> w bf16 [N, K]:
 * w[n, k] = bf16( bf16(q[n, k] - z[n, g]) * s[n, g] ), g = k / group.
 * q - z is exact in double (an integer below 16 against 8 significant bits,
 * the bf16 inputs kept away from the far ends of the exponent range) and a
 * product of two bf16 values has at most 16 significant bits, so each
 * double_to_bf16_rne rounds the exact result once. */
void oracle_hqq_dequant(const uint8_t* packed, const uint16_t* scale, const uint16_t* zero,
                        int64_t N, int64_t K, int64_t group, int is_signed, uint16_t* w) {
    fesetround(FE_TONEAREST);
    const int64_t G = K / group;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            const uint8_t b = packed[n * (K / 2) + k / 2];
            const uint8_t nib = (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0x0fu);
            const double q = (double)nibble_code(nib, is_signed);
            const double z = (double)bf16_bits_to_float(zero[n * G + k / group]);
            const double s = (double)bf16_bits_to_float(scale[n * G + k / group]);
            const uint16_t t = double_to_bf16_rne(q - z);
            w[n * K + k] = double_to_bf16_rne((double)bf16_bits_to_float(t) * s);
        }
}

/* out[m, n] = sum_k x[m, k] * w[n, k] in double (x [M, K], w [N, K], bf16).
 * Each product of two bf16 values is exact in double; the sum rounds in
 * double, an error far below that of any fp32 accumulation. */
void oracle_hqq_linear_f64(const uint16_t* x, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                           double* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += (double)bf16_bits_to_float(x[m * K + k]) * (double)bf16_bits_to_float(w[n * K + k]);
            out[m * N + n] = s;
        }
}

/* Transposed product: out[m, k] = sum_n y[m, n] * w[n, k] (y [M, N], w [N, K]). */
void oracle_hqq_linear_t_f64(const uint16_t* y, const uint16_t* w, int64_t M, int64_t N, int64_t K,
                             double* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n)
                s += (double)bf16_bits_to_float(y[m * N + n]) * (double)bf16_bits_to_float(w[n * K + k]);
            out[m * K + k] = s;
        }
}

/* ---- 2:4 semi-structured sparse int8 weight -----------------------------
 *
 * "sparse_fc supported" (PaddlePaddle PR 41770, description and the
 * SpmmPluginDynamic review): fully connected layers whose weights are
 * already 2:4 sparse (at most two nonzeros in every group of four
 * consecutive in-features) run through a 2:4 sparse matmul after the weight
 * is compressed on the device; the quantized layer computes the same int8
 * product and dequantization as the dense one.  The compressed form is this
 * library's own (the page's comes from a closed library):
 *   values [N, K/2] int8: group g of row n keeps two values, values[2g] and
 *     values[2g+1], found at positions p0 < p1 (0..3) of the group;
 *   meta [N, K/8] uint8: byte b holds group 2b in bits 0..3 and group 2b+1
 *     in bits 4..7, each as p0 | p1 << 2.
 *   A group with fewer than two nonzeros keeps its nonzero positions and
 *   fills up with the lowest free positions (their values are zero).
 * The product itself is the plain int8 GEMM of the activations with the
 * decompressed weight (oracle_gemm_s32), then the same bf16 epilogue.
 */

/* Wq int8 [N, K] (K % 8 == 0) -> values, meta.  Returns the number of
 * groups with more than two nonzeros (those keep their two lowest nonzero
 * positions). */
int64_t oracle_s24_compress(const int8_t* W, int64_t N, int64_t K, int8_t* values, uint8_t* meta) {
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < K / 4; ++g) {
            const int8_t* grp = W + n * K + 4 * g;
            int pos[2];
            int cnt = 0, nz = 0;
            for (int j = 0; j < 4; ++j)
                if (grp[j] != 0) {
                    ++nz;
                    if (cnt < 2) pos[cnt++] = j;
                }
            if (nz > 2) ++bad;
            for (int j = 0; j < 4 && cnt < 2; ++j) {       /* fill with the lowest free positions */
                if (cnt == 1 && pos[0] == j) continue;
                if (grp[j] == 0) pos[cnt++] = j;
            }
            if (pos[0] > pos[1]) { const int t = pos[0]; pos[0] = pos[1]; pos[1] = t; }
            values[n * (K / 2) + 2 * g] = grp[pos[0]];
            values[n * (K / 2) + 2 * g + 1] = grp[pos[1]];
            const uint8_t nib = (uint8_t)(pos[0] | (pos[1] << 2));
            uint8_t* mb = meta + n * (K / 8) + g / 2;
            if (g % 2 == 0) *mb = (uint8_t)((*mb & 0xf0u) | nib);
            else *mb = (uint8_t)((*mb & 0x0fu) | (nib << 4));
        }
    }
    return bad;
}

/* values, meta -> Wq int8 [N, K] (zeros outside the kept positions; a
 * group whose two positions coincide adds both values there). */
void oracle_s24_decompress(const int8_t* values, const uint8_t* meta, int64_t N, int64_t K, int8_t* W) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint8_t mb = meta[n * (K / 8) + g / 2];
            const uint8_t nib = (g % 2 == 0) ? (uint8_t)(mb & 0x0fu) : (uint8_t)(mb >> 4);
            int8_t* grp = W + n * K + 4 * g;
            for (int j = 0; j < 4; ++j) grp[j] = 0;
            grp[nib & 3] = (int8_t)(grp[nib & 3] + values[n * (K / 2) + 2 * g]);
            grp[(nib >> 2) & 3] = (int8_t)(grp[(nib >> 2) & 3] + values[n * (K / 2) + 2 * g + 1]);
        }
}
