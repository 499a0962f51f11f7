/*
 * bitnet_ref.c -- the oracle: a plain, slow CPU implementation of the
 * BitNet b1.58 BitLinear forward (ternary weights, int8 activations).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load the library built from this file.  It
 * shares no code, header, table or constant with the CUDA library, and the
 * CUDA library never calls it.
 *
 * What it follows (web pages on BitNet b1.58; cited by title and section):
 *  [RR] "Microsoft BitNet 深度研究报告" (BitNet research report,
 *       conanxin.github.io), section "技术原理" (technical principles):
 *       item 2 "AbsMean 量化" gives Q(w) = round(clamp(w/gamma, -1, 1)) with
 *       gamma = (1/n) sum_i |w_i|, and the stored 2-bit value
 *       {0 -> 0, +1 -> 1, -1 -> 2}; item 3 "查找表优化" gives the
 *       add/subtract form of a ternary product (w=+1: C += A, w=0: nothing,
 *       w=-1: C -= A).
 *  [MC] "BitNet b1.58 2B4T" model card (model.aibase.cn), section "模型详情"
 *       (model details), "量化" (quantisation): absmean ternary weights in the
 *       forward pass; 8-bit integer activations by per-token absmax (W1.58A8);
 *       "架构": ReLU^2 in the FFN, no bias terms.
 *  [TR] tanhuajipinx.com write-up of the 2B4T technical report, section
 *       "GPU端：CUDA内核的定制魔法" (GPU: custom CUDA kernel): four ternary
 *       weights packed into one int8.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - gamma is summed in fp64: each row sequentially in k, then the row sums
 *    sequentially in n; gamma = (float)(sum / (N*K)).  gamma == 0 (an all-zero
 *    matrix) gives all-zero codes.  No epsilon is added.
 *  - "round" is round-half-away-from-zero (C99 roundf).
 *  - 4-per-byte layout: inside each group of 16 elements of a row, one
 *    little-endian 32-bit word holds element 16g + 4j + i at bits
 *    [8i + 2j, 8i + 2j + 2), i, j in 0..3.
 *  - per-token scale s = 127 / max|x| (fp32 division); xq = clamp(round(x*s),
 *    -127, 127); an all-zero row gives s = 1 and xq = 0.
 *  - y = (float)acc * (gamma / s) (fp32 division, then fp32 multiply);
 *    ReLU^2 is y = (y > 0 ? y : 0); y = y * y.  bf16 output rounds to
 *    nearest, ties to even.
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fPIC -shared [-fopenmp].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define REF_OK 0
#define REF_ERR_ARG 1
#define REF_ERR_RANGE 2     /* non-finite input, or 127/amax overflows */
#define REF_ERR_CODE 3      /* unpacking met the never-written code 3   */
#define REF_ERR_OVERFLOW 4  /* accumulator outside int32                */

/* ------------------------------------------------------------ weights */

/* gamma = (1/n) sum |w|, [RR] item 2.  Fixed order, fp64. */
float ref_absmean_gamma(const float *W, int64_t N, int64_t K)
{
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double row = 0.0;
        for (int64_t k = 0; k < K; ++k)
            row += fabs((double)W[n * K + k]);
        total += row;
    }
    return (float)(total / (double)(N * K));
}

/* Q(w) = round(clamp(w / gamma, -1, 1)) in {-1, 0, +1}, [RR] item 2. */
int ref_ternary(float w, float gamma)
{
    if (gamma == 0.0f)
        return 0;
    float t = w / gamma;
    if (t < -1.0f) t = -1.0f;
    if (t > 1.0f) t = 1.0f;
    return (int)roundf(t);
}

/* Stored 2-bit value {0 -> 0, +1 -> 1, -1 -> 2}, [RR] item 2. */
unsigned ref_code_of(int q)
{
    return q == 0 ? 0u : (q > 0 ? 1u : 2u);
}

/* Inverse of ref_code_of; -2 for the code 3, which is never written. */
int ref_value_of(unsigned code)
{
    switch (code) {
    case 0: return 0;
    case 1: return 1;
    case 2: return -1;
    default: return -2;
    }
}

/* Bit position of element e (0..15) of a 16-element group inside its word. */
static int ref_bitpos(int e)
{
    int i = e % 4, j = e / 4;
    return 8 * i + 2 * j;
}

/* Pack one row of K codes (K % 16 == 0) into K/4 bytes, [TR]: 4 per byte. */
void ref_pack_row(const uint8_t *codes, int64_t K, uint8_t *out)
{
    for (int64_t g = 0; g < K / 16; ++g) {
        uint32_t word = 0;
        for (int e = 0; e < 16; ++e)
            word |= (uint32_t)(codes[16 * g + e] & 3u) << ref_bitpos(e);
        for (int b = 0; b < 4; ++b)
            out[4 * g + b] = (uint8_t)(word >> (8 * b));
    }
}

/* Code of element k of a packed row. */
unsigned ref_unpack_code(const uint8_t *packed_row, int64_t k)
{
    int64_t g = k / 16;
    int e = (int)(k % 16);
    int pos = ref_bitpos(e);
    return (packed_row[4 * g + pos / 8] >> (pos % 8)) & 3u;
}

/* Whole weight path: gamma, codes, packing.  packed is [N][K/4]. */
int ref_quantize_weights(const float *W, int64_t N, int64_t K, uint8_t *packed, float *gamma_out)
{
    if (N <= 0 || K <= 0 || K % 16 != 0)
        return REF_ERR_ARG;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i]))
            return REF_ERR_RANGE;
    float gamma = ref_absmean_gamma(W, N, K);
    uint8_t *codes = (uint8_t *)malloc((size_t)K);
    if (!codes)
        return REF_ERR_ARG;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k)
            codes[k] = (uint8_t)ref_code_of(ref_ternary(W[n * K + k], gamma));
        ref_pack_row(codes, K, packed + n * (K / 4));
    }
    free(codes);
    *gamma_out = gamma;
    return REF_OK;
}

/* Ternary values [N][K] of a packed matrix; REF_ERR_CODE on a code 3. */
int ref_unpack_weights(const uint8_t *packed, int64_t N, int64_t K, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int v = ref_value_of(ref_unpack_code(packed + n * (K / 4), k));
            if (v == -2)
                return REF_ERR_CODE;
            q[n * K + k] = (int8_t)v;
        }
    return REF_OK;
}

/* ------------------------------------------------------------ activations */

/* Per-token absmax int8, [MC] "量化": s_m = 127 / max_k |x_mk|. */
int ref_quantize_act(const float *X, int64_t M, int64_t K, int8_t *xq, float *s)
{
    if (M < 0 || K <= 0)
        return REF_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const float *x = X + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(x[k]))
                return REF_ERR_RANGE;
            float a = fabsf(x[k]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            s[m] = 1.0f;
            for (int64_t k = 0; k < K; ++k)
                xq[m * K + k] = 0;
            continue;
        }
        float sm = 127.0f / amax;
        if (!isfinite(sm))
            return REF_ERR_RANGE;
        s[m] = sm;
        for (int64_t k = 0; k < K; ++k) {
            float v = x[k] * sm;
            float r = roundf(v);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            xq[m * K + k] = (int8_t)r;
        }
    }
    return REF_OK;
}

/* ------------------------------------------------------------ contraction */

/* acc[m][n] = sum_k xq[m][k] * Q(W)[n][k], exact (int64, then range check). */
int ref_matmul_acc(const int8_t *xq, const uint8_t *packed, int64_t M, int64_t N, int64_t K,
                   int32_t *acc)
{
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0)
        return REF_ERR_ARG;
    int bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) reduction(| : bad)
#endif
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = packed + n * (K / 4);
        for (int64_t m = 0; m < M; ++m) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k) {
                int v = ref_value_of(ref_unpack_code(row, k));
                if (v == -2) { bad |= 1; v = 0; }
                sum += (int64_t)xq[m * K + k] * v;
            }
            if (sum > INT32_MAX || sum < INT32_MIN) { bad |= 2; sum = 0; }
            acc[m * N + n] = (int32_t)sum;
        }
    }
    if (bad & 1) return REF_ERR_CODE;
    if (bad & 2) return REF_ERR_OVERFLOW;
    return REF_OK;
}

/* ------------------------------------------------------------ epilogue */

/* y = (float)acc * (gamma / s_m); optional ReLU^2 ([MC] "架构"; no bias). */
void ref_epilogue(const int32_t *acc, const float *s, float gamma, int64_t M, int64_t N,
                  int relu2, float *y)
{
    for (int64_t m = 0; m < M; ++m) {
        float r = gamma / s[m];
        for (int64_t n = 0; n < N; ++n) {
            float v = (float)acc[m * N + n] * r;
            if (relu2) {
                v = v > 0.0f ? v : 0.0f;
                v = v * v;
            }
            y[m * N + n] = v;
        }
    }
}

/* fp32 -> bf16 bits, round to nearest, ties to even (NaN stays NaN). */
uint16_t ref_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void ref_to_bf16(const float *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ref_bf16_bits(y[i]);
}

/* Whole BitLinear forward: act quant -> int32 contraction -> rescale. */
int ref_bitlinear(const float *X, int64_t M, int64_t K, const uint8_t *packed, float gamma,
                  int64_t N, int relu2, int8_t *xq, float *s, int32_t *acc, float *y)
{
    int st = ref_quantize_act(X, M, K, xq, s);
    if (st != REF_OK)
        return st;
    st = ref_matmul_acc(xq, packed, M, N, K, acc);
    if (st != REF_OK)
        return st;
    ref_epilogue(acc, s, gamma, M, N, relu2, y);
    return REF_OK;
}

/* Per-token RMS normalisation x / sqrt(mean(x^2) + 1e-6), fp32: the weightless
 * stand-in for the model card's "subln" between chained BitLinears (the pages
 * give no formula).  Not part of the bit-exact BitLinear contract. */
void ref_rms_norm(const float *X, int64_t M, int64_t K, float *Y)
{
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k)
            ss += (double)X[m * K + k] * (double)X[m * K + k];
        float inv = (float)(1.0 / sqrt(ss / (double)K + 1e-6));
        for (int64_t k = 0; k < K; ++k)
            Y[m * K + k] = X[m * K + k] * inv;
    }
}

/* Threads the parallel loop above will use (1 without OpenMP). */
int ref_num_threads(void)
{
#ifdef _OPENMP
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
#else
    return 1;
#endif
}
