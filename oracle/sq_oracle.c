/*
 * CPU oracle for the W8A8 quantized linear layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The product path
 * (the CUDA library and its Python binding) never calls it, and the two share
 * no code: this file includes only the C standard library.
 *
 * Every function is the plain definition written out with scalar loops in IEEE
 * single precision (compiled with -ffp-contract=off, no fast-math), with int64
 * integer sums and fp64 for the reference outputs. OpenMP splits work over
 * independent rows or columns only; each output element is produced by one
 * thread in a fixed order, so results do not depend on the thread count.
 *
 * Pages cited (by title):
 *   [BASICS]  "量化基础与INT8" (quantization fundamentals and INT8)
 *   [LLMINT8] "LLM.int8()技术解析：8位量化如何优化大语言模型计算"
 *   [SQ]      "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地"
 *
 * Readings of the pages that the code takes (where they are silent or differ):
 *   - quantize by multiplying with a once-per-row fp32 reciprocal r = 127/absmax
 *     ([LLMINT8] §2.2 quantize), dequant scale d = absmax/127 ([BASICS] symmetric
 *     quantization), clamp to [-128,127] ([BASICS] quantization-flow example);
 *   - round half to even (torch.round in [BASICS] quantization-flow example);
 *   - absmax == 0 gives r = 0, codes 0 and scale 0;
 *   - smoothed values x*inv_s and w*s stay in fp32, never rounded to 16 bits;
 *   - the smoothing factor is s_j = max(a_j,1e-8)^alpha / max(w_j,1e-8)^(1-alpha)
 *     evaluated in fp64 with pow() and rounded once to fp32, inv_s_j = 1/s_j in
 *     fp32 ([SQ] §2.1 formula, §3.3 clamps); the s/s.max()*127 normalisation of
 *     [SQ] §3.3 is not applied;
 *   - LLM.int8: outlier columns are those whose column absmax is strictly greater
 *     than the threshold; the activation row scale is taken over the other
 *     columns only and the outlier columns get code 0; the outlier product uses
 *     the original bf16 values ([LLMINT8] §2.1, §3.1).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PER_TENSOR 0
#define ORACLE_PER_CHANNEL 1

static float bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round-to-nearest-even from fp32 to bf16 (the definition of the rounding on
 * the bit pattern: add half an ulp of bf16 plus the tie-break bit, truncate). */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* q = clamp(round_half_even(v), -128, 127). */
static int8_t round_clamp_int8(float v) {
    float r = nearbyintf(v); /* default FE_TONEAREST: ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -128.0f) r = -128.0f;
    return (int8_t)r;
}

/* Per-column absmax of X [M,K] (leading dimension ldx):
 * amax_j = max_m |X[m,j]|, or max(amax_j, .) when accumulate != 0.
 * [SQ] §3.2 calibration hook (x.abs().amax over the token dims, running maximum
 * across batches); [LLMINT8] §2.1 step 1 (column-wise absolute maximum). */
void oracle_act_channel_absmax(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                               float *amax, int accumulate) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        float m = accumulate ? amax[j] : 0.0f;
        for (int64_t i = 0; i < M; ++i) {
            float a = fabsf(bf16_to_float(X[i * ldx + j]));
            if (a > m) m = a;
        }
        amax[j] = m;
    }
}

/* Smoothing factor, [SQ] §2.1 and §3.3:
 *   wmax_j = max_n |W[n,j]|   (W is [out=N, in=K]; the max runs over output rows)
 *   s_j    = max(amax_j,1e-8)^alpha / max(wmax_j,1e-8)^(1-alpha)
 *   inv_s_j = 1 / s_j */
void oracle_smooth_scale(const float *act_amax, const uint16_t *W, int64_t N, int64_t K,
                         int64_t ldw, float alpha, float *s, float *inv_s) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        float wmax = 0.0f;
        for (int64_t n = 0; n < N; ++n) {
            float a = fabsf(bf16_to_float(W[n * ldw + j]));
            if (a > wmax) wmax = a;
        }
        float a_cl = act_amax[j] > 1e-8f ? act_amax[j] : 1e-8f;
        float w_cl = wmax > 1e-8f ? wmax : 1e-8f;
        double num = pow((double)a_cl, (double)alpha);
        double den = pow((double)w_cl, 1.0 - (double)alpha);
        float sj = (float)(num / den);
        s[j] = sj;
        inv_s[j] = 1.0f / sj;
    }
}

/* Symmetric absmax quantization of one row of n fp32 values already smoothed.
 * r = 127/a (fp32 divide), q = clamp(rne(v*r)), d = a/127. */
static void quantize_with_absmax(const float *v, int64_t n, float a, int8_t *q) {
    float r = (a > 0.0f) ? 127.0f / a : 0.0f;
    for (int64_t k = 0; k < n; ++k) {
        float p = v[k] * r;
        q[k] = round_clamp_int8(p);
    }
}

/* Weight smoothing + quantization, [BASICS] per-tensor / per-channel granularity
 * and quantization-flow example (W_scale = max|W|/127, W_int8 =
 * round(W/W_scale).clamp(-128,127)); [SQ] §3.3 (W' = W * s broadcast over the
 * input dimension) and §3.4 (w_scale = w_max/127).
 *   w'_{nk} = W[n,k] * s_k  (fp32; s == NULL means s_k = 1)
 *   per-channel: a_n = max_k |w'_{nk}|, e_n = a_n/127, q = clamp(rne(w' * (127/a_n)))
 *   per-tensor : a   = max_{n,k} |w'|,  e_0 = a/127,   likewise. */
void oracle_smooth_quant_weight(const uint16_t *W, int64_t N, int64_t K, int64_t ldw,
                                const float *s, int gran, int8_t *Wq, float *w_scale) {
    float *wp = (float *)malloc(sizeof(float) * (size_t)N * (size_t)K);
    float *rowmax = (float *)malloc(sizeof(float) * (size_t)N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float w = bf16_to_float(W[n * ldw + k]);
            float v = s ? w * s[k] : w;
            wp[n * K + k] = v;
            float a = fabsf(v);
            if (a > m) m = a;
        }
        rowmax[n] = m;
    }
    if (gran == ORACLE_PER_TENSOR) {
        float a = 0.0f;
        for (int64_t n = 0; n < N; ++n)
            if (rowmax[n] > a) a = rowmax[n];
        w_scale[0] = a / 127.0f;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) quantize_with_absmax(wp + n * K, K, a, Wq + n * K);
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            w_scale[n] = rowmax[n] / 127.0f;
            quantize_with_absmax(wp + n * K, K, rowmax[n], Wq + n * K);
        }
    }
    free(rowmax);
    free(wp);
}

/* Per-token dynamic activation quantization, [BASICS] per-token granularity and
 * quantization-flow example (X_scale = X.abs().max(dim=-1)/127); [SQ] §3.4
 * (x = x / scale before quantizing, here as x * inv_s).
 *   x'_{mk} = X[m,k] * inv_s_k  (inv_s == NULL means 1)
 *   a_m = max over k not in skip of |x'_{mk}|, d_m = a_m/127,
 *   q_{mk} = clamp(rne(x'_{mk} * (127/a_m))), and q = 0 where bit k of skip is set.
 * skip (NULL or ceil(K/32) words, bit k%32 of word k/32) marks LLM.int8 outlier
 * columns ([LLMINT8] §2.1 step 3: outlier columns are handled apart). */
void oracle_quant_act_per_token(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                const float *inv_s, const uint32_t *skip, int8_t *Xq,
                                float *x_scale) {
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            float a = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float x = bf16_to_float(X[m * ldx + k]);
                v[k] = inv_s ? x * inv_s[k] : x;
                int skipped = skip && ((skip[k >> 5] >> (k & 31)) & 1u);
                if (skipped) {
                    v[k] = 0.0f;
                    continue;
                }
                float ab = fabsf(v[k]);
                if (ab > a) a = ab;
            }
            x_scale[m] = a / 127.0f;
            quantize_with_absmax(v, K, a, Xq + m * K);
        }
        free(v);
    }
}

/* INT8 x INT8 -> INT32 GEMM, [BASICS] INT8 inference flow ("(M,K) x (K,N) ->
 * INT32 accumulate") and quantization-flow example (F.linear(X_int8, W_int8)):
 *   acc_{mn} = sum_k Xq[m,k] * Wq[n,k]   (both K-contiguous, Wq is [N,K])
 * Summed in int64; returns the number of sums that do not fit int32 (0 expected). */
int64_t oracle_int8_gemm(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                         int32_t *acc) {
    int64_t overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t t = 0;
            const int8_t *xr = Xq + m * K;
            const int8_t *wr = Wq + n * K;
            for (int64_t k = 0; k < K; ++k) t += (int64_t)xr[k] * (int64_t)wr[k];
            if (t > INT32_MAX || t < INT32_MIN) ++overflow;
            acc[m * N + n] = (int32_t)t;
        }
    }
    return overflow;
}

/* Dequantization, [BASICS] quantization-flow example (Y = Y_int32 * X_scale *
 * W_scale) and [SQ] §3.4 (out * (x_scale * w_scale), then + bias; bias stays in
 * floating point, [SQ] §4.5 first detail):
 *   y_ref_{mn} = acc_{mn} * d_m * e_n + o_{mn} + bias_n   (fp64, not rounded)
 *   y_bf16_{mn} = bf16_rne( ((float)acc * d_m) * e_n + (float)o_{mn} + bias_n )  (fp32 sequence)
 * e has N entries when e_per_channel, else 1; o (fp64 [M,N]) and bias may be NULL. */
void oracle_dequant(const int32_t *acc, int64_t M, int64_t N, const float *d, const float *e,
                    int e_per_channel, const uint16_t *bias, const double *o, double *y_ref,
                    uint16_t *y_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float en = e_per_channel ? e[n] : e[0];
            float bn = bias ? bf16_to_float(bias[n]) : 0.0f;
            double on = o ? o[m * N + n] : 0.0;
            int32_t a = acc[m * N + n];
            if (y_ref) y_ref[m * N + n] = (double)a * (double)d[m] * (double)en + on + (double)bn;
            if (y_bf16) {
                float y = ((float)a * d[m]) * en;
                y = y + (float)on;
                y = y + bn;
                y_bf16[m * N + n] = float_to_bf16_rne(y);
            }
        }
    }
}

/* LLM.int8 outlier columns, [LLMINT8] §2.1 steps 1-2 and §3.1 real-time
 * detection (column max over threshold, marked in a bitmask):
 *   O = { j : amax_j > threshold }; mask bit j%32 of word j/32; idx = O ascending.
 * Returns |O| (also written to *count when count != NULL). */
int32_t oracle_outlier_columns(const float *amax, int64_t K, float threshold, uint32_t *mask,
                               int32_t *idx, int32_t *count) {
    int64_t words = (K + 31) / 32;
    for (int64_t w = 0; w < words; ++w) mask[w] = 0u;
    int32_t c = 0;
    for (int64_t j = 0; j < K; ++j) {
        if (amax[j] > threshold) {
            mask[j >> 5] |= 1u << (j & 31);
            if (idx) idx[c] = (int32_t)j;
            ++c;
        }
    }
    if (count) *count = c;
    return c;
}

/* LLM.int8 outlier product, [LLMINT8] §3.1 mixed computation (outlier columns go
 * through a 16-bit GEMM): o_{mn} = sum_{j in idx} X[m,j] * W[n,j], in fp64 over
 * the original bf16 values, j in ascending order. */
void oracle_outlier_product(const uint16_t *X, int64_t ldx, const uint16_t *W, int64_t ldw,
                            int64_t M, int64_t N, const int32_t *idx, int32_t count, double *o) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double t = 0.0;
            for (int32_t c = 0; c < count; ++c) {
                int64_t j = idx[c];
                t += (double)bf16_to_float(X[m * ldx + j]) * (double)bf16_to_float(W[n * ldw + j]);
            }
            o[m * N + n] = t;
        }
    }
}

/* Widen bf16 bits to fp32 and round fp32 to bf16 (exposed for the oracle's own
 * tests of its conversions). */
void oracle_bf16_to_float(const uint16_t *b, int64_t n, float *f) {
    for (int64_t i = 0; i < n; ++i) f[i] = bf16_to_float(b[i]);
}

void oracle_float_to_bf16(const float *f, int64_t n, uint16_t *b) {
    for (int64_t i = 0; i < n; ++i) b[i] = float_to_bf16_rne(f[i]);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
