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
 *   [QAT]     "从自动驾驶芯片到大语言模型INT8量化训练实战解析" (mean + 3 std outliers)
 *   [PREC]    "大语言模型轻量化与量化精度" (choosing quantization precision; §3.2 calibration)
 *
 * Readings of the pages that the code takes (where they are silent or differ):
 *   - quantize by multiplying with a once-per-row fp32 reciprocal r = 127/absmax
 *     ([LLMINT8] §2.2 quantize), dequant scale d = absmax/127 ([BASICS] symmetric
 *     quantization), clamp to [-128,127] ([BASICS] quantization-flow example);
 *   - round half to even (the rounding of the [BASICS] quantization-flow example);
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
 *
 * Variants (functions after oracle_outlier_product), readings:
 *   - per-tensor activation scale ([SQ] §3.4 forward: x_max over the whole tensor),
 *     or a given clip value (static calibration), codes saturate by the clamp;
 *   - normalisation s <- max(s / max_j s_j * 127, 1e-5) of [SQ] §3.3, in fp32 in
 *     that order, inv_s = 1/s;
 *   - fused normalisation before smoothing ([SQ] §4.2, §4.5 second detail: the
 *     smoothing folds into the LayerNorm output): row statistics summed in fp64
 *     and rounded once to fp32 (mean, 1/sqrt(var + eps)), then
 *     y = ((x - mean) * rstd) * gamma + beta in fp32 (RMSNorm: y = (x * rstd) * gamma),
 *     x' = y * inv_s, then per-token quantization as above;
 *   - dynamic outlier threshold mu + k*sigma over all elements of X ([LLMINT8]
 *     §3.1 pre-screening, [QAT] §2.1), mean and unbiased standard deviation in
 *     fp64, threshold rounded once to fp32;
 *   - percentile calibration ([PREC] §3.2): nearest-rank percentile of |X|
 *     over all elements, rank = ceil(p/100 * n) (at least 1);
 *   - asymmetric per-token activations ([BASICS] asymmetric quantization) over
 *     the range [min(0, min x'), max(0, max x')] so that 0 is exact:
 *     r = 255/range, d = range/255, z = -128 - rne(lo * r),
 *     q = clamp(rne(x' * r) + z, -128, 127), x' ~ d * (q - z); the GEMM result is
 *     corrected exactly in integers: acc - z_m * sum_k Wq[n,k].
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
 * [SQ] §3.2 calibration hook (each input channel's absolute maximum over the token
 * dimensions, running maximum across batches); [LLMINT8] §2.1 step 1 (column-wise
 * absolute maximum). */
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
 * and quantization-flow example (the scale is the absolute maximum over 127; codes are
 * rounded and clamped to [-128, 127]); [SQ] §3.3 (each input channel of the weight
 * multiplied by its s) and §3.4 (weight scale = weight maximum over 127).
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
 * quantization-flow example (each token row's scale is its absolute maximum over 127);
 * [SQ] §3.4 (activations divided by s before quantizing, here as x * inv_s).
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

/* ------------------------------------------------------------------ variants */

/* Per-tensor activation quantization, [SQ] §3.4 (the reference module's activation scale is one
 * maximum over the whole tensor, divided by 127; codes rounded half to even and clamped):
 *   x' = X * inv_s (inv_s NULL: 1); a = clip if clip >= 0 (static calibration, e.g. a
 *   percentile), else max over all |x'|; x_scale[0] = a/127; q = clamp(rne(x' * (127/a))). */
void oracle_quant_act_per_tensor(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                 const float *inv_s, float clip, int8_t *Xq, float *x_scale) {
    float a = clip;
    if (!(clip >= 0.0f)) {
        a = 0.0f;
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = 0; k < K; ++k) {
                float x = bf16_to_float(X[m * ldx + k]);
                float v = inv_s ? x * inv_s[k] : x;
                if (fabsf(v) > a) a = fabsf(v);
            }
    }
    x_scale[0] = a / 127.0f;
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            for (int64_t k = 0; k < K; ++k) {
                float x = bf16_to_float(X[m * ldx + k]);
                v[k] = inv_s ? x * inv_s[k] : x;
            }
            quantize_with_absmax(v, K, a, Xq + m * K);
        }
        free(v);
    }
}

/* Normalisation of the smoothing factors, [SQ] §3.3 compute_smooth_scale:
 *   s_j <- s_j / max_i s_i * 127 (fp32, in that order); s_j <- max(s_j, 1e-5); inv_s_j = 1/s_j. */
void oracle_smooth_scale_normalize(float *s, float *inv_s, int64_t K) {
    float smax = 0.0f;
    for (int64_t j = 0; j < K; ++j)
        if (s[j] > smax) smax = s[j];
    for (int64_t j = 0; j < K; ++j) {
        float t = (s[j] / smax) * 127.0f;
        if (t < 1e-5f) t = 1e-5f;
        s[j] = t;
        inv_s[j] = 1.0f / t;
    }
}

#define ORACLE_NORM_LAYER 0
#define ORACLE_NORM_RMS 1

/* Normalisation + smoothing + per-token quantization of one fused pass, [SQ] §4.2 and
 * §4.5 second detail (the smoothing folds into the LayerNorm output). Per row m:
 *   LayerNorm: mean = sum x / K, var = sum (x - mean)^2 / K (fp64, mean from the fp64 sum);
 *              mean_f = fp32(mean), rstd_f = fp32(1 / sqrt(var + eps));
 *              y = ((x - mean_f) * rstd_f) * gamma_k + beta_k            (fp32, beta NULL: 0)
 *   RMSNorm:   ms = sum x^2 / K (fp64); rstd_f = fp32(1 / sqrt(ms + eps));
 *              y = (x * rstd_f) * gamma_k + beta_k                       (fp32, beta NULL: 0)
 *   x' = y * inv_s_k (inv_s NULL: 1); a = max |x'|; d_m = a/127; q = clamp(rne(x' * (127/a))).
 * gamma, beta are bf16 [K]. stats [M,2] (mean_f or 0 for RMSNorm, rstd_f) receives the row
 * statistics, or, with stats_given, supplies them: fp64 sums in another order may round
 * to a neighbouring fp32 value, so the steps after the statistics can be checked on the
 * statistics another implementation produced. */
void oracle_norm_smooth_quant(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, int norm,
                              const uint16_t *gamma, const uint16_t *beta, float eps,
                              const float *inv_s, int8_t *Xq, float *x_scale, float *y_out,
                              float *stats, int stats_given) {
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            const uint16_t *xr = X + m * ldx;
            float mean_f = 0.0f, rstd_f;
            if (stats && stats_given) {
                mean_f = stats[2 * m];
                rstd_f = stats[2 * m + 1];
            } else if (norm == ORACLE_NORM_LAYER) {
                double sum = 0.0;
                for (int64_t k = 0; k < K; ++k) sum += (double)bf16_to_float(xr[k]);
                double mean = sum / (double)K;
                double ss = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double c = (double)bf16_to_float(xr[k]) - mean;
                    ss += c * c;
                }
                double var = ss / (double)K;
                mean_f = (float)mean;
                rstd_f = (float)(1.0 / sqrt(var + (double)eps));
            } else {
                double ss = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double x = (double)bf16_to_float(xr[k]);
                    ss += x * x;
                }
                rstd_f = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
            }
            if (stats && !stats_given) {
                stats[2 * m] = mean_f;
                stats[2 * m + 1] = rstd_f;
            }
            float a = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float x = bf16_to_float(xr[k]);
                float y = (norm == ORACLE_NORM_LAYER) ? (x - mean_f) * rstd_f : x * rstd_f;
                y = y * bf16_to_float(gamma[k]);
                if (beta) y = y + bf16_to_float(beta[k]);
                if (y_out) y_out[m * K + k] = y;
                v[k] = inv_s ? y * inv_s[k] : y;
                if (fabsf(v[k]) > a) a = fabsf(v[k]);
            }
            x_scale[m] = a / 127.0f;
            quantize_with_absmax(v, K, a, Xq + m * K);
        }
        free(v);
    }
}

/* Dynamic outlier threshold, [LLMINT8] §3.1 pre-screening (threshold = mu + 6 sigma from
 * the layer's activation mean and variance) and [QAT] §2.1 (mean + 3 std of all elements,
 * torch's unbiased std): mean and std over all M*K elements in fp64 (two passes), the
 * threshold mean + k*std rounded once to fp32. Writes mean and std when non-NULL. */
float oracle_mean_std_threshold(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, double k,
                                double *mean_out, double *std_out) {
    double n = (double)M * (double)K;
    double sum = 0.0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < K; ++j) sum += (double)bf16_to_float(X[m * ldx + j]);
    double mean = sum / n;
    double ss = 0.0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < K; ++j) {
            double c = (double)bf16_to_float(X[m * ldx + j]) - mean;
            ss += c * c;
        }
    double sd = n > 1.0 ? sqrt(ss / (n - 1.0)) : 0.0;
    if (mean_out) *mean_out = mean;
    if (std_out) *std_out = sd;
    return (float)(mean + k * sd);
}

static int cmp_float(const void *a, const void *b) {
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

/* Percentile calibration, [PREC] §3.2 (a max calibrator with the percentile method,
 * 99.99): the nearest-rank p-th percentile of |X| over all M*K elements: sort the absolute
 * values ascending and take the element of 1-based rank ceil(p/100 * n), at least 1. */
float oracle_abs_percentile(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, double p) {
    int64_t n = M * K;
    float *v = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < K; ++j) v[m * K + j] = fabsf(bf16_to_float(X[m * ldx + j]));
    qsort(v, (size_t)n, sizeof(float), cmp_float);
    int64_t rank = (int64_t)ceil((p / 100.0) * (double)n);
    if (rank < 1) rank = 1;
    if (rank > n) rank = n;
    float r = v[rank - 1];
    free(v);
    return r;
}

/* Asymmetric per-token activation quantization, [BASICS] asymmetric quantization
 * (scale = (max - min)/255 with a zero point), on signed 8-bit codes, over the range
 * extended to contain 0:
 *   x' = X * inv_s; lo = min(0, min_k x'), hi = max(0, max_k x'); range = hi - lo (fp32);
 *   r = range > 0 ? 255/range : 0; d_m = range/255; z_m = -128 - rne(lo * r);
 *   q = clamp(rne(x' * r) + z_m, -128, 127);  x' ~ d_m * (q - z_m). */
void oracle_quant_act_per_token_asym(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                     const float *inv_s, int8_t *Xq, float *x_scale,
                                     int32_t *x_zero) {
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            float lo = 0.0f, hi = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float x = bf16_to_float(X[m * ldx + k]);
                v[k] = inv_s ? x * inv_s[k] : x;
                if (v[k] < lo) lo = v[k];
                if (v[k] > hi) hi = v[k];
            }
            float range = hi - lo;
            float r = range > 0.0f ? 255.0f / range : 0.0f;
            int32_t z = -128 - (int32_t)nearbyintf(lo * r);
            x_scale[m] = range / 255.0f;
            x_zero[m] = z;
            for (int64_t k = 0; k < K; ++k) {
                float t = nearbyintf(v[k] * r) + (float)z;
                if (t > 127.0f) t = 127.0f;
                if (t < -128.0f) t = -128.0f;
                Xq[m * K + k] = (int8_t)t;
            }
        }
        free(v);
    }
}

/* Row sums of the int8 weight, rs_n = sum_k Wq[n,k] (the zero-point correction term of an
 * asymmetric activation: sum_k (q - z) w = sum_k q w - z * rs_n). */
void oracle_weight_row_sums(const int8_t *Wq, int64_t N, int64_t K, int32_t *rs) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        int64_t t = 0;
        for (int64_t k = 0; k < K; ++k) t += Wq[n * K + k];
        rs[n] = (int32_t)t;
    }
}

/* Dequantization with the variants' operands: d per token ([M]) or per tensor ([1]),
 * e per channel ([N]) or per tensor ([1]); with x_zero (int32 [M]) and rs (int32 [N])
 * the accumulator is first corrected exactly, a = acc - z_m * rs_n (int64):
 *   y_ref = a * d * e + bias (fp64), y_bf16 = bf16_rne(((float)a * d) * e + bias). */
void oracle_dequant_ex(const int32_t *acc, int64_t M, int64_t N, const float *d, int d_per_token,
                       const float *e, int e_per_channel, const int32_t *x_zero, const int32_t *rs,
                       const uint16_t *bias, double *y_ref, uint16_t *y_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float dm = d_per_token ? d[m] : d[0];
            float en = e_per_channel ? e[n] : e[0];
            float bn = bias ? bf16_to_float(bias[n]) : 0.0f;
            int64_t a = acc[m * N + n];
            if (x_zero) a -= (int64_t)x_zero[m] * (int64_t)rs[n];
            if (y_ref) y_ref[m * N + n] = (double)a * (double)dm * (double)en + (double)bn;
            if (y_bf16) {
                float y = ((float)a * dm) * en;
                y = y + bn;
                y_bf16[m * N + n] = float_to_bf16_rne(y);
            }
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
