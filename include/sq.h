/*
 * sq.h — C ABI of libsq: a W8A8 INT8 quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes Y = dequant( int8(X * diag(s)^-1) . int8(diag(s) * W)^T ) + bias
 * (SmoothQuant smoothing, symmetric absmax INT8 quantization, INT8 x INT8 -> INT32
 * accumulation, per-token x per-channel/per-tensor dequantization), and the
 * LLM.int8() decomposition in which activation columns whose absmax exceeds a
 * threshold go through a bf16 product that is added back.
 *
 * Pages the operations follow (cited by title and section):
 *   [BASICS]  "量化基础与INT8" (quantization fundamentals and INT8)
 *   [LLMINT8] "LLM.int8()技术解析：8位量化如何优化大语言模型计算"
 *   [SQ]      "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地"
 *   [QAT]     "从自动驾驶芯片到大语言模型INT8量化训练实战解析"
 *   [PREC]    "大语言模型轻量化与量化精度" (choosing quantization precision)
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller; the library keeps no
 *     reference to them after the call returns and allocates no memory itself. Where
 *     an operation needs scratch space the caller passes it (ws, ws_bytes), sized by
 *     sq_workspace_size().
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream). Results
 *     are ready once the stream is synchronised.
 *   - Matrices are row-major. bf16 values are passed as their 16-bit patterns
 *     (`const void*`). X is [M, K] (tokens x in-features) with leading dimension ldx
 *     (elements); W is [N, K] (out-features x in-features, the nn.Linear layout) with
 *     leading dimension ldw. Int8 code matrices Xq [M, K] and Wq [N, K] and the output
 *     Y [M, N] are dense (leading dimension K, K and N).
 *   - Shape limits: 1 <= M, N <= 2^31-1; 16 <= K <= 65536 with K % 16 == 0 (so that
 *     |acc| <= K*128*128 < 2^31 and every row is a whole number of 16-byte vectors);
 *     ldx, ldw >= K and multiples of 8; N % 8 == 0 for outputs.
 *   - Alignment: every tensor base 16-byte aligned (float vectors included).
 *   - Arguments are validated before anything is launched; a violation returns
 *     SQ_ERR_INVALID / SQ_ERR_ALIGN / SQ_ERR_WORKSPACE, launches nothing and leaves
 *     outputs untouched. sq_last_error() then gives a message (thread-local).
 *   - NaN or Inf inputs are outside the contract (outputs undefined, no error). What the
 *     kernels happen to produce is not a guarantee: a NaN inside a row quantized by its
 *     own maximum (per token, per channel) currently gets code -1, one in a row whose
 *     factor 127/absmax overflowed, or under a per-tensor or clipped scale, gets -128, and
 *     one under the zero-point form gets the row's zero point (maxima ignore NaNs).
 *   - Rounding: codes use round-half-to-even of (value * (127/absmax)) in fp32 and are
 *     clamped to [-128, 127]; absmax == 0 gives codes 0 and scale 0. The reciprocal
 *     127/absmax and the scale absmax/127 are IEEE fp32 divisions.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sq_stream_t; /* same handle as cudaStream_t */

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID = -1,     /* null pointer, bad size, bad enum */
  SQ_ERR_ALIGN = -2,       /* pointer or leading dimension not aligned as required */
  SQ_ERR_CUDA = -3,        /* a CUDA runtime / driver call failed (message has the code) */
  SQ_ERR_TIMEOUT = -4,     /* a bounded device-side wait gave up (see sq_sync_status) */
  SQ_ERR_WORKSPACE = -5,   /* ws NULL or smaller than sq_workspace_size() */
  SQ_ERR_UNSUPPORTED = -6, /* no sm_100a device, or the library was built without it */
  SQ_ERR_BOUNDS = -7       /* a device-side bounds guard fired (libsq_debug.so only; see sq_sync_status) */
} sq_status;

typedef enum { SQ_PER_TENSOR = 0, SQ_PER_CHANNEL = 1 } sq_gran;

typedef enum { SQ_NORM_LAYER = 0, SQ_NORM_RMS = 1 } sq_norm;

typedef enum {
  SQ_OP_SMOOTH_QUANT_WEIGHT = 1,
  SQ_OP_INT8_GEMM_DEQUANT = 2, /* also sq_int8_gemm_dequant_ex */
  SQ_OP_LLMINT8 = 3,           /* also llmint8_decomposed_linear_ex */
  SQ_OP_QUANT_ACT_PER_TENSOR = 4,
  SQ_OP_MEAN_STD_THRESHOLD = 5,
  SQ_OP_ABS_PERCENTILE = 6
} sq_op;

/*
 * Per-input-channel absolute maximum of the activations (calibration statistic).
 *   amax[j] = max_m |X[m, j]|                  (accumulate == 0)
 *   amax[j] = max(amax[j], max_m |X[m, j]|)    (accumulate != 0: running maximum
 *                                               over calibration batches)
 * [SQ] §3.2 (a forward hook records each input channel's absolute maximum over the token
 * dimensions and keeps the running maximum across calibration batches); [LLMINT8] §2.1
 * step 1 (column-wise absolute maximum).
 * X: bf16 [M, K], ldx. amax: fp32 [K], read (accumulate) and written. Exact (a max).
 */
SQ_API sq_status sq_act_channel_absmax(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, float* amax,
                                int accumulate, sq_stream_t stream);

/*
 * SmoothQuant smoothing factors. [SQ] §2.1 (s_j = max|X_j|^alpha / max|W_j|^(1-alpha))
 * and §3.3 (weight maximum over the output dimension, both maxima clamped at 1e-8):
 *   wmax_j  = max_n |W[n, j]|
 *   s_j     = fp32( pow(max(act_amax_j,1e-8), alpha) / pow(max(wmax_j,1e-8), 1-alpha) )
 *             (evaluated in fp64, rounded once)
 *   inv_s_j = 1 / s_j   (fp32)
 * act_amax: fp32 [K] (from sq_act_channel_absmax). W: bf16 [N, K], ldw.
 * alpha in [0, 1]. s, inv_s: fp32 [K], written (s may not alias act_amax).
 */
SQ_API sq_status sq_smooth_scale(const float* act_amax, const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                          float alpha, float* s, float* inv_s, sq_stream_t stream);

/*
 * Smoothed weight quantization. [SQ] §3.3 (W' = W * s over the input dimension) and
 * §3.4 (w_scale = max|W'|/127); [BASICS] per-tensor / per-channel granularity and the
 * quantization-flow example:
 *   w'[n,k] = W[n,k] * s[k]       (fp32, never rounded; s == NULL means s = 1)
 *   SQ_PER_CHANNEL: a_n = max_k |w'[n,k]|, w_scale[n] = a_n/127, Wq[n,k] = q(w', a_n)
 *   SQ_PER_TENSOR : a   = max |w'|,       w_scale[0] = a/127,   Wq[n,k] = q(w', a)
 *   q(v, a) = clamp(rne(v * (127/a)), -128, 127)
 * W: bf16 [N, K], ldw. Wq: int8 [N, K] dense. w_scale: fp32 [N] or [1].
 * ws: SQ_PER_TENSOR needs sq_workspace_size(SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K) bytes
 * (one global maximum); SQ_PER_CHANNEL needs none (ws may be NULL).
 */
SQ_API sq_status sq_smooth_quant_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s,
                                 sq_gran gran, int8_t* Wq, float* w_scale, void* ws, size_t ws_bytes,
                                 sq_stream_t stream);

/*
 * Smoothing + per-token dynamic activation quantization in one pass over X.
 * [BASICS] per-token granularity and quantization-flow example (each token row's scale is
 * its absolute maximum over 127); [SQ] §2.3 and §3.4 (divide by s before quantizing,
 * fused into one light kernel), here as a multiply by inv_s:
 *   x'[m,k] = X[m,k] * inv_s[k]   (fp32; inv_s == NULL means 1)
 *   a_m = max_k |x'[m,k]|, x_scale[m] = a_m/127, Xq[m,k] = clamp(rne(x' * (127/a_m)), -128, 127)
 * X: bf16 [M, K], ldx. Xq: int8 [M, K] dense. x_scale: fp32 [M].
 */
SQ_API sq_status sq_quant_act_per_token(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                 int8_t* Xq, float* x_scale, sq_stream_t stream);

/*
 * INT8 GEMM with fused dequantization epilogue on the 5th-generation tensor cores.
 * [BASICS] INT8 inference flow ("(M,K) x (K,N) -> INT32 accumulate, INT32 -> 16-bit
 * dequantized output") and quantization-flow example (Y = Y_int32 * X_scale * W_scale);
 * [SQ] §3.4 (out * (x_scale * w_scale) + bias, bias kept in floating point, §4.5):
 *   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]                         (exact int32)
 *   Y[m,n]   = bf16_rne( (float(acc) * x_scale[m]) * w_scale[n or 0] + bias[n] )
 * Xq: int8 [M, K]; Wq: int8 [N, K]; x_scale: fp32 [M]; w_scale: fp32 [N] (SQ_PER_CHANNEL)
 * or [1] (SQ_PER_TENSOR); bias: bf16 [N] or NULL; Y: bf16 [M, N].
 * acc_out: int32 [M, N] or NULL — when given, the raw INT32 accumulator is written too
 * (for exact checking). ws: sq_workspace_size(SQ_OP_INT8_GEMM_DEQUANT, M, N, K) bytes: zero
 * for shapes with enough output tiles to fill the GPU (ws may then be NULL). Small-M shapes
 * split every tile along K: each part writes its exact int32 partial to ws and the last part
 * to arrive sums them and runs the epilogue, so the result is bit-identical to the unsplit
 * one. Such a ws must be zero-filled before its first use; every completed call leaves its
 * arrival counters at zero again (after SQ_ERR_TIMEOUT, zero it again). Calls that share
 * one ws must not overlap on the GPU.
 */
SQ_API sq_status sq_int8_gemm_dequant(const int8_t* Xq, const int8_t* Wq, const float* x_scale, const float* w_scale,
                               sq_gran w_gran, const void* bias_bf16, void* Y_bf16, int64_t M, int64_t N,
                               int64_t K, int32_t* acc_out, void* ws, size_t ws_bytes, sq_stream_t stream);

/*
 * LLM.int8() mixed-precision decomposed linear. [LLMINT8] §2.1 (column absmax of the
 * input, columns over the threshold are outliers, handled apart; the rest in 8 bits),
 * §2.2 (quantize / dequantize), §3.1 (bitmask of outlier columns, INT8 GEMM for the
 * normal columns, 16-bit GEMM for the outlier columns, results merged):
 *   amax_j = max_m |X[m,j]|;   O = { j : amax_j > threshold }   (strict)
 *   a_m = max_{k not in O} |X[m,k]|, d_m = a_m/127, Xq[m,k] = q(X[m,k], a_m) for k not in O,
 *         Xq[m,k] = 0 for k in O
 *   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]                                  (exact int32)
 *   o[m,n]   = sum_{j in O} X[m,j] * W[n,j]     (bf16 inputs, fp32 tensor-core accumulate)
 *   Y[m,n]   = bf16_rne( (float(acc) * d_m) * w_scale[n] + o[m,n] + bias[n] )
 * X: bf16 [M, K], ldx == K. W: bf16 [N, K], ldw == K (the original weight; its outlier
 * columns feed the 16-bit product). Wq, w_scale: the per-channel int8 weight and scales
 * of the UNSMOOTHED W (sq_smooth_quant_weight(W, s = NULL, SQ_PER_CHANNEL)).
 * bias: bf16 [N] or NULL. Y: bf16 [M, N].
 * mask_out: uint32 [ceil(K/32)] or NULL (bit j%32 of word j/32 set for j in O).
 * n_outliers_out: int32 [1] device or NULL (|O|). acc_out: int32 [M, N] or NULL.
 * ws: sq_workspace_size(SQ_OP_LLMINT8, M, N, K) bytes (holds the int8 activations, the
 * outlier index list and the gathered outlier columns of X and W).
 */
SQ_API sq_status llmint8_decomposed_linear(const void* X_bf16, const void* W_bf16, const int8_t* Wq,
                                    const float* w_scale, float threshold, const void* bias_bf16, void* Y_bf16,
                                    int64_t M, int64_t N, int64_t K, uint32_t* mask_out,
                                    int32_t* n_outliers_out, int32_t* acc_out, void* ws, size_t ws_bytes,
                                    sq_stream_t stream);

/*
 * Variant of sq_smooth_quant_weight that allocates nothing and takes no workspace, for
 * callers that cannot allocate device memory: components running inside a host engine,
 * server or plugin interface that owns the whole device-memory plan and passes them only
 * the tensors of the current call, and services that fix their memory footprint at
 * start-up. It has no counterpart on the pages; the quantization it performs is exactly
 * that of sq_smooth_quant_weight (same arguments minus ws/ws_bytes, same results).
 * Scratch: a 256-byte static device array inside the library (the per-tensor form keeps its
 * global maximum there; the per-channel form needs none). Every GPU that loads the library
 * holds those bytes until the process exits. A shape that would need more scratch than the
 * array holds is rejected with SQ_ERR_WORKSPACE and a message naming both sizes.
 * Set-up: every call looks the array's device address up on the current device (a host-side
 * query, so no address outlives a device reset); the first call on a device may load the
 * library's device code, so make that first call before any stream capture.
 * Concurrency: all calls share the array and it keeps the last call's contents; each
 * per-tensor call resets the maximum it needs before use, but calls that overlap on the GPU
 * (different streams, or several host threads) race on it and must be serialised.
 */
SQ_API sq_status sq_smooth_quant_weight_noalloc(const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                                                const float* s, sq_gran gran, int8_t* Wq, float* w_scale,
                                                sq_stream_t stream);

/* ============================================================================ variants
 * The calls below add the variants the pages describe beside the method: a per-tensor
 * activation scale (dynamic or calibrated), the normalisation of the smoothing factors,
 * normalisation layers fused with smoothing and quantization, a data-dependent outlier
 * threshold, percentile calibration and asymmetric (zero-point) activations. They follow
 * the conventions above. */

/*
 * Per-tensor activation quantization. [SQ] §3.4 (the reference module scales activations by
 * one maximum over the whole tensor): a = max |x'| over all elements, scale a/127, codes
 * clamp(rne(x' * 127/a), -128, 127):
 *   x'[m,k] = X[m,k] * inv_s[k]     (fp32; inv_s == NULL means 1)
 *   a = *clip when clip != NULL (a static calibration value, e.g. from sq_act_abs_percentile;
 *       values beyond it saturate at the clamp), else max |x'| over the tensor
 *   x_scale[0] = a/127, Xq[m,k] = clamp(rne(x' * (127/a)), -128, 127)
 * X: bf16 [M, K], ldx. clip: fp32 [1] device or NULL. Xq: int8 [M, K]. x_scale: fp32 [1].
 * ws: with clip == NULL, sq_workspace_size(SQ_OP_QUANT_ACT_PER_TENSOR, M, 0, K) bytes (the
 * running maximum); with a clip none (ws may be NULL). Two passes over X without a clip.
 */
SQ_API sq_status sq_quant_act_per_tensor(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                         const float* clip, int8_t* Xq, float* x_scale, void* ws, size_t ws_bytes,
                                         sq_stream_t stream);

/*
 * Smoothing factors with the optional normalisation of [SQ] §3.3 compute_smooth_scale:
 * normalize == 0 is sq_smooth_scale; otherwise, after s is formed,
 *   s_j <- max( (s_j / max_i s_i) * 127, 1e-5 )   (fp32, in that order),  inv_s_j = 1/s_j.
 * Any positive s keeps X.W^T = (X diag(s)^-1)(diag(s) W)^T, so the layer's result is the
 * same function; only the split of the quantization difficulty moves.
 */
SQ_API sq_status sq_smooth_scale_ex(const float* act_amax, const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                                    float alpha, int normalize, float* s, float* inv_s, sq_stream_t stream);

/*
 * INT8 GEMM + dequantization with the variants' activation forms:
 *   x_gran SQ_PER_CHANNEL: x_scale is per token, fp32 [M] (as sq_int8_gemm_dequant);
 *   x_gran SQ_PER_TENSOR : x_scale is fp32 [1] (sq_quant_act_per_tensor).
 *   x_zero (int32 [M], per-token zero points from sq_quant_act_per_token_asym) with
 *   w_rowsum (int32 [N], sum_k Wq[n,k] from sq_weight_row_sums): the accumulator is
 *   corrected exactly before the dequantization, [BASICS] asymmetric quantization
 *   (x ~ scale * (q - z), so sum_k (q - z) w = acc - z * rowsum):
 *     acc'[m,n] = acc[m,n] - x_zero[m] * w_rowsum[n]     (64-bit integer arithmetic)
 *     Y[m,n]    = bf16_rne( (float(acc') * x_scale[m]) * w_scale[n or 0] + bias[n] )
 *   x_zero needs x_gran == SQ_PER_CHANNEL and a w_rowsum; x_zero == NULL is symmetric.
 * Everything else as sq_int8_gemm_dequant (acc_out receives the uncorrected acc; ws is
 * sized by SQ_OP_INT8_GEMM_DEQUANT).
 */
SQ_API sq_status sq_int8_gemm_dequant_ex(const int8_t* Xq, const int8_t* Wq, const float* x_scale, sq_gran x_gran,
                                         const int32_t* x_zero, const float* w_scale, sq_gran w_gran,
                                         const int32_t* w_rowsum, const void* bias_bf16, void* Y_bf16, int64_t M,
                                         int64_t N, int64_t K, int32_t* acc_out, void* ws, size_t ws_bytes,
                                         sq_stream_t stream);

/*
 * Normalisation layer, smoothing and per-token quantization in one pass over X: the
 * smoothing folded into the output of the LayerNorm that precedes the linear layer
 * ([SQ] §4.2 fuse the scaling into the previous operation's output; §4.5 second detail).
 * Per row m, statistics in fp64 rounded once to fp32 (computed in one pass from the sums of
 * x and x^2; for K > 4096 the division by K is a multiply by 1/K and 1/sqrt a reciprocal
 * square root, each within a few fp64 ulps; so on rare rows a statistic may differ from a
 * two-pass evaluation by one fp32 ulp):
 *   SQ_NORM_LAYER: mean = sum_k x / K, var = sum_k (x - mean)^2 / K,
 *                  rstd = fp32(1/sqrt(var + eps)), y = ((x - fp32(mean)) * rstd) * gamma_k + beta_k
 *   SQ_NORM_RMS:   rstd = fp32(1/sqrt(sum_k x^2 / K + eps)),   y = (x * rstd) * gamma_k + beta_k
 *   x' = y * inv_s_k (inv_s == NULL means 1), a_m = max_k |x'|, x_scale[m] = a_m/127,
 *   Xq[m,k] = clamp(rne(x' * (127/a_m)), -128, 127)                  (fp32, no contraction)
 * X: bf16 [M, K], ldx. gamma: bf16 [K]. beta: bf16 [K] or NULL (0). eps >= 0.
 * mean_rstd: fp32 [M, 2] (fp32(mean) or 0 for RMS, rstd) or NULL. K <= 16384.
 */
SQ_API sq_status sq_norm_smooth_quant(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, sq_norm norm,
                                      const void* gamma_bf16, const void* beta_bf16, float eps, const float* inv_s,
                                      int8_t* Xq, float* x_scale, float* mean_rstd, sq_stream_t stream);

/*
 * Data-dependent outlier threshold: threshold = mean + k * std over all M*K elements of X,
 * std the unbiased standard deviation. [LLMINT8] §3.1 pre-screening (threshold = mu + 6
 * sigma from the layer's activation statistics); [QAT] §2.1 (mean + 3 std).
 * One pass over X: the sums of x and x^2 in fp64 (fixed summation order, so the result is
 * deterministic), mean = S1/n, var = (S2 - S1*mean)/(n-1); the threshold is rounded once
 * to fp32.
 * threshold: fp32 [1] device. mean_std: fp64 [2] device (mean, std) or NULL.
 * ws: sq_workspace_size(SQ_OP_MEAN_STD_THRESHOLD, M, 0, K) bytes.
 */
SQ_API sq_status sq_act_mean_std_threshold(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double k,
                                           float* threshold, double* mean_std, void* ws, size_t ws_bytes,
                                           sq_stream_t stream);

/*
 * llmint8_decomposed_linear with the threshold read from device memory (for instance the
 * output of sq_act_mean_std_threshold), so that a data-dependent threshold needs no host
 * round trip. threshold: fp32 [1] device. Everything else as llmint8_decomposed_linear.
 */
SQ_API sq_status llmint8_decomposed_linear_ex(const void* X_bf16, const void* W_bf16, const int8_t* Wq,
                                              const float* w_scale, const float* threshold, const void* bias_bf16,
                                              void* Y_bf16, int64_t M, int64_t N, int64_t K, uint32_t* mask_out,
                                              int32_t* n_outliers_out, int32_t* acc_out, void* ws, size_t ws_bytes,
                                              sq_stream_t stream);

/*
 * Percentile calibration: the nearest-rank p-th percentile of |X| over all n = M*K
 * elements, [PREC] §3.2 (a max calibrator with the percentile method, 99.99): the element
 * of 1-based rank ceil(p/100 * n) (at least 1) of the ascending absolute values. Exact (a
 * histogram of the 2^15 bf16 magnitudes and a scan). 0 <= p <= 100.
 * out: fp32 [1] device. ws: sq_workspace_size(SQ_OP_ABS_PERCENTILE, M, 0, K) bytes.
 */
SQ_API sq_status sq_act_abs_percentile(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double p, float* out,
                                       void* ws, size_t ws_bytes, sq_stream_t stream);

/*
 * Asymmetric per-token activation quantization, [BASICS] asymmetric quantization
 * (scale = (max - min)/255 and a zero point), on signed codes and over the row's range
 * extended to contain 0 (so that 0 is represented exactly):
 *   x' = X * inv_s (inv_s == NULL means 1); lo = min(0, min_k x'), hi = max(0, max_k x')
 *   range = hi - lo, r = 255/range (0 if range == 0), x_scale[m] = range/255,
 *   x_zero[m] = -128 - rne(lo * r), Xq[m,k] = clamp(rne(x' * r) + x_zero[m], -128, 127)
 *   so that x' ~ x_scale[m] * (Xq - x_zero[m]).
 * X: bf16 [M, K], ldx. Xq: int8 [M, K]. x_scale: fp32 [M]. x_zero: int32 [M].
 */
SQ_API sq_status sq_quant_act_per_token_asym(const void* X_bf16, int64_t M, int64_t K, int64_t ldx,
                                             const float* inv_s, int8_t* Xq, float* x_scale, int32_t* x_zero,
                                             sq_stream_t stream);

/*
 * Row sums of an int8 weight, rowsum[n] = sum_k Wq[n,k] (exact int32): the zero-point
 * correction term of sq_int8_gemm_dequant_ex. Wq: int8 [N, K]. rowsum: int32 [N].
 */
SQ_API sq_status sq_weight_row_sums(const int8_t* Wq, int64_t N, int64_t K, int32_t* rowsum, sq_stream_t stream);

/* Bytes of scratch an operation needs for the given shape (0 if none). Returns 0 for an
 * unknown op; never fails otherwise. */
SQ_API size_t sq_workspace_size(int op, int64_t M, int64_t N, int64_t K);

/* Message for the last non-OK status returned on the calling thread ("" if none). The
 * pointer stays valid until the next call on that thread. */
SQ_API const char* sq_last_error(void);

/* Synchronises `stream`, then reads and clears the current device's error word, which
 * kernels set when a bounded wait gives up (a device-side stall or lost arrival) instead
 * of spinning forever, and, in the debug build libsq_debug.so (same ABI, kernels compiled
 * with device-side bounds guards that skip and record an out-of-range access), when a guard
 * fires. Returns SQ_OK, SQ_ERR_TIMEOUT, SQ_ERR_BOUNDS or SQ_ERR_CUDA. */
SQ_API sq_status sq_sync_status(sq_stream_t stream);

/* Library version string and the compute capability it was built for ("sm_100a"). */
SQ_API const char* sq_version(void);

/* Number of kernels this library has launched in this process (all devices, all threads),
 * for checking which work ran on the GPU. */
SQ_API uint64_t sq_kernel_launch_count(void);

/* Test hook for the failure path (no counterpart on the pages). Arms the NEXT
 * sq_int8_gemm_dequant call made on the calling thread: its device-side waits give up after
 * wait_limit_ns nanoseconds (0 = the default of 2 s) and, when fault == 1, its TMA producer
 * withholds one pipeline stage, so the consumer's bounded wait runs out. The kernel then
 * records the timeout, drains its own copies, frees its tensor memory and returns;
 * sq_sync_status() reports SQ_ERR_TIMEOUT and the context stays usable. Not for production
 * use; the output of the armed call is undefined. */
SQ_API void sq_debug_arm_fault(int fault, uint64_t wait_limit_ns);

/* Test hook (no counterpart on the pages): the launch plan that sq_int8_gemm_dequant
 * (outliers = 0) or the GEMM of llmint8_decomposed_linear (outliers = 1) uses for an
 * M x N x K product, computed on the host without touching a device. plan (caller-owned,
 * 7 entries) receives: [0] path (0 = the CUDA-core product for a few tokens, 1 = tensor
 * cores with one CTA per output tile, 2 = tensor cores with CTA pairs on 256-row tiles),
 * [1] 1 if the operands are swapped (weight rows on the 128-row MMA operand), [2] the tile
 * width BN, [3] whole-tile work units, [4] tiles split along K, [5] parts per split tile,
 * [6] k-blocks (128 bytes of K) per part. Returns SQ_ERR_INVALID (plan untouched) when a
 * size is not positive or plan is NULL. */
SQ_API sq_status sq_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int outliers, int64_t* plan);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
