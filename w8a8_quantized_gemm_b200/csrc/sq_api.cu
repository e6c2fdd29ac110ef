// C ABI of libsq (declared in include/sq.h): argument validation, workspace layout,
// error reporting, and the sequencing of the kernels of each operation on the
// caller's stream. Nothing here allocates device memory.
#include "sq.h"
#include "sq_internal.h"

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

namespace sq {

// Per-device error word set by kernels whose bounded waits give up.
__device__ unsigned int g_status_word;

// Looked up on every launch (a host-side query on the current device): no address is kept
// across calls, so none outlives a device reset and concurrent host threads share no state.
unsigned int* device_status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

namespace {
std::atomic<uint64_t> g_launches{0};
}
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace sq

namespace {

thread_local std::string g_last_error;
thread_local int g_arm_fault = 0;
thread_local uint64_t g_arm_limit_ns = 0;

sq_status fail(sq_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
sq_status fail(sq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

}  // namespace

int sq::record_error(int st, const char* msg) {
  g_last_error = msg;
  return st;
}

namespace {

sq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxK = 65536;
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1;

sq_status check_rows(const char* fn, const char* what, const void* ptr, int64_t rows, int64_t K, int64_t ld) {
  if (ptr == nullptr) return fail(SQ_ERR_INVALID, "%s: %s is NULL", fn, what);
  if (rows < 1 || rows > kMaxRows) return fail(SQ_ERR_INVALID, "%s: %s rows=%lld out of [1, 2^31-1]", fn, what,
                                               static_cast<long long>(rows));
  if (K < 16 || K > kMaxK || K % 16 != 0)
    return fail(SQ_ERR_INVALID, "%s: K=%lld must be a multiple of 16 in [16, 65536]", fn, static_cast<long long>(K));
  if (ld < K) return fail(SQ_ERR_INVALID, "%s: leading dimension %lld < K", fn, static_cast<long long>(ld));
  if (ld % 8 != 0) return fail(SQ_ERR_ALIGN, "%s: leading dimension of %s must be a multiple of 8", fn, what);
  if (!aligned16(ptr)) return fail(SQ_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, what);
  return SQ_OK;
}

sq_status check_vec(const char* fn, const char* what, const void* p, bool required) {
  if (p == nullptr) return required ? fail(SQ_ERR_INVALID, "%s: %s is NULL", fn, what) : SQ_OK;
  if (!aligned16(p)) return fail(SQ_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, what);
  return SQ_OK;
}

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Workspace of llmint8_decomposed_linear, in this order (each 256-byte aligned):
//   amax fp32[K] | mask u32[W] | prefix i32[W] | idx i32[K] | count i32[1] |
//   Xq int8[M,K] | d fp32[M] | Xo bf16[M, ldo] | Wo bf16[N, ldo]
// with W = ceil(K/32) and ldo = roundup(K, 64).
struct LlmLayout {
  size_t amax, mask, prefix, idx, count, xq, d, xo, wo, total;
  int64_t ldo;
};

LlmLayout llm_layout(int64_t M, int64_t N, int64_t K) {
  LlmLayout L{};
  const size_t W = static_cast<size_t>((K + 31) / 32);
  L.ldo = (K + 63) / 64 * 64;
  size_t o = 0;
  L.amax = o; o += up(sizeof(float) * K);
  L.mask = o; o += up(sizeof(uint32_t) * W);
  L.prefix = o; o += up(sizeof(int32_t) * W);
  L.idx = o; o += up(sizeof(int32_t) * K);
  L.count = o; o += up(sizeof(int32_t));
  L.xq = o; o += up(static_cast<size_t>(M) * K);
  L.d = o; o += up(sizeof(float) * M);
  L.xo = o; o += up(sizeof(uint16_t) * static_cast<size_t>(M) * L.ldo);
  L.wo = o; o += up(sizeof(uint16_t) * static_cast<size_t>(N) * L.ldo);
  L.total = o;
  return L;
}

bool tiles_fit(int64_t M, int64_t N) { return ((M + 127) / 128) * ((N + 63) / 64) < (int64_t(1) << 31); }

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

}  // namespace

extern "C" {

sq_status sq_act_channel_absmax(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, float* amax,
                                int accumulate, sq_stream_t stream) {
  const char* fn = "sq_act_channel_absmax";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "amax", amax, true)) != SQ_OK) return st;
  cudaError_t e = sq::launch_col_absmax(static_cast<const uint16_t*>(X_bf16), M, K, ldx, amax, accumulate != 0,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_smooth_scale(const float* act_amax, const void* W_bf16, int64_t N, int64_t K, int64_t ldw, float alpha,
                          float* s, float* inv_s, sq_stream_t stream) {
  const char* fn = "sq_smooth_scale";
  sq_status st = check_rows(fn, "W", W_bf16, N, K, ldw);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "act_amax", act_amax, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "s", s, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "inv_s", inv_s, true)) != SQ_OK) return st;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return fail(SQ_ERR_INVALID, "%s: alpha=%g outside [0, 1]", fn, alpha);
  if (static_cast<const void*>(s) == static_cast<const void*>(act_amax) || s == inv_s)
    return fail(SQ_ERR_INVALID, "%s: s must not alias act_amax or inv_s", fn);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e =
      sq::launch_smooth_scale(act_amax, static_cast<const uint16_t*>(W_bf16), N, K, ldw, alpha, s, inv_s, cs);
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_smooth_quant_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s,
                                 sq_gran gran, int8_t* Wq, float* w_scale, void* ws, size_t ws_bytes,
                                 sq_stream_t stream) {
  const char* fn = "sq_smooth_quant_weight";
  sq_status st = check_rows(fn, "W", W_bf16, N, K, ldw);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "s", s, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Wq", Wq, true)) != SQ_OK) return st;
  if (w_scale == nullptr) return fail(SQ_ERR_INVALID, "%s: w_scale is NULL", fn);
  if (gran != SQ_PER_TENSOR && gran != SQ_PER_CHANNEL) return fail(SQ_ERR_INVALID, "%s: bad granularity", fn);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (gran == SQ_PER_CHANNEL) {
    e = sq::launch_quant_rows(static_cast<const uint16_t*>(W_bf16), N, K, ldw, s, sq::OutlierView{}, Wq, w_scale,
                              cs);
  } else {
    const size_t need = sq_workspace_size(SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K);
    if (ws == nullptr || ws_bytes < need)
      return fail(SQ_ERR_WORKSPACE, "%s: per-tensor needs %zu workspace bytes, got %zu", fn, need,
                  ws == nullptr ? size_t(0) : ws_bytes);
    if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0) return fail(SQ_ERR_ALIGN, "%s: ws not 4-byte aligned", fn);
    e = sq::launch_quant_tensor(static_cast<const uint16_t*>(W_bf16), N, K, ldw, s, static_cast<unsigned int*>(ws),
                                Wq, w_scale, cs);
  }
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_quant_act_per_token(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                 int8_t* Xq, float* x_scale, sq_stream_t stream) {
  const char* fn = "sq_quant_act_per_token";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "inv_s", inv_s, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Xq", Xq, true)) != SQ_OK) return st;
  if (x_scale == nullptr) return fail(SQ_ERR_INVALID, "%s: x_scale is NULL", fn);
  cudaError_t e = sq::launch_quant_rows(static_cast<const uint16_t*>(X_bf16), M, K, ldx, inv_s, sq::OutlierView{},
                                        Xq, x_scale, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

}  // extern "C"

namespace {

sq_status gemm_impl(const char* fn, const int8_t* Xq, const int8_t* Wq, const float* x_scale, sq_gran x_gran,
                    const int32_t* x_zero, const float* w_scale, sq_gran w_gran, const int32_t* w_rowsum,
                    const void* bias_bf16, void* Y_bf16, int64_t M, int64_t N, int64_t K, int32_t* acc_out, void* ws,
                    size_t ws_bytes, sq_stream_t stream) {
  sq_status st;
  if (x_gran != SQ_PER_TENSOR && x_gran != SQ_PER_CHANNEL) return fail(SQ_ERR_INVALID, "%s: bad x granularity", fn);
  if (x_zero != nullptr && (x_gran != SQ_PER_CHANNEL || w_rowsum == nullptr))
    return fail(SQ_ERR_INVALID, "%s: x_zero needs per-token x_scale and w_rowsum", fn);
  if ((x_zero != nullptr && (reinterpret_cast<uintptr_t>(x_zero) & 3u)) ||
      (w_rowsum != nullptr && (reinterpret_cast<uintptr_t>(w_rowsum) & 3u)))
    return fail(SQ_ERR_ALIGN, "%s: x_zero / w_rowsum not 4-byte aligned", fn);
  if ((st = check_rows(fn, "Xq", Xq, M, K, K)) != SQ_OK) return st;
  if ((st = check_rows(fn, "Wq", Wq, N, K, K)) != SQ_OK) return st;
  if (x_scale == nullptr || w_scale == nullptr) return fail(SQ_ERR_INVALID, "%s: scale pointer is NULL", fn);
  if (w_gran != SQ_PER_TENSOR && w_gran != SQ_PER_CHANNEL) return fail(SQ_ERR_INVALID, "%s: bad granularity", fn);
  if (w_gran == SQ_PER_CHANNEL && !aligned16(w_scale))
    return fail(SQ_ERR_ALIGN, "%s: per-channel w_scale is not 16-byte aligned", fn);
  if ((st = check_vec(fn, "bias", bias_bf16, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Y", Y_bf16, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "acc_out", acc_out, false)) != SQ_OK) return st;
  if (N % 8 != 0) return fail(SQ_ERR_INVALID, "%s: N=%lld must be a multiple of 8", fn, static_cast<long long>(N));
  if (!tiles_fit(M, N)) return fail(SQ_ERR_INVALID, "%s: M x N too large", fn);
  const size_t need = sq::gemm_workspace_bytes(M, N, K, false);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(SQ_ERR_WORKSPACE, "%s: needs %zu workspace bytes", fn, need);
  sq::GemmArgs a;
  a.Xq = Xq;
  a.Wq = Wq;
  a.x_scale = x_scale;
  a.x_per_token = (x_gran == SQ_PER_CHANNEL);
  a.x_zero = x_zero;
  a.w_rowsum = w_rowsum;
  a.w_scale = w_scale;
  a.w_per_channel = (w_gran == SQ_PER_CHANNEL);
  a.bias = static_cast<const uint16_t*>(bias_bf16);
  a.Y = static_cast<uint16_t*>(Y_bf16);
  a.acc_out = acc_out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  if (g_arm_limit_ns != 0) {
    a.wait_limit_ns = g_arm_limit_ns;
    a.fault = g_arm_fault;
    g_arm_limit_ns = 0;
    g_arm_fault = 0;
  }
  if (sq::device_status_word() == nullptr) return fail(SQ_ERR_CUDA, "%s: device status word not found", fn);
  const char* why = "kernel launch";
  cudaError_t e = sq::launch_gemm(a, reinterpret_cast<cudaStream_t>(stream), &why);
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, why);
}

sq_status llm_impl(const char* fn, const void* X_bf16, const void* W_bf16, const int8_t* Wq, const float* w_scale,
                   float threshold, const float* threshold_dev, const void* bias_bf16, void* Y_bf16, int64_t M,
                   int64_t N, int64_t K, uint32_t* mask_out, int32_t* n_outliers_out, int32_t* acc_out, void* ws,
                   size_t ws_bytes, sq_stream_t stream) {
  sq_status st;
  if ((st = check_rows(fn, "X", X_bf16, M, K, K)) != SQ_OK) return st;
  if ((st = check_rows(fn, "W", W_bf16, N, K, K)) != SQ_OK) return st;
  if ((st = check_rows(fn, "Wq", Wq, N, K, K)) != SQ_OK) return st;
  if ((st = check_vec(fn, "w_scale", w_scale, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "bias", bias_bf16, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Y", Y_bf16, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "acc_out", acc_out, false)) != SQ_OK) return st;
  if (mask_out != nullptr && (reinterpret_cast<uintptr_t>(mask_out) & 3u))
    return fail(SQ_ERR_ALIGN, "%s: mask_out not 4-byte aligned", fn);
  if (n_outliers_out != nullptr && (reinterpret_cast<uintptr_t>(n_outliers_out) & 3u))
    return fail(SQ_ERR_ALIGN, "%s: n_outliers_out not 4-byte aligned", fn);
  if (N % 8 != 0) return fail(SQ_ERR_INVALID, "%s: N=%lld must be a multiple of 8", fn, static_cast<long long>(N));
  if (!tiles_fit(M, N)) return fail(SQ_ERR_INVALID, "%s: M x N too large", fn);
  if (threshold_dev == nullptr && threshold != threshold) return fail(SQ_ERR_INVALID, "%s: threshold is NaN", fn);
  if (threshold_dev != nullptr && (reinterpret_cast<uintptr_t>(threshold_dev) & 3u))
    return fail(SQ_ERR_ALIGN, "%s: threshold not 4-byte aligned", fn);
  const LlmLayout L = llm_layout(M, N, K);
  if (ws == nullptr || ws_bytes < L.total)
    return fail(SQ_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", fn, L.total,
                ws == nullptr ? size_t(0) : ws_bytes);
  if (!aligned16(ws)) return fail(SQ_ERR_ALIGN, "%s: ws not 16-byte aligned", fn);

  if (sq::device_status_word() == nullptr) return fail(SQ_ERR_CUDA, "%s: device status word not found", fn);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* X = static_cast<const uint16_t*>(X_bf16);
  const uint16_t* W = static_cast<const uint16_t*>(W_bf16);
  float* amax = at<float>(ws, L.amax);
  uint32_t* mask = at<uint32_t>(ws, L.mask);
  int32_t* prefix = at<int32_t>(ws, L.prefix);
  int32_t* idx = at<int32_t>(ws, L.idx);
  int32_t* count = at<int32_t>(ws, L.count);
  int8_t* Xq = at<int8_t>(ws, L.xq);
  float* d = at<float>(ws, L.d);
  uint16_t* Xo = at<uint16_t>(ws, L.xo);
  uint16_t* Wo = at<uint16_t>(ws, L.wo);

  cudaError_t e = sq::launch_col_absmax(X, M, K, K, amax, false, cs);
  if (e == cudaSuccess)
    e = sq::launch_outlier_mask(amax, K, threshold, threshold_dev, mask, prefix, idx, count, mask_out,
                                n_outliers_out, cs);
  if (e == cudaSuccess) {
    sq::OutlierView ov;
    ov.mask = mask;
    ov.prefix = prefix;
    ov.count = count;
    ov.gathered = Xo;
    ov.ld_gathered = L.ldo;
    ov.w_src = W;
    ov.w_rows = N;
    ov.w_ld = K;
    ov.idx = idx;
    ov.w_gathered = Wo;
    e = sq::launch_quant_rows(X, M, K, K, nullptr, ov, Xq, d, cs);
  }
  if (e != cudaSuccess) return cuda_fail(e, fn);
  sq::GemmArgs a;
  a.Xq = Xq;
  a.Wq = Wq;
  a.x_scale = d;
  a.w_scale = w_scale;
  a.w_per_channel = true;
  a.bias = static_cast<const uint16_t*>(bias_bf16);
  a.Y = static_cast<uint16_t*>(Y_bf16);
  a.acc_out = acc_out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.Xo = Xo;
  a.Wo = Wo;
  a.o_count = count;
  a.ld_o = L.ldo;
  const char* why = "kernel launch";
  e = sq::launch_gemm(a, cs, &why);
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, why);
}

}  // namespace

extern "C" {

sq_status sq_int8_gemm_dequant(const int8_t* Xq, const int8_t* Wq, const float* x_scale, const float* w_scale,
                               sq_gran w_gran, const void* bias_bf16, void* Y_bf16, int64_t M, int64_t N, int64_t K,
                               int32_t* acc_out, void* ws, size_t ws_bytes, sq_stream_t stream) {
  return gemm_impl("sq_int8_gemm_dequant", Xq, Wq, x_scale, SQ_PER_CHANNEL, nullptr, w_scale, w_gran, nullptr,
                   bias_bf16, Y_bf16, M, N, K, acc_out, ws, ws_bytes, stream);
}

sq_status sq_int8_gemm_dequant_ex(const int8_t* Xq, const int8_t* Wq, const float* x_scale, sq_gran x_gran,
                                  const int32_t* x_zero, const float* w_scale, sq_gran w_gran, const int32_t* w_rowsum,
                                  const void* bias_bf16, void* Y_bf16, int64_t M, int64_t N, int64_t K,
                                  int32_t* acc_out, void* ws, size_t ws_bytes, sq_stream_t stream) {
  return gemm_impl("sq_int8_gemm_dequant_ex", Xq, Wq, x_scale, x_gran, x_zero, w_scale, w_gran, w_rowsum, bias_bf16,
                   Y_bf16, M, N, K, acc_out, ws, ws_bytes, stream);
}

sq_status llmint8_decomposed_linear(const void* X_bf16, const void* W_bf16, const int8_t* Wq, const float* w_scale,
                                    float threshold, const void* bias_bf16, void* Y_bf16, int64_t M, int64_t N,
                                    int64_t K, uint32_t* mask_out, int32_t* n_outliers_out, int32_t* acc_out,
                                    void* ws, size_t ws_bytes, sq_stream_t stream) {
  return llm_impl("llmint8_decomposed_linear", X_bf16, W_bf16, Wq, w_scale, threshold, nullptr, bias_bf16, Y_bf16, M,
                  N, K, mask_out, n_outliers_out, acc_out, ws, ws_bytes, stream);
}

sq_status llmint8_decomposed_linear_ex(const void* X_bf16, const void* W_bf16, const int8_t* Wq,
                                       const float* w_scale, const float* threshold, const void* bias_bf16,
                                       void* Y_bf16, int64_t M, int64_t N, int64_t K, uint32_t* mask_out,
                                       int32_t* n_outliers_out, int32_t* acc_out, void* ws, size_t ws_bytes,
                                       sq_stream_t stream) {
  if (threshold == nullptr) return fail(SQ_ERR_INVALID, "llmint8_decomposed_linear_ex: threshold is NULL");
  return llm_impl("llmint8_decomposed_linear_ex", X_bf16, W_bf16, Wq, w_scale, 0.0f, threshold, bias_bf16, Y_bf16,
                  M, N, K, mask_out, n_outliers_out, acc_out, ws, ws_bytes, stream);
}

sq_status sq_quant_act_per_tensor(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                  const float* clip, int8_t* Xq, float* x_scale, void* ws, size_t ws_bytes,
                                  sq_stream_t stream) {
  const char* fn = "sq_quant_act_per_tensor";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "inv_s", inv_s, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Xq", Xq, true)) != SQ_OK) return st;
  if (x_scale == nullptr) return fail(SQ_ERR_INVALID, "%s: x_scale is NULL", fn);
  if (clip != nullptr && (reinterpret_cast<uintptr_t>(clip) & 3u))
    return fail(SQ_ERR_ALIGN, "%s: clip not 4-byte aligned", fn);
  if (clip == nullptr) {
    const size_t need = sq_workspace_size(SQ_OP_QUANT_ACT_PER_TENSOR, M, 0, K);
    if (ws == nullptr || ws_bytes < need)
      return fail(SQ_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", fn, need,
                  ws == nullptr ? size_t(0) : ws_bytes);
    if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0) return fail(SQ_ERR_ALIGN, "%s: ws not 4-byte aligned", fn);
  }
  cudaError_t e = sq::launch_quant_tensor(static_cast<const uint16_t*>(X_bf16), M, K, ldx, inv_s,
                                          static_cast<unsigned int*>(ws), Xq, x_scale,
                                          reinterpret_cast<cudaStream_t>(stream), clip);
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_smooth_scale_ex(const float* act_amax, const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                             float alpha, int normalize, float* s, float* inv_s, sq_stream_t stream) {
  sq_status st = sq_smooth_scale(act_amax, W_bf16, N, K, ldw, alpha, s, inv_s, stream);
  if (st != SQ_OK || !normalize) return st;
  cudaError_t e = sq::launch_normalize_scale(s, inv_s, K, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, "sq_smooth_scale_ex");
}

sq_status sq_norm_smooth_quant(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, sq_norm norm,
                               const void* gamma_bf16, const void* beta_bf16, float eps, const float* inv_s,
                               int8_t* Xq, float* x_scale, float* mean_rstd, sq_stream_t stream) {
  const char* fn = "sq_norm_smooth_quant";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if (K > 16384) return fail(SQ_ERR_INVALID, "%s: K=%lld above 16384", fn, static_cast<long long>(K));
  if (norm != SQ_NORM_LAYER && norm != SQ_NORM_RMS) return fail(SQ_ERR_INVALID, "%s: bad norm", fn);
  if (!(eps >= 0.0f) || eps == INFINITY) return fail(SQ_ERR_INVALID, "%s: eps must be finite and >= 0", fn);
  if ((st = check_vec(fn, "gamma", gamma_bf16, true)) != SQ_OK) return st;
  if ((st = check_vec(fn, "beta", beta_bf16, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "inv_s", inv_s, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Xq", Xq, true)) != SQ_OK) return st;
  if (x_scale == nullptr) return fail(SQ_ERR_INVALID, "%s: x_scale is NULL", fn);
  if (mean_rstd != nullptr && (reinterpret_cast<uintptr_t>(mean_rstd) & 7u))
    return fail(SQ_ERR_ALIGN, "%s: mean_rstd not 8-byte aligned", fn);
  cudaError_t e = sq::launch_norm_quant(static_cast<const uint16_t*>(X_bf16), M, K, ldx, static_cast<int>(norm),
                                        static_cast<const uint16_t*>(gamma_bf16),
                                        static_cast<const uint16_t*>(beta_bf16), eps, inv_s, Xq, x_scale, mean_rstd,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_act_mean_std_threshold(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double k, float* threshold,
                                    double* mean_std, void* ws, size_t ws_bytes, sq_stream_t stream) {
  const char* fn = "sq_act_mean_std_threshold";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if (threshold == nullptr) return fail(SQ_ERR_INVALID, "%s: threshold is NULL", fn);
  if (reinterpret_cast<uintptr_t>(threshold) & 3u) return fail(SQ_ERR_ALIGN, "%s: threshold not aligned", fn);
  if (mean_std != nullptr && (reinterpret_cast<uintptr_t>(mean_std) & 7u))
    return fail(SQ_ERR_ALIGN, "%s: mean_std not 8-byte aligned", fn);
  if (k != k) return fail(SQ_ERR_INVALID, "%s: k is NaN", fn);
  const size_t need = sq_workspace_size(SQ_OP_MEAN_STD_THRESHOLD, M, 0, K);
  if (ws == nullptr || ws_bytes < need)
    return fail(SQ_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", fn, need,
                ws == nullptr ? size_t(0) : ws_bytes);
  if (reinterpret_cast<uintptr_t>(ws) & 7u) return fail(SQ_ERR_ALIGN, "%s: ws not 8-byte aligned", fn);
  cudaError_t e = sq::launch_mean_std_threshold(static_cast<const uint16_t*>(X_bf16), M, K, ldx, k, threshold,
                                                mean_std, ws, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_act_abs_percentile(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double p, float* out,
                                void* ws, size_t ws_bytes, sq_stream_t stream) {
  const char* fn = "sq_act_abs_percentile";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if (out == nullptr) return fail(SQ_ERR_INVALID, "%s: out is NULL", fn);
  if (reinterpret_cast<uintptr_t>(out) & 3u) return fail(SQ_ERR_ALIGN, "%s: out not 4-byte aligned", fn);
  if (!(p >= 0.0 && p <= 100.0)) return fail(SQ_ERR_INVALID, "%s: p=%g outside [0, 100]", fn, p);
  const size_t need = sq_workspace_size(SQ_OP_ABS_PERCENTILE, M, 0, K);
  if (ws == nullptr || ws_bytes < need)
    return fail(SQ_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", fn, need,
                ws == nullptr ? size_t(0) : ws_bytes);
  if (reinterpret_cast<uintptr_t>(ws) & 7u) return fail(SQ_ERR_ALIGN, "%s: ws not 8-byte aligned", fn);
  // 1-based nearest rank, computed on the host in fp64 exactly as written
  const int64_t n = M * K;
  int64_t rank = static_cast<int64_t>(std::ceil((p / 100.0) * static_cast<double>(n)));
  if (rank < 1) rank = 1;
  if (rank > n) rank = n;
  cudaError_t e = sq::launch_abs_percentile(static_cast<const uint16_t*>(X_bf16), M, K, ldx,
                                            static_cast<uint64_t>(rank), out, ws,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_quant_act_per_token_asym(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                      int8_t* Xq, float* x_scale, int32_t* x_zero, sq_stream_t stream) {
  const char* fn = "sq_quant_act_per_token_asym";
  sq_status st = check_rows(fn, "X", X_bf16, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((st = check_vec(fn, "inv_s", inv_s, false)) != SQ_OK) return st;
  if ((st = check_vec(fn, "Xq", Xq, true)) != SQ_OK) return st;
  if (x_scale == nullptr || x_zero == nullptr) return fail(SQ_ERR_INVALID, "%s: x_scale / x_zero is NULL", fn);
  if ((reinterpret_cast<uintptr_t>(x_zero) & 3u)) return fail(SQ_ERR_ALIGN, "%s: x_zero not 4-byte aligned", fn);
  cudaError_t e = sq::launch_quant_rows_asym(static_cast<const uint16_t*>(X_bf16), M, K, ldx, inv_s, Xq, x_scale,
                                             x_zero, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

sq_status sq_weight_row_sums(const int8_t* Wq, int64_t N, int64_t K, int32_t* rowsum, sq_stream_t stream) {
  const char* fn = "sq_weight_row_sums";
  sq_status st = check_rows(fn, "Wq", Wq, N, K, K);
  if (st != SQ_OK) return st;
  if (rowsum == nullptr) return fail(SQ_ERR_INVALID, "%s: rowsum is NULL", fn);
  if (reinterpret_cast<uintptr_t>(rowsum) & 3u) return fail(SQ_ERR_ALIGN, "%s: rowsum not 4-byte aligned", fn);
  cudaError_t e = sq::launch_row_sums(Wq, N, K, rowsum, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SQ_OK : cuda_fail(e, fn);
}

size_t sq_workspace_size(int op, int64_t M, int64_t N, int64_t K) {
  switch (op) {
    case SQ_OP_SMOOTH_QUANT_WEIGHT:
      return kAlign;
    case SQ_OP_INT8_GEMM_DEQUANT:
      return sq::gemm_workspace_bytes(M, N, K, false);
    case SQ_OP_LLMINT8:
      return (M < 1 || N < 1 || K < 1) ? 0 : llm_layout(M, N, K).total;
    case SQ_OP_QUANT_ACT_PER_TENSOR:
      return kAlign;
    case SQ_OP_MEAN_STD_THRESHOLD:
      return M < 1 ? 0 : sq::mean_std_workspace_bytes(M);
    case SQ_OP_ABS_PERCENTILE:
      return sq::abs_percentile_workspace_bytes();
    default:
      return 0;
  }
}

const char* sq_last_error(void) { return g_last_error.c_str(); }

sq_status sq_sync_status(sq_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sq_sync_status: cudaStreamSynchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, sq::g_status_word, sizeof word);
  if (e != cudaSuccess) return cuda_fail(e, "sq_sync_status: read status word");
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(sq::g_status_word, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "sq_sync_status: clear status word");
    if (word & sq::kErrBounds)
      return fail(SQ_ERR_BOUNDS, "device bounds guard fired (status bits 0x%x)", word);
    return fail(SQ_ERR_TIMEOUT, "device wait timed out (status bits 0x%x: 1 producer, 2 mma, 4 epilogue, 8 teardown)",
                word);
  }
  return SQ_OK;
}

const char* sq_version(void) { return "libsq 0.1 sm_100a"; }

uint64_t sq_kernel_launch_count(void) { return sq::g_launches.load(); }

void sq_debug_arm_fault(int fault, uint64_t wait_limit_ns) {
  g_arm_fault = fault;
  g_arm_limit_ns = wait_limit_ns == 0 ? sq::kDefaultWaitLimitNs : wait_limit_ns;
}

sq_status sq_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int outliers, int64_t* plan) {
  if (plan == nullptr || M <= 0 || N <= 0 || K <= 0)
    return fail(SQ_ERR_INVALID, "sq_debug_gemm_plan: sizes must be positive and plan non-NULL");
  sq::gemm_plan_numbers(M, N, K, outliers != 0, plan);
  return SQ_OK;
}

}  // extern "C"
