// Internal launch interfaces shared by the translation units of libsq.
// Every launcher returns the status of enqueueing its work on `stream`.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <utility>

namespace sq {

// Bit flags of the per-device error word written by kernels with bounded waits.
enum : unsigned int {
  kErrProducerWait = 1u,
  kErrMmaWait = 2u,
  kErrEpilogueWait = 4u,
  kErrTeardownWait = 8u,
  kErrBounds = 16u,  // a device-side bounds guard fired (builds with SQ_DEBUG_GUARDS only)
};

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s per wait

// Device address of the error word of the current device.
unsigned int* device_status_word();

// Host-side count of kernels this library has launched (diagnostics).
void note_launch();

// Records the message returned by sq_last_error() on this thread; returns st.
int record_error(int st, const char* msg);

// Kernel launch used for every kernel of the library. Each kernel executes griddep_wait()
// in every thread before its first global-memory access and griddep_launch_dependents()
// once it has started. With `programmatic` set, the grid is launched with programmatic
// stream serialization: it may be scheduled while the previous kernel on the stream is
// still finishing, so its launch and set-up (barrier init, TMEM allocation, descriptor
// prefetch) overlap that kernel's tail; the wait returns once the previous grid has
// completed and its writes are visible, so the stream order of the data is unchanged.
// The GEMM launches and the short, latency-bound launches take it: measured on the whole
// SmoothQuant + LLM.int8 step (2048 x 11008 x 4096), setting it on every launch made the step
// 1-3% slower, on the GEMM launches alone about 1% faster, and a 4096 x 4096 decode GEMM gains
// ~0.8 us (of ~10.6).
// `cluster_x` > 1 groups consecutive CTAs into clusters of that many (CTA pairs: 2).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    bool programmatic, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = programmatic ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  note_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          bool programmatic, Args&&... args) {
  return launch_kernel_clustered(kernel, grid, block, smem, stream, programmatic, 1u, std::forward<Args>(args)...);
}

#ifdef __CUDACC__
// Device-side bounds guards. In the SQ_DEBUG_GUARDS build (libsq_debug.so) SQ_GUARD(c) checks
// c, and when it is false records kErrBounds in the device error word (sq_sync_status then
// reports SQ_ERR_BOUNDS) so that the caller skips the access; in the product build it is the
// constant true and costs nothing.
#ifdef SQ_DEBUG_GUARDS
extern __device__ unsigned int g_status_word;
__device__ __forceinline__ bool guard_ok(bool c) {
  if (!c) atomicOr(&g_status_word, kErrBounds);
  return c;
}
#define SQ_GUARD(c) (::sq::guard_ok(c))
#else
#define SQ_GUARD(c) true
#endif

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

// ---- reductions (sq_reduce.cu)
// words[0..n) = 0.
cudaError_t launch_zero_words(uint32_t* words, int64_t n, cudaStream_t stream);
// Column absmax of a bf16 [rows, K] matrix into amax (fp32 [K]); with `accumulate` the
// maximum with the values amax already holds. One launch, no reset.
cudaError_t launch_col_absmax(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, float* amax,
                              bool accumulate, cudaStream_t stream);
// Smoothing factors s / inv_s from act_amax and the column absmax of W, in one pass over W.
cudaError_t launch_smooth_scale(const float* act_amax, const uint16_t* W, int64_t N, int64_t K, int64_t ldw,
                                float alpha, float* s, float* inv_s, cudaStream_t stream);

// ---- row quantization (sq_quant.cu)
struct OutlierView {
  const uint32_t* mask = nullptr;    // [ceil(K/32)] skip bits (nullptr: no skipping)
  const int32_t* prefix = nullptr;   // [ceil(K/32)] outliers before each word
  const int32_t* count = nullptr;    // [1] number of outliers
  uint16_t* gathered = nullptr;      // [rows, ld_gathered] bf16 outlier values (zero padded to 64)
  int64_t ld_gathered = 0;
  // the same kernel also gathers the weight's outlier columns (one thread per weight row):
  const uint16_t* w_src = nullptr;   // [w_rows, w_ld] bf16, or nullptr
  int64_t w_rows = 0, w_ld = 0;
  const int32_t* idx = nullptr;      // [count] ascending outlier column indices
  uint16_t* w_gathered = nullptr;    // [w_rows, ld_gathered]
};

// Per-row smooth + quantize: q[r,k] = clamp(rne(src[r,k]*vec[k] * 127/a_r)), scale[r] = a_r/127.
cudaError_t launch_quant_rows(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                              const OutlierView& ov, int8_t* q, float* scale, cudaStream_t stream);
// Per-tensor: global absmax of src*vec into *gmax_bits (reset first), then quantize with it;
// with `clip` (device fp32 [1]) no maximum is taken and *clip is used instead.
cudaError_t launch_quant_tensor(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                                unsigned int* gmax_bits, int8_t* q, float* scale1, cudaStream_t stream,
                                const float* clip = nullptr);
// Asymmetric per-row: scale[r] = range/255, zero[r] = -128 - rne(lo * 255/range).
cudaError_t launch_quant_rows_asym(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                                   int8_t* q, float* scale, int32_t* zero, cudaStream_t stream);

// ---- LLM.int8 outlier bookkeeping (sq_outlier.cu)
// Outlier columns amax_j > threshold (threshold_dev, device fp32 [1], replaces the value when
// given).
cudaError_t launch_outlier_mask(const float* amax, int64_t K, float threshold, const float* threshold_dev,
                                uint32_t* mask, int32_t* prefix, int32_t* idx, int32_t* count, uint32_t* mask_out,
                                int32_t* count_out, cudaStream_t stream);

// ---- variants (sq_variants.cu)
// s <- max(s / max(s) * 127, 1e-5), inv_s = 1/s (one CTA).
cudaError_t launch_normalize_scale(float* s, float* inv_s, int64_t K, cudaStream_t stream);
// rowsum[n] = sum_k Wq[n,k].
cudaError_t launch_row_sums(const int8_t* Wq, int64_t N, int64_t K, int32_t* rowsum, cudaStream_t stream);
// LayerNorm (norm 0) / RMSNorm (norm 1) + smoothing + per-row quantization; K <= 16384.
cudaError_t launch_norm_quant(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, int norm,
                              const uint16_t* gamma, const uint16_t* beta, float eps, const float* vec, int8_t* q,
                              float* scale, float* mean_rstd, cudaStream_t stream);
// threshold = fp32(mean + k * std) over all elements; ws of mean_std_workspace_bytes(rows).
size_t mean_std_workspace_bytes(int64_t rows);
cudaError_t launch_mean_std_threshold(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, double k,
                                      float* threshold, double* mean_std, void* ws, cudaStream_t stream);
// *out = the element of 1-based rank `rank` of the ascending |src|; ws of abs_percentile_workspace_bytes().
size_t abs_percentile_workspace_bytes();
cudaError_t launch_abs_percentile(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, uint64_t rank,
                                  float* out, void* ws, cudaStream_t stream);

// ---- tensor-core GEMM (sq_gemm.cu)
struct GemmArgs {
  const int8_t* Xq = nullptr;       // [M, K]
  const int8_t* Wq = nullptr;       // [N, K]
  const float* x_scale = nullptr;   // [M] (x_per_token) or [1]
  bool x_per_token = true;
  const int32_t* x_zero = nullptr;  // [M] asymmetric-activation zero points, or nullptr
  const int32_t* w_rowsum = nullptr;// [N] sum_k Wq[n,k] (with x_zero)
  const float* w_scale = nullptr;   // [N] or [1]
  bool w_per_channel = true;
  const uint16_t* bias = nullptr;   // [N] bf16 or nullptr
  uint16_t* Y = nullptr;            // [M, N] bf16
  int32_t* acc_out = nullptr;       // [M, N] or nullptr
  int64_t M = 0, N = 0, K = 0;
  // LLM.int8 outlier operands (bf16, K-contiguous, leading dimension ld_o), or nullptr.
  const uint16_t* Xo = nullptr;     // [M, ld_o]
  const uint16_t* Wo = nullptr;     // [N, ld_o]
  const int32_t* o_count = nullptr; // [1] number of outlier columns (device)
  int64_t ld_o = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  uint64_t wait_limit_ns = kDefaultWaitLimitNs;
  int fault = 0;                    // test hook: 1 = producer withholds one stage
};
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, bool outliers);
// The launch plan of launch_gemm as 7 numbers (see sq_debug_gemm_plan).
void gemm_plan_numbers(int64_t M, int64_t N, int64_t K, bool outliers, int64_t* out);
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream, const char** why);

// ---- CUDA-core product for M <= 4 tokens (sq_gemv.cu): same arguments and results as the GEMM.
bool gemv_applies(int64_t M, int64_t K, bool outliers);
cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t stream);

}  // namespace sq
