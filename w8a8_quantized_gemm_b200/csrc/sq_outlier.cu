// LLM.int8() outlier-column bookkeeping: bitmask, ascending index list, per-word
// prefix counts, and the gather of outlier columns into a dense bf16 operand.
//
// "LLM.int8()技术解析：8位量化如何优化大语言模型计算" §2.1 (a column whose absmax exceeds the
// threshold is an outlier column) and §3.1 (real-time detection marks outlier
// columns in a bitmask; the outlier columns go through a 16-bit GEMM).
#include "sq_internal.h"

#include <algorithm>

namespace sq {
namespace {

constexpr int kMaskThreads = 1024;

// One CTA. Column j is handled by thread j % 1024 of pass j / 1024: a warp covers one
// 32-column mask word, so the ballot is the word and the scan runs over warps. The flags of
// the first kPrefetch passes are computed from loads issued before the scan loop (one memory
// round trip for K <= 8192).
constexpr int kPrefetch = 8;

__global__ void __launch_bounds__(kMaskThreads)
outlier_mask_kernel(const float* __restrict__ amax, int64_t K, float threshold_value,
                    const float* __restrict__ threshold_dev, uint32_t* __restrict__ mask,
                    int32_t* __restrict__ prefix, int32_t* __restrict__ idx, int32_t* __restrict__ count,
                    uint32_t* __restrict__ mask_out, int32_t* __restrict__ count_out) {
  __shared__ int32_t warp_cnt[kMaskThreads / 32];
  __shared__ int32_t warp_off[kMaskThreads / 32];
  __shared__ int32_t running;
  griddep_wait();
  griddep_launch_dependents();
  const float threshold = threshold_dev != nullptr ? __ldg(threshold_dev) : threshold_value;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t words = (K + 31) / 32;
  bool pre[kPrefetch];
#pragma unroll
  for (int i = 0; i < kPrefetch; ++i) {
    const int64_t j = static_cast<int64_t>(i) * kMaskThreads + threadIdx.x;
    pre[i] = (j < K) && (__ldg(amax + j) > threshold);
  }
  if (threadIdx.x == 0) running = 0;
  __syncthreads();
  int pass = 0;
  for (int64_t base = 0; base < K; base += kMaskThreads, ++pass) {
    const int64_t j = base + threadIdx.x;
    bool flag = false;
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i)
      if (i == pass) flag = pre[i];
    if (pass >= kPrefetch) flag = (j < K) && (__ldg(amax + j) > threshold);
    const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_cnt[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
      const int32_t c = warp_cnt[lane];
      int32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      warp_off[lane] = running + incl - c;
    }
    __syncthreads();
    const int64_t word = (base >> 5) + warp;
    if (lane == 0 && word < words) {
      mask[word] = ballot;
      prefix[word] = warp_off[warp];
      if (mask_out) mask_out[word] = ballot;
    }
    if (flag) idx[warp_off[warp] + __popc(ballot & ((1u << lane) - 1u))] = static_cast<int32_t>(j);
    __syncthreads();
    if (threadIdx.x == kMaskThreads - 1) running = warp_off[warp] + __popc(ballot);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    count[0] = running;
    if (count_out) count_out[0] = running;
  }
}

// One thread per row: dst[r, c] = src[r, idx[c]] for c < count, 0 for count <= c <
// roundup(count, 64), written 8 columns (16 bytes) at a time.
__global__ void gather_columns_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t ld,
                                      const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                                      uint16_t* __restrict__ dst, int64_t ld_dst) {
  griddep_wait();
  griddep_launch_dependents();
  const int32_t cnt = __ldg(count);
  const int32_t padded = (cnt + 63) & ~63;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint16_t* srow = src + r * ld;
    uint4* drow = reinterpret_cast<uint4*>(dst + r * ld_dst);
    for (int32_t c0 = 0; c0 < padded; c0 += 8) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int32_t c = c0 + 2 * i;
        const uint32_t lo = c < cnt ? srow[__ldg(idx + c)] : 0u;
        const uint32_t hi = c + 1 < cnt ? srow[__ldg(idx + c + 1)] : 0u;
        w[i] = lo | (hi << 16);
      }
      drow[c0 / 8] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace

cudaError_t launch_outlier_mask(const float* amax, int64_t K, float threshold, const float* threshold_dev,
                                uint32_t* mask, int32_t* prefix, int32_t* idx, int32_t* count, uint32_t* mask_out,
                                int32_t* count_out, cudaStream_t stream) {
  return launch_kernel(outlier_mask_kernel, dim3(1), dim3(kMaskThreads), 0, stream, false, amax, K, threshold,
                       threshold_dev, mask, prefix, idx, count, mask_out, count_out);
}

cudaError_t launch_gather_columns(const uint16_t* src, int64_t rows, int64_t ld, const int32_t* idx,
                                  const int32_t* count, uint16_t* dst, int64_t ld_dst, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = std::min<int64_t>((rows + 127) / 128, static_cast<int64_t>(sms) * 8);
  return launch_kernel(gather_columns_kernel, dim3(static_cast<unsigned>(blocks)), dim3(128), 0, stream, false,
                       src, rows, ld, idx, count, dst, ld_dst);
}

}  // namespace sq
