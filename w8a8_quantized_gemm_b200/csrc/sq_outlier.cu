// LLM.int8() outlier-column bookkeeping: bitmask, ascending index list and per-word prefix
// counts (the gathers of the outlier columns run inside the masked row quantization).
//
// "LLM.int8()技术解析：8位量化如何优化大语言模型计算" §2.1 (a column whose absmax exceeds the
// threshold is an outlier column) and §3.1 (real-time detection marks outlier
// columns in a bitmask; the outlier columns go through a 16-bit GEMM).
#include "sq_internal.h"

#include <algorithm>

namespace sq {
namespace {

constexpr int kMaskThreads = 1024;
constexpr int kMaskWarps = kMaskThreads / 32;
constexpr int kMaxWords = 65536 / 32;  // K <= 65536

// One CTA. Warp w owns the mask words [w*wpw, (w+1)*wpw), wpw = ceil(words/32); in batch b
// lane l handles word w*wpw + 32b + l and reads its 32 column maxima (128 contiguous bytes).
// Pass 1 forms the words (kept in shared memory) and each warp's outlier count; one scan
// over the 32 warp counts gives each warp's base; pass 2 scans the words' popcounts within
// the warp, batch by batch, and writes each word, its prefix and the ascending index list.
// Two block-wide barriers in all, whatever K.
__global__ void __launch_bounds__(kMaskThreads)
outlier_mask_kernel(const float* __restrict__ amax, int64_t K, float threshold_value,
                    const float* __restrict__ threshold_dev, uint32_t* __restrict__ mask,
                    int32_t* __restrict__ prefix, int32_t* __restrict__ idx, int32_t* __restrict__ count,
                    uint32_t* __restrict__ mask_out, int32_t* __restrict__ count_out) {
  __shared__ uint32_t words_s[kMaxWords];
  __shared__ int32_t warp_base[kMaskWarps + 1];
  griddep_wait();
  griddep_launch_dependents();
  const float threshold = threshold_dev != nullptr ? __ldg(threshold_dev) : threshold_value;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t words = (K + 31) / 32;
  const int64_t wpw = (words + kMaskWarps - 1) / kMaskWarps;
  const int64_t w_begin = warp * wpw;
  const int64_t w_end = w_begin + wpw < words ? w_begin + wpw : words;

  // pass 1: the words and this warp's count
  int32_t warp_total = 0;
  for (int64_t b0 = w_begin; b0 < w_end; b0 += 32) {
    const int64_t word = b0 + lane;
    uint32_t bits = 0u;
    if (word < w_end) {
      const int64_t j0 = word * 32;
      if (j0 + 32 <= K) {
        const float4* p = reinterpret_cast<const float4*>(amax + j0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = __ldg(p + q);
          bits |= (v.x > threshold ? 1u : 0u) << (4 * q);
          bits |= (v.y > threshold ? 1u : 0u) << (4 * q + 1);
          bits |= (v.z > threshold ? 1u : 0u) << (4 * q + 2);
          bits |= (v.w > threshold ? 1u : 0u) << (4 * q + 3);
        }
      } else {
        for (int i = 0; i < 32 && j0 + i < K; ++i) bits |= (__ldg(amax + j0 + i) > threshold ? 1u : 0u) << i;
      }
      words_s[word] = bits;
    }
    int32_t c = __popc(bits);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    warp_total += c;
  }
  if (lane == 0) warp_base[warp] = warp_total;
  __syncthreads();
  if (warp == 0) {
    const int32_t c = warp_base[lane];
    int32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __syncwarp();
    warp_base[lane] = incl - c;
    if (lane == 31) warp_base[kMaskWarps] = incl;
  }
  __syncthreads();

  // pass 2: prefixes and the index list
  int32_t running = warp_base[warp];
  for (int64_t b0 = w_begin; b0 < w_end; b0 += 32) {
    const int64_t word = b0 + lane;
    const uint32_t bits = word < w_end ? words_s[word] : 0u;
    const int32_t c = __popc(bits);
    int32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int32_t excl = running + incl - c;
    if (word < w_end) {
      mask[word] = bits;
      prefix[word] = excl;
      if (mask_out) mask_out[word] = bits;
      uint32_t rest = bits;
      int32_t pos = excl;
      while (rest) {
        const int i = __ffs(rest) - 1;
        if (SQ_GUARD(pos < K && word * 32 + i < K)) idx[pos] = static_cast<int32_t>(word * 32 + i);
        ++pos;
        rest &= rest - 1u;
      }
    }
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (threadIdx.x == 0) {
    count[0] = warp_base[kMaskWarps];
    if (count_out) count_out[0] = warp_base[kMaskWarps];
  }
}

}  // namespace

cudaError_t launch_outlier_mask(const float* amax, int64_t K, float threshold, const float* threshold_dev,
                                uint32_t* mask, int32_t* prefix, int32_t* idx, int32_t* count, uint32_t* mask_out,
                                int32_t* count_out, cudaStream_t stream) {
  return launch_kernel(outlier_mask_kernel, dim3(1), dim3(kMaskThreads), 0, stream, false, amax, K, threshold,
                       threshold_dev, mask, prefix, idx, count, mask_out, count_out);
}

}  // namespace sq
