// Fused smooth + symmetric absmax INT8 quantization of rows (activations per token,
// weights per output channel or per tensor), one HBM pass for the per-row form.
//
// "量化基础与INT8" (对称量化; 量化粒度: per-tensor / per-channel / per-token; 量化流程示例)
// "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §2.3/§3.3/§3.4 (activation divided by
//   s and weight multiplied by s per input channel, fused into one light kernel)
// "LLM.int8()技术解析" §2.1 step 3, §2.2 (outlier columns skipped in the int8 part)
//
// A row is split over TPR threads; each thread owns 16 consecutive elements per
// chunk (two 16-byte bf16 loads, one 16-byte int8 store) and keeps its smoothed
// fp32 values in registers between the absmax reduction (warp shuffles, then
// shared memory across the warps of the row) and the quantization. Rows longer
// than the register budget take a second read (TWO_PASS) that hits L2.
//
// Arithmetic, all IEEE fp32 with no contraction: x' = x * vec[k] (__fmul_rn),
// a = max|x'|, r = 127/a (__fdiv_rn), d = a/127 (__fdiv_rn),
// q = clamp(__float2int_rn(x' * r), -128, 127) (round half to even).
#include "sq_internal.h"

#include <algorithm>

namespace sq {
namespace {

constexpr int kCta = 256;

__device__ __forceinline__ void load16(const uint16_t* p, float (&v)[16]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p + 8));
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void scale16(const float* __restrict__ vec, int64_t k, float (&v)[16]) {
  if (vec == nullptr) return;
  const float4* p = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 f = __ldg(p + i);
    v[4 * i + 0] = __fmul_rn(v[4 * i + 0], f.x);
    v[4 * i + 1] = __fmul_rn(v[4 * i + 1], f.y);
    v[4 * i + 2] = __fmul_rn(v[4 * i + 2], f.z);
    v[4 * i + 3] = __fmul_rn(v[4 * i + 3], f.w);
  }
}

// 16 skip bits for columns k..k+15 (k % 16 == 0).
__device__ __forceinline__ uint32_t skip_bits16(const uint32_t* __restrict__ mask, int64_t k) {
  return (__ldg(mask + (k >> 5)) >> (k & 31)) & 0xFFFFu;
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

__device__ __forceinline__ int q8(float x, float r) {
  int q = __float2int_rn(__fmul_rn(x, r));
  return min(127, max(-128, q));
}

__device__ __forceinline__ void store_q16(int8_t* dst, const float (&v)[16], float r) {
  uint4 o;
  o.x = pack4(q8(v[0], r), q8(v[1], r), q8(v[2], r), q8(v[3], r));
  o.y = pack4(q8(v[4], r), q8(v[5], r), q8(v[6], r), q8(v[7], r));
  o.z = pack4(q8(v[8], r), q8(v[9], r), q8(v[10], r), q8(v[11], r));
  o.w = pack4(q8(v[12], r), q8(v[13], r), q8(v[14], r), q8(v[15], r));
  *reinterpret_cast<uint4*>(dst) = o;
}

// Max over the TPR threads of one row group; every thread of the group gets the result.
template <int TPR>
__device__ __forceinline__ float group_max(float a, float* red /* [kCta/32] */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if constexpr (TPR > 32) {
    constexpr int kWarpsPerGroup = TPR / 32;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g0 = (warp / kWarpsPerGroup) * kWarpsPerGroup;
    if (lane == 0) red[warp] = a;
    __syncthreads();
    float t = red[g0];
#pragma unroll
    for (int w = 1; w < kWarpsPerGroup; ++w) t = fmaxf(t, red[g0 + w]);
    __syncthreads();
    a = t;
  }
  return a;
}

enum Mode { kPerRow = 0, kTensorMax = 1, kTensorQuant = 2 };

// Load 16 elements of a row starting at column k, zero the LLM.int8 outlier columns
// (copying their bf16 values to the gathered matrix when `gather`), then smooth.
template <bool OUTLIERS>
__device__ __forceinline__ void load_chunk(const uint16_t* __restrict__ srow, int64_t row, int64_t k,
                                           const float* __restrict__ vec, const OutlierView& ov, bool gather,
                                           float (&v)[16]) {
  load16(srow + k, v);
  if constexpr (OUTLIERS) {
    const uint32_t sk = skip_bits16(ov.mask, k);
    if (sk) {
      const int64_t w = k >> 5;
      int32_t pos = __ldg(ov.prefix + w) + __popc(__ldg(ov.mask + w) & ((1u << (k & 31)) - 1u));
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((sk >> i) & 1u) {
          if (gather) ov.gathered[row * ov.ld_gathered + pos] = srow[k + i];
          ++pos;
          v[i] = 0.0f;
        }
      }
    }
  }
  scale16(vec, k, v);
}

// Grid: one row group per (blockIdx.x, threadIdx.x / TPR); CTA = max(kCta, TPR) threads.
template <int TPR, int CHUNKS, bool TWO_PASS, bool OUTLIERS, int MODE>
__global__ void __launch_bounds__(TPR > kCta ? TPR : kCta)
quant_rows_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                  const float* __restrict__ vec, OutlierView ov, int8_t* __restrict__ q,
                  float* __restrict__ scale, unsigned int* __restrict__ gmax_bits) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  constexpr int kGroups = kThreads / TPR;
  __shared__ float red[kThreads / 32];
  const int g = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kGroups + g;
  const bool row_ok = row < rows;
  const uint16_t* srow = src + (row_ok ? row : 0) * ld;
  const int64_t step = static_cast<int64_t>(TPR) * 16;

  float a = 0.0f;
  float v[TWO_PASS ? 1 : CHUNKS][16];
  if constexpr (!TWO_PASS) {
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int64_t k = c * step + t * 16;
      if (row_ok && k < K) {
        load_chunk<OUTLIERS>(srow, row, k, vec, ov, MODE != kTensorMax, v[c]);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[c][i]));
      }
    }
  } else if constexpr (MODE != kTensorQuant) {
    for (int64_t k = t * 16; row_ok && k < K; k += step) {
      float w[16];
      load_chunk<OUTLIERS>(srow, row, k, vec, ov, false, w);
#pragma unroll
      for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
    }
  }

  if constexpr (MODE == kTensorQuant) {
    a = __uint_as_float(*reinterpret_cast<volatile unsigned int*>(gmax_bits));
  } else {
    a = group_max<TPR>(a, red);
  }

  if constexpr (MODE == kTensorMax) {
    if (t == 0 && row_ok) atomicMax(gmax_bits, __float_as_uint(a));
  } else {
    const float r = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    if (row_ok) {
      if constexpr (MODE == kPerRow) {
        if (t == 0) scale[row] = __fdiv_rn(a, 127.0f);
      } else {
        if (t == 0 && row == 0) scale[0] = __fdiv_rn(a, 127.0f);
      }
      int8_t* qrow = q + row * K;
      if constexpr (!TWO_PASS) {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const int64_t k = c * step + t * 16;
          if (k < K) store_q16(qrow + k, v[c], r);
        }
      } else {
        for (int64_t k = t * 16; k < K; k += step) {
          float w[16];
          load_chunk<OUTLIERS>(srow, row, k, vec, ov, true, w);
          store_q16(qrow + k, w, r);
        }
      }
      if constexpr (OUTLIERS) {
        // zero the padding of the gathered row up to the next multiple of 64 columns
        const int32_t cnt = __ldg(ov.count);
        const int32_t padded = (cnt + 63) & ~63;
        for (int32_t c = cnt + t; c < padded; c += TPR) ov.gathered[row * ov.ld_gathered + c] = 0;
      }
    }
  }
}

template <int TPR, int CHUNKS, bool TWO_PASS, bool OUTLIERS, int MODE>
cudaError_t launch_t(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                     const OutlierView& ov, int8_t* q, float* scale, unsigned int* gmax, cudaStream_t stream) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  constexpr int kGroups = kThreads / TPR;
  const int64_t blocks = (rows + kGroups - 1) / kGroups;
  note_launch();
  quant_rows_kernel<TPR, CHUNKS, TWO_PASS, OUTLIERS, MODE>
      <<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(src, rows, K, ld, vec, ov, q, scale, gmax);
  return cudaGetLastError();
}

// Shape dispatch: the smallest threads-per-row that keeps <= 32 (<= 64 for long rows)
// smoothed values per thread in registers.
template <bool OUTLIERS, int MODE>
cudaError_t dispatch(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                     const OutlierView& ov, int8_t* q, float* scale, unsigned int* gmax, cudaStream_t stream) {
  if (K <= 512) return launch_t<32, 1, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  if (K <= 1024) return launch_t<32, 2, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  if (K <= 2048) return launch_t<64, 2, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  if (K <= 4096) return launch_t<128, 2, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  if (K <= 8192) return launch_t<256, 2, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  if (K <= 16384) return launch_t<512, 2, false, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
  return launch_t<512, 1, true, OUTLIERS, MODE>(src, rows, K, ld, vec, ov, q, scale, gmax, stream);
}

}  // namespace

cudaError_t launch_quant_rows(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                              const OutlierView& ov, int8_t* q, float* scale, cudaStream_t stream) {
  if (ov.mask != nullptr) return dispatch<true, kPerRow>(src, rows, K, ld, vec, ov, q, scale, nullptr, stream);
  return dispatch<false, kPerRow>(src, rows, K, ld, vec, ov, q, scale, nullptr, stream);
}

cudaError_t launch_quant_tensor(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                                unsigned int* gmax_bits, int8_t* q, float* scale1, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(gmax_bits, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  OutlierView none;
  e = dispatch<false, kTensorMax>(src, rows, K, ld, vec, none, nullptr, nullptr, gmax_bits, stream);
  if (e != cudaSuccess) return e;
  return dispatch<false, kTensorQuant>(src, rows, K, ld, vec, none, q, scale1, gmax_bits, stream);
}

}  // namespace sq
