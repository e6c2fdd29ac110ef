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
// Asymmetric rows ("量化基础与INT8" 非对称量化, over the range extended to contain 0):
// lo = min(0, min x'), hi = max(0, max x'), range = hi - lo, r = 255/range, d = range/255,
// z = -128 - rne(lo * r), q = clamp(rne(x' * r) + z, -128, 127).
#include "sq_internal.h"
#include "sq_rows.cuh"

#include <algorithm>

namespace sq {
namespace {

using namespace rows;

// 16 skip bits for columns k..k+15 (k % 16 == 0).
__device__ __forceinline__ uint32_t skip_bits16(const uint32_t* __restrict__ mask, int64_t k) {
  return (__ldg(mask + (k >> 5)) >> (k & 31)) & 0xFFFFu;
}

enum Mode { kPerRow = 0, kTensorMax = 1, kTensorQuant = 2, kAsym = 3 };

// Zero the LLM.int8 outlier columns among k..k+15 (copying their bf16 values to the gathered
// matrix when `gather`), then smooth with the thread's slice of the vector (if any).
template <bool OUTLIERS, bool HAS_VEC>
__device__ __forceinline__ void finish_chunk(const uint4 (&r)[2], int64_t row, int64_t k, const float (&vs)[16],
                                             const OutlierView& ov, bool gather, float (&v)[16]) {
  widen16(r, v);
  if constexpr (OUTLIERS) {
    const uint32_t sk = skip_bits16(ov.mask, k);
    if (sk) {
      const int64_t w = k >> 5;
      int32_t pos = __ldg(ov.prefix + w) + __popc(__ldg(ov.mask + w) & ((1u << (k & 31)) - 1u));
      const uint16_t* h = reinterpret_cast<const uint16_t*>(&r[0]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((sk >> i) & 1u) {
          if (gather && SQ_GUARD(pos >= 0 && pos < ov.ld_gathered)) ov.gathered[row * ov.ld_gathered + pos] = h[i];
          ++pos;
          v[i] = 0.0f;
        }
      }
    }
  }
  if constexpr (HAS_VEC) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], vs[i]);
  }
}

// Persistent over rows: CTA = max(kCta, TPR) threads = kGroups row groups of TPR threads;
// the groups walk the rows with a grid stride. A thread keeps its slice of the smoothing
// vector in registers for all its rows and prefetches its next row's bf16 data before the
// current row's absmax reduction.
template <int TPR, int CHUNKS, bool TWO_PASS, bool OUTLIERS, bool HAS_VEC, int MODE>
__global__ void __launch_bounds__(TPR > kCta ? TPR : kCta)
quant_rows_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                  const float* __restrict__ vec, OutlierView ov, int8_t* __restrict__ q,
                  float* __restrict__ scale, unsigned int* __restrict__ gmax_bits, int32_t* __restrict__ zero) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  griddep_wait();
  griddep_launch_dependents();
  constexpr int kGroups = kThreads / TPR;
  constexpr int kVC = (HAS_VEC && !TWO_PASS) ? CHUNKS : 1;
  __shared__ float red[kThreads / 32];
  const int g = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int64_t step = static_cast<int64_t>(TPR) * 16;
  const int64_t row_stride = static_cast<int64_t>(gridDim.x) * kGroups;

  if constexpr (OUTLIERS) {
    if (ov.w_src != nullptr) {
      // the weight's outlier columns first, a warp per weight row, spread over every CTA
      // (warp w of CTA b takes rows b + w * grid, then every grid * warps rows):
      // w_gathered[r, c] = w[r, idx[c]] for c < count, 0 up to the next multiple of 64. Lane
      // l gathers the column pair (2l, 2l + 1) of each 64-column block: its loads of the
      // scattered weight values are independent, so a row costs about one memory round trip,
      // and the warp stores 128 contiguous bytes per block.
      const int32_t cnt = __ldg(ov.count);
      const int32_t padded = (cnt + 63) & ~63;
      const int lane = threadIdx.x & 31;
      constexpr int kWarpsPerCta = kThreads / 32;
      for (int64_t r = static_cast<int64_t>(threadIdx.x >> 5) * gridDim.x + blockIdx.x; padded > 0 && r < ov.w_rows;
           r += static_cast<int64_t>(gridDim.x) * kWarpsPerCta) {
        const uint16_t* srow = ov.w_src + r * ov.w_ld;
        uint32_t* drow = reinterpret_cast<uint32_t*>(ov.w_gathered + r * ov.ld_gathered);
        for (int32_t c0 = 0; c0 < padded; c0 += 64) {
          const int32_t c = c0 + 2 * lane;
          const int32_t jl = c < cnt ? __ldg(ov.idx + c) : 0;
          const int32_t jh = c + 1 < cnt ? __ldg(ov.idx + c + 1) : 0;
          const uint32_t lo = (c < cnt && SQ_GUARD(jl >= 0 && jl < ov.w_ld)) ? srow[jl] : 0u;
          const uint32_t hi = (c + 1 < cnt && SQ_GUARD(jh >= 0 && jh < ov.w_ld)) ? srow[jh] : 0u;
          if (SQ_GUARD(c + 2 <= ov.ld_gathered)) drow[c / 2] = lo | (hi << 16);
        }
      }
    }
  }

  float vs[kVC][16];
  if constexpr (HAS_VEC && !TWO_PASS) {
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int64_t k = c * step + t * 16;
      if (k < K) {
        const float4* p4 = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 f = __ldg(p4 + i);
          vs[c][4 * i] = f.x;
          vs[c][4 * i + 1] = f.y;
          vs[c][4 * i + 2] = f.z;
          vs[c][4 * i + 3] = f.w;
        }
      }
    }
  }

  uint4 raw[TWO_PASS ? 1 : CHUNKS][2];
  int64_t row = static_cast<int64_t>(blockIdx.x) * kGroups + g;
  if constexpr (!TWO_PASS) {
    if (row < rows) {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int64_t k = c * step + t * 16;
        if (k < K) raw16(src + row * ld + k, raw[c]);
      }
    }
  }

  // uniform trip count across the CTA (block-wide reductions inside)
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kGroups; base < rows; base += row_stride, row += row_stride) {
    const bool row_ok = row < rows;
    const uint16_t* srow = src + (row_ok ? row : 0) * ld;
    float a = 0.0f;
    float lo = 0.0f;  // kAsym: a holds max(0, max x'), lo holds min(0, min x')
    float v[TWO_PASS ? 1 : CHUNKS][16];
    if constexpr (!TWO_PASS) {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int64_t k = c * step + t * 16;
        if (row_ok && k < K) {
          finish_chunk<OUTLIERS, HAS_VEC>(raw[c], row, k, vs[HAS_VEC ? c : 0], ov, MODE != kTensorMax, v[c]);
          if constexpr (MODE == kAsym) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              a = fmaxf(a, v[c][i]);
              lo = fminf(lo, v[c][i]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[c][i]));
          }
        }
      }
      // prefetch this thread's next row while the current one is reduced
      const int64_t nrow = row + row_stride;
      if (nrow < rows) {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const int64_t k = c * step + t * 16;
          if (k < K) raw16(src + nrow * ld + k, raw[c]);
        }
      }
    } else if constexpr (MODE != kTensorQuant) {
      for (int64_t k = t * 16; row_ok && k < K; k += step) {
        uint4 r[2];
        float w[16], vv[16];
        raw16(srow + k, r);
        if constexpr (HAS_VEC) {
          const float4* p4 = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 f = __ldg(p4 + i);
            vv[4 * i] = f.x; vv[4 * i + 1] = f.y; vv[4 * i + 2] = f.z; vv[4 * i + 3] = f.w;
          }
        }
        finish_chunk<OUTLIERS, HAS_VEC>(r, row, k, vv, ov, false, w);
        if constexpr (MODE == kAsym) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            a = fmaxf(a, w[i]);
            lo = fminf(lo, w[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
        }
      }
    }

    if constexpr (MODE == kTensorQuant) {
      a = __uint_as_float(*reinterpret_cast<volatile unsigned int*>(gmax_bits));
    } else if constexpr (MODE == kAsym) {
      a = group_max<TPR>(a, red);
      lo = -group_max<TPR>(-lo, red);
    } else {
      a = group_max<TPR>(a, red);
    }

    if constexpr (MODE == kAsym) {
      const float range = __fsub_rn(a, lo);
      const float r = range > 0.0f ? __fdiv_rn(255.0f, range) : 0.0f;
      const int z = -128 - __float2int_rn(__fmul_rn(lo, r));
      if (row_ok) {
        if (t == 0) {
          scale[row] = __fdiv_rn(range, 255.0f);
          zero[row] = z;
        }
        int8_t* qrow = q + row * K;
        if constexpr (!TWO_PASS) {
#pragma unroll
          for (int c = 0; c < CHUNKS; ++c) {
            const int64_t k = c * step + t * 16;
            if (k < K) store_q16z(qrow + k, v[c], r, z);
          }
        } else {
          for (int64_t k = t * 16; k < K; k += step) {
            uint4 rr[2];
            float w[16], vv[16];
            raw16(srow + k, rr);
            if constexpr (HAS_VEC) {
              const float4* p4 = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 f = __ldg(p4 + i);
                vv[4 * i] = f.x; vv[4 * i + 1] = f.y; vv[4 * i + 2] = f.z; vv[4 * i + 3] = f.w;
              }
            }
            finish_chunk<false, HAS_VEC>(rr, row, k, vv, ov, false, w);
            store_q16z(qrow + k, w, r, z);
          }
        }
      }
    } else if constexpr (MODE == kTensorMax) {
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
            if (k < K) {
              if constexpr (MODE == kPerRow)
                store_q16_own_max(qrow + k, v[c], r);
              else
                store_q16(qrow + k, v[c], r);
            }
          }
        } else {
          for (int64_t k = t * 16; k < K; k += step) {
            uint4 rr[2];
            float w[16], vv[16];
            raw16(srow + k, rr);
            if constexpr (HAS_VEC) {
              const float4* p4 = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 f = __ldg(p4 + i);
                vv[4 * i] = f.x; vv[4 * i + 1] = f.y; vv[4 * i + 2] = f.z; vv[4 * i + 3] = f.w;
              }
            }
            finish_chunk<OUTLIERS, HAS_VEC>(rr, row, k, vv, ov, true, w);
            if constexpr (MODE == kPerRow)
              store_q16_own_max(qrow + k, w, r);
            else
              store_q16(qrow + k, w, r);
          }
        }
        if constexpr (OUTLIERS) {
          // zero the padding of the gathered row up to the next multiple of 64 columns
          const int32_t cnt = __ldg(ov.count);
          const int32_t padded = (cnt + 63) & ~63;
          for (int32_t c = cnt + t; c < padded; c += TPR)
            if (SQ_GUARD(c < ov.ld_gathered)) ov.gathered[row * ov.ld_gathered + c] = 0;
        }
      }
    }
  }

}

int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  return sms;
}

// One resident wave: as many CTAs as fit on every SM at once (registers decide); the
// row-group loop and the prefetch of the next row keep the loads in flight.
template <typename Kernel>
int64_t resident_grid(Kernel kernel, int threads, int64_t groups, int& per_sm_cache) {
  if (per_sm_cache <= 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    per_sm_cache = per_sm;
  }
  return std::min<int64_t>(groups, static_cast<int64_t>(num_sms()) * per_sm_cache);
}

// A decode step's activation rows (up to 64 tokens) are a short, latency-bound launch: it
// takes programmatic dependent launch like the decode GEMM, so its launch and set-up overlap
// the previous kernel's tail (measured on the decode step quantization + GEMM, 4096 x 4096:
// 5.7 / 8.6 / 12.2 / 13.1 -> 5.5 / 8.2 / 11.4 / 12.6 us at 1 / 4 / 16 / 64 tokens).
constexpr int64_t kShortRows = 64;

template <int TPR, int CHUNKS, bool TWO_PASS, bool OUTLIERS, int MODE>
cudaError_t launch_t(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                     const OutlierView& ov, int8_t* q, float* scale, unsigned int* gmax, int32_t* zero,
                     cudaStream_t stream) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  constexpr int kGroups = kThreads / TPR;
  const int64_t groups = (rows + kGroups - 1) / kGroups;
  if (vec != nullptr) {
    static int per_sm = 0;
    auto kernel = quant_rows_kernel<TPR, CHUNKS, TWO_PASS, OUTLIERS, true, MODE>;
    const int64_t blocks = resident_grid(kernel, kThreads, groups, per_sm);
    return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, stream, rows <= kShortRows,
                         src, rows, K, ld, vec, ov, q, scale, gmax, zero);
  }
  static int per_sm = 0;
  auto kernel = quant_rows_kernel<TPR, CHUNKS, TWO_PASS, OUTLIERS, false, MODE>;
  const int64_t blocks = resident_grid(kernel, kThreads, groups, per_sm);
  return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, stream, rows <= kShortRows, src,
                       rows, K, ld, vec, ov, q, scale, gmax, zero);
}

// Shape dispatch: one 16-element chunk per thread up to K = 4096 (a row over up to 256
// threads, few registers, several CTAs per SM); longer rows take two chunks per thread, and
// rows longer than 16384 the two-read path. (Measured: one chunk per thread is faster at
// K = 4096, two chunks at K = 8192.)
template <bool OUTLIERS, int MODE>
cudaError_t dispatch(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                     const OutlierView& ov, int8_t* q, float* scale, unsigned int* gmax, cudaStream_t stream,
                     int32_t* zero = nullptr) {
  if (K <= 512) return launch_t<32, 1, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  if (K <= 1024) return launch_t<64, 1, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  if (K <= 2048) return launch_t<128, 1, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  if (K <= 4096) return launch_t<256, 1, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  if (K <= 8192) return launch_t<256, 2, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  if (K <= 16384) return launch_t<512, 2, false, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
  return launch_t<512, 1, true, OUTLIERS, MODE>(
      src, rows, K, ld, vec, ov, q, scale, gmax, zero, stream);
}

}  // namespace

cudaError_t launch_quant_rows(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                              const OutlierView& ov, int8_t* q, float* scale, cudaStream_t stream) {
  if (ov.mask != nullptr) return dispatch<true, kPerRow>(src, rows, K, ld, vec, ov, q, scale, nullptr, stream);
  return dispatch<false, kPerRow>(src, rows, K, ld, vec, ov, q, scale, nullptr, stream);
}

cudaError_t launch_quant_tensor(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                                unsigned int* gmax_bits, int8_t* q, float* scale1, cudaStream_t stream,
                                const float* clip) {
  OutlierView none;
  if (clip != nullptr) {
    // a calibrated value: one pass, the kernel reads the maximum from `clip`
    unsigned int* c = reinterpret_cast<unsigned int*>(const_cast<float*>(clip));
    return dispatch<false, kTensorQuant>(src, rows, K, ld, vec, none, q, scale1, c, stream);
  }
  cudaError_t e = launch_zero_words(gmax_bits, 1, stream);
  if (e != cudaSuccess) return e;
  e = dispatch<false, kTensorMax>(src, rows, K, ld, vec, none, nullptr, nullptr, gmax_bits, stream);
  if (e != cudaSuccess) return e;
  return dispatch<false, kTensorQuant>(src, rows, K, ld, vec, none, q, scale1, gmax_bits, stream);
}

cudaError_t launch_quant_rows_asym(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const float* vec,
                                   int8_t* q, float* scale, int32_t* zero, cudaStream_t stream) {
  return dispatch<false, kAsym>(src, rows, K, ld, vec, OutlierView{}, q, scale, nullptr, stream, zero);
}

}  // namespace sq
