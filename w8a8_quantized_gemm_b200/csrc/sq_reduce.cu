// Column-wise absolute maximum (calibration statistic and LLM.int8 column detection)
// and the SmoothQuant smoothing factors.
//
// "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §3.2 (per-channel amax over the
// token dimensions, running maximum across batches) and §2.1/§3.3 (smoothing factor);
// "LLM.int8()技术解析" §2.1 step 1 (column-wise absolute maximum of the input).
//
// HBM-bound: each element of the source is read once with 16-byte loads; a warp
// covers 256 consecutive columns of one row (512 contiguous bytes). Partial maxima
// from the warps of a CTA meet in shared memory and go to global memory with one
// atomicMax per column per CTA (non-negative floats order like their bit patterns).
#include "sq_internal.h"

#include <algorithm>

namespace sq {
namespace {

constexpr int kColWarps = 8;          // warps per CTA
constexpr int kColsPerCta = 256;      // 32 lanes x 8 bf16
constexpr int kRowUnroll = 4;         // independent 16-byte loads in flight per thread

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kColWarps * 32)
col_absmax_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int64_t rows_per_cta,
                  unsigned int* __restrict__ out_bits) {
  __shared__ float part[kColWarps][kColsPerCta];
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kColsPerCta + lane * 8;
  const bool col_ok = col0 < K;  // K % 16 == 0, so a lane's 8 columns are all in or all out
  const int64_t r_begin = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r_end = min(rows, r_begin + rows_per_cta);

  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;

  if (col_ok) {
    const uint16_t* base = src + col0;
    int64_t r = r_begin + warp;
    // kRowUnroll rows per step so that several loads are outstanding per thread
    for (; r + (kRowUnroll - 1) * kColWarps < r_end; r += kRowUnroll * kColWarps) {
      uint4 v[kRowUnroll];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(base + (r + u * kColWarps) * ld));
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          m[2 * i] = fmaxf(m[2 * i], fabsf(bf16lo(w[i])));
          m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16hi(w[i])));
        }
      }
    }
    for (; r < r_end; r += kColWarps) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + r * ld));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        m[2 * i] = fmaxf(m[2 * i], fabsf(bf16lo(w[i])));
        m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16hi(w[i])));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[warp][lane * 8 + i] = m[i];
  __syncthreads();
  const int c = threadIdx.x;  // one column per thread (256 threads, 256 columns)
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColsPerCta + c;
  if (col < K) {
    float t = part[0][c];
#pragma unroll
    for (int w = 1; w < kColWarps; ++w) t = fmaxf(t, part[w][c]);
    atomicMax(out_bits + col, __float_as_uint(t));
  }
}

// s_j = fp32( pow(max(a_j,1e-8), alpha) / pow(max(w_j,1e-8), 1-alpha) ) in fp64; inv_s = 1/s in fp32.
__global__ void smooth_factors_kernel(const float* __restrict__ act_amax, float* __restrict__ s_inout,
                                      float* __restrict__ inv_s, int64_t K, float alpha) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const float a = fmaxf(act_amax[j], 1e-8f);
  const float w = fmaxf(s_inout[j], 1e-8f);
  const double num = pow(static_cast<double>(a), static_cast<double>(alpha));
  const double den = pow(static_cast<double>(w), 1.0 - static_cast<double>(alpha));
  const float sj = __double2float_rn(num / den);
  s_inout[j] = sj;
  inv_s[j] = __fdiv_rn(1.0f, sj);
}

__global__ void zero_words_kernel(uint32_t* __restrict__ words, int64_t n) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    words[i] = 0u;
}

}  // namespace

cudaError_t launch_zero_words(uint32_t* words, int64_t n, cudaStream_t stream) {
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>(std::max<int64_t>(1, (n + threads - 1) / threads), 1024);
  return launch_kernel(zero_words_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream, false,
                       words, n);
}

cudaError_t launch_col_absmax(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, float* amax,
                              bool accumulate, cudaStream_t stream) {
  if (!accumulate) {
    cudaError_t e = launch_zero_words(reinterpret_cast<uint32_t*>(amax), K, stream);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t col_blocks = (K + kColsPerCta - 1) / kColsPerCta;
  // one wave of ~4 CTAs per SM, at least 64 rows per CTA (few atomics per column)
  const int64_t target = static_cast<int64_t>(sms) * 4;
  int64_t row_blocks = std::max<int64_t>(1, target / col_blocks);
  int64_t rows_per_cta = (rows + row_blocks - 1) / row_blocks;
  rows_per_cta = std::max<int64_t>(64, ((rows_per_cta + kColWarps - 1) / kColWarps) * kColWarps);
  row_blocks = (rows + rows_per_cta - 1) / rows_per_cta;
  if (row_blocks > 65535) {
    row_blocks = 65535;
    rows_per_cta = (rows + row_blocks - 1) / row_blocks;
  }
  dim3 grid(static_cast<unsigned>(col_blocks), static_cast<unsigned>(row_blocks));
  return launch_kernel(col_absmax_kernel, grid, dim3(kColWarps * 32), 0, stream, false, src, rows, K, ld,
                       rows_per_cta, reinterpret_cast<unsigned int*>(amax));
}

cudaError_t launch_smooth_factors(const float* act_amax, float* s_inout, float* inv_s, int64_t K, float alpha,
                                  cudaStream_t stream) {
  const int threads = 256;
  const int64_t blocks = (K + threads - 1) / threads;
  return launch_kernel(smooth_factors_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream, false,
                       act_amax, s_inout, inv_s, K, alpha);
}

}  // namespace sq
