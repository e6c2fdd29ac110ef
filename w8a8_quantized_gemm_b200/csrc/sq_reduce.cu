// Column-wise absolute maximum (calibration statistic and LLM.int8 column detection)
// and the SmoothQuant smoothing factors.
//
// "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §3.2 (per-channel amax over the
// token dimensions, running maximum across batches) and §2.1/§3.3 (smoothing factor);
// "LLM.int8()技术解析" §2.1 step 1 (column-wise absolute maximum of the input).
//
// HBM-bound: each element of the source is read once with 16-byte loads. A cluster of up to
// sixteen CTAs covers a block of W columns (64, 128 or 256) and splits the rows between its
// CTAs; a warp reads 512 contiguous bytes per load instruction (one row of 256 columns, or
// 2 / 4 rows of 128 / 64 columns) with four loads in flight per thread. Lanes that share
// columns meet through shuffles and the warps of a CTA in shared memory; each CTA then
// stores its column maxima into its own slot of the cluster's first CTA (distributed shared
// memory), which after one cluster barrier takes the maximum over the slots and writes each
// column once: no atomics, no reset of the output, no scratch.
// The same pass can finish the SmoothQuant smoothing factors of its columns (the W side).
#include "sq_internal.h"
#include "sq_ptx.cuh"

#include <algorithm>
#include <atomic>

namespace sq {
namespace {

constexpr int kColWarps = 8;   // warps per CTA
constexpr int kRowUnroll = 4;  // independent 16-byte loads in flight per thread
constexpr int kMaxCluster = 16;  // CTAs per cluster (above 8: the non-portable cluster sizes)

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void absmax8(float (&m)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[2 * i] = fmaxf(m[2 * i], fabsf(bf16lo(w[i])));
    m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16hi(w[i])));
  }
}

// s_j = fp32( pow(max(a_j,1e-8), alpha) / pow(max(w_j,1e-8), 1-alpha) ) in fp64; inv_s = 1/s in fp32.
__device__ __forceinline__ void smooth_factor(float a_amax, float w_amax, float alpha, float* s, float* inv_s) {
  const float a = fmaxf(a_amax, 1e-8f);
  const float w = fmaxf(w_amax, 1e-8f);
  const double num = pow(static_cast<double>(a), static_cast<double>(alpha));
  const double den = pow(static_cast<double>(w), 1.0 - static_cast<double>(alpha));
  const float sj = __double2float_rn(num / den);
  *s = sj;
  *inv_s = __fdiv_rn(1.0f, sj);
}

// Grid: (column blocks x cluster size) CTAs, clusters along x (the CTAs of a cluster share a
// column block and split its rows). Output: out[j] = max_r |src[r, j]| (max with the old
// out[j] when `accumulate`), or, when `act_amax` is given, the smoothing factors of the
// columns: out = s, inv_s = 1/s with w_j the column maximum.
template <int W>
__global__ void __launch_bounds__(kColWarps * 32)
col_absmax_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int64_t rows_per_cta,
                  float* __restrict__ out, int accumulate, const float* __restrict__ act_amax,
                  float* __restrict__ inv_s, float alpha) {
  constexpr int kLanesPerRow = W / 8;           // each lane holds 8 columns
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;  // rows one warp load instruction covers
  __shared__ float part[kColWarps][W];
  __shared__ float slot[kMaxCluster][W];  // first CTA only: each CTA's column maxima
  cluster_arrive_relaxed();  // paired with the wait before the first remote store
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t nrank = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int64_t cblock = static_cast<int64_t>(blockIdx.x) / nrank;
  const int64_t col0 = cblock * W + (lane % kLanesPerRow) * 8;
  const bool col_ok = col0 < K;  // K % 16 == 0, so a lane's 8 columns are all in or all out
  const int64_t r_begin = static_cast<int64_t>(rank) * rows_per_cta;
  const int64_t r_end = min(rows, r_begin + rows_per_cta);
  constexpr int kStep = kColWarps * kRowsPerWarp;  // rows per load instruction of the CTA

  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  if (col_ok) {
    const uint16_t* base = src + col0;
    int64_t r = r_begin + warp * kRowsPerWarp + lane / kLanesPerRow;
    for (; r + (kRowUnroll - 1) * kStep < r_end; r += kRowUnroll * kStep) {
      uint4 v[kRowUnroll];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + (r + u * kStep) * ld));
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) absmax8(m, v[u]);
    }
    for (; r < r_end; r += kStep) absmax8(m, __ldg(reinterpret_cast<const uint4*>(base + r * ld)));
  }
  // lanes with the same columns (lane % kLanesPerRow) meet through shuffles
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], off));
  }
  if (lane < kLanesPerRow) {
#pragma unroll
    for (int i = 0; i < 8; ++i) part[warp][lane * 8 + i] = m[i];
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster has started: its shared memory may be written
  if (threadIdx.x < W) {
    float t = part[0][threadIdx.x];
#pragma unroll
    for (int w = 1; w < kColWarps; ++w) t = fmaxf(t, part[w][threadIdx.x]);
    st_cluster_f32(mapa_shared(&slot[rank][threadIdx.x], 0), t);
  }
  cluster_sync();  // every CTA's column maxima have reached the first CTA
  if (rank == 0 && threadIdx.x < W) {
    const int64_t col = cblock * W + threadIdx.x;
    float t = slot[0][threadIdx.x];
    for (uint32_t q = 1; q < nrank; ++q) t = fmaxf(t, slot[q][threadIdx.x]);
    if (col < K) {
      if (act_amax != nullptr) {
        smooth_factor(act_amax[col], t, alpha, out + col, inv_s + col);
      } else {
        if (accumulate) t = fmaxf(out[col], t);
        out[col] = t;
      }
    }
  }
}

__global__ void zero_words_kernel(uint32_t* __restrict__ words, int64_t n) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    words[i] = 0u;
}

template <int W>
cudaError_t launch_cols(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, float* out, bool accumulate,
                        const float* act_amax, float* inv_s, float alpha, int cluster, cudaStream_t stream) {
  const int64_t col_blocks = (K + W - 1) / W;
  const int64_t rows_per_cta = (rows + cluster - 1) / cluster;
  if (cluster > 8) {
    static std::atomic<uint64_t> attr_done{0};  // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
      cudaError_t e = cudaFuncSetAttribute(col_absmax_kernel<W>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      attr_done.fetch_or(bit);
    }
  }
  return launch_kernel_clustered(col_absmax_kernel<W>, dim3(static_cast<unsigned>(col_blocks * cluster)),
                                 dim3(kColWarps * 32), 0, stream, false, static_cast<unsigned>(cluster), src, rows, K,
                                 ld, rows_per_cta, out, accumulate ? 1 : 0, act_amax, inv_s, alpha);
}

// Column blocks of 256, 128 or 64 columns: the widest that still gives three CTAs per SM
// with clusters of sixteen (fewer CTAs per cluster when there are few rows: at least 64 rows
// per CTA). With fewer CTAs the SMs that hold one more CTA than the others set the time.
cudaError_t launch_col_reduce(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, float* out, bool accumulate,
                              const float* act_amax, float* inv_s, float alpha, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cluster = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kMaxCluster, rows / 64)));
  const int64_t want = 3 * static_cast<int64_t>(sms);
  if (((K + 255) / 256) * cluster >= want)
    return launch_cols<256>(src, rows, K, ld, out, accumulate, act_amax, inv_s, alpha, cluster, stream);
  if (((K + 127) / 128) * cluster >= want)
    return launch_cols<128>(src, rows, K, ld, out, accumulate, act_amax, inv_s, alpha, cluster, stream);
  return launch_cols<64>(src, rows, K, ld, out, accumulate, act_amax, inv_s, alpha, cluster, stream);
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
  return launch_col_reduce(src, rows, K, ld, amax, accumulate, nullptr, nullptr, 0.0f, stream);
}

cudaError_t launch_smooth_scale(const float* act_amax, const uint16_t* W, int64_t N, int64_t K, int64_t ldw,
                                float alpha, float* s, float* inv_s, cudaStream_t stream) {
  return launch_col_reduce(W, N, K, ldw, s, false, act_amax, inv_s, alpha, stream);
}

}  // namespace sq
