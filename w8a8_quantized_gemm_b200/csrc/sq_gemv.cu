// INT8 x INT8 -> INT32 products for a handful of tokens (M <= 4) on the CUDA cores, with
// the same dequantization epilogue as the tensor-core GEMM.
//
// "量化基础与INT8" INT8推理流程 (INT8 x INT8 -> INT32 accumulate, dequantized 16-bit output)
// and 量化流程示例 (Y = Y_int32 * X_scale * W_scale); "SmoothQuant量化实战" §3.4 (+ bias).
//
// With M <= 4 the product is a stream over the weight (N*K bytes) with M*N*K/4 dp4a
// operations: an HBM-bound pass, not a contraction worth the tensor cores' set-up (TMEM
// allocation, descriptor prefetch, K-split partials). Each CTA stages the M activation rows
// in shared memory once; each warp owns whole output channels: its lanes read 512 contiguous
// bytes of the channel's weight row per step (16-byte loads, up to eight in flight), multiply
// them with dp4a against the staged activations, and reduce the M int32 sums with shuffles.
// The epilogue is exactly the GEMM's: y = bf16_rne((float(acc) * d_m) * e_n + bias_n), the
// accumulator first corrected by acc - z_m * rowsum_n for asymmetric activations.
#include "sq_internal.h"
#include "sq_ptx.cuh"

#include <cuda_bf16.h>

#include <algorithm>

namespace sq {
namespace {

constexpr int kGemvThreads = 256;

// 16-byte weight loads in flight per lane: a whole 4096-byte row for one token; four for
// more tokens (measured: eight there cost registers and time)
template <int MT>
constexpr int gemv_unroll() {
  return MT == 1 ? 8 : 4;
}

template <int MT>
__global__ void __launch_bounds__(kGemvThreads)
gemv_i8_kernel(const int8_t* __restrict__ Xq, const int8_t* __restrict__ Wq, const float* __restrict__ x_scale,
               int x_per_token, const int32_t* __restrict__ x_zero, const float* __restrict__ w_scale,
               int w_per_channel, const int32_t* __restrict__ w_rowsum, const uint16_t* __restrict__ bias,
               uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out, int M, int64_t N, int64_t K) {
  constexpr int kGemvUnroll = gemv_unroll<MT>();
  extern __shared__ int4 xs[];  // [MT][K/16], rows past M zero
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kGemvThreads / 32);
  const int64_t n_first = static_cast<int64_t>(blockIdx.x) * (kGemvThreads / 32) + (threadIdx.x >> 5);
  // the weight does not depend on the previous kernel in a decode step: each warp starts
  // bringing its first channel row into L2 before waiting for that kernel (a prefetch is a
  // hint, safe even when the previous kernel wrote the weight)
  if (lane == 0 && n_first < N) bulk_prefetch_l2(Wq + n_first * K, static_cast<uint32_t>(K));
  griddep_wait();
  griddep_launch_dependents();
  const int64_t vecs = K / 16;
  for (int64_t i = threadIdx.x; i < MT * vecs; i += kGemvThreads) {
    const int m = static_cast<int>(i / vecs);
    xs[i] = m < M ? __ldg(reinterpret_cast<const int4*>(Xq + m * K) + (i - m * vecs)) : make_int4(0, 0, 0, 0);
  }
  __syncthreads();
  for (int64_t n = n_first; n < N; n += warps) {
    const int4* wrow = reinterpret_cast<const int4*>(Wq + n * K);
    int acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
    for (int64_t v0 = lane; v0 < vecs; v0 += 32 * kGemvUnroll) {
      int4 w[kGemvUnroll];
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        const int64_t v = v0 + u * 32;
        w[u] = v < vecs ? __ldcs(wrow + v) : make_int4(0, 0, 0, 0);  // streamed once
      }
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        const int64_t v = v0 + u * 32;
        if (v < vecs) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const int4 x = xs[m * vecs + v];
            acc[m] = __dp4a(w[u].x, x.x, acc[m]);
            acc[m] = __dp4a(w[u].y, x.y, acc[m]);
            acc[m] = __dp4a(w[u].z, x.z, acc[m]);
            acc[m] = __dp4a(w[u].w, x.w, acc[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
    }
    // lane m finishes token m of channel n
    if (lane < M && SQ_GUARD(n < N)) {
      int a = acc[0];
#pragma unroll
      for (int m = 1; m < MT; ++m)
        if (lane == m) a = acc[m];
      if (acc_out != nullptr) acc_out[static_cast<int64_t>(lane) * N + n] = a;
      float af;
      if (x_zero != nullptr)
        af = __ll2float_rn(static_cast<long long>(a) -
                           static_cast<long long>(__ldg(x_zero + lane)) * static_cast<long long>(__ldg(w_rowsum + n)));
      else
        af = static_cast<float>(a);
      const float d = __ldg(x_scale + (x_per_token ? lane : 0));
      const float e = __ldg(w_scale + (w_per_channel ? n : 0));
      float y = __fmul_rn(__fmul_rn(af, d), e);
      if (bias != nullptr) y = __fadd_rn(y, __uint_as_float(static_cast<uint32_t>(__ldg(bias + n)) << 16));
      Y[static_cast<int64_t>(lane) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
  }
}

template <int MT>
cudaError_t launch_t(const GemmArgs& a, cudaStream_t stream) {
  auto kernel = gemv_i8_kernel<MT>;
  const size_t smem = static_cast<size_t>(MT) * static_cast<size_t>(a.K);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kGemvThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t warps_needed = a.N;
  const int64_t blocks =
      std::max<int64_t>(1, std::min<int64_t>((warps_needed + kGemvThreads / 32 - 1) / (kGemvThreads / 32),
                                             static_cast<int64_t>(sms) * per_sm));
  return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kGemvThreads), smem, stream, true, a.Xq, a.Wq,
                       a.x_scale, a.x_per_token ? 1 : 0, a.x_zero, a.w_scale, a.w_per_channel ? 1 : 0, a.w_rowsum,
                       a.bias, a.Y, a.acc_out, static_cast<int>(a.M), a.N, a.K);
}

}  // namespace

bool gemv_applies(int64_t M, int64_t K, bool outliers) { return !outliers && M <= 4 && K <= 16384; }

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t stream) {
  if (a.M <= 1) return launch_t<1>(a, stream);
  if (a.M <= 2) return launch_t<2>(a, stream);
  return launch_t<4>(a, stream);
}

}  // namespace sq
