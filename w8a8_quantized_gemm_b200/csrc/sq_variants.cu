// Kernels of the variants around the W8A8 layer:
//   - normalisation of the smoothing factors,
//     "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §3.3 (s / s.max() * 127, clamp 1e-5);
//   - LayerNorm / RMSNorm fused with smoothing and per-token quantization, the same page
//     §4.2 and §4.5 second detail (the smoothing folds into the LayerNorm output);
//   - mean + k*std outlier threshold over the activations, "LLM.int8()技术解析" §3.1
//     (threshold = mu + 6 sigma) and "从自动驾驶芯片到大语言模型INT8量化训练实战解析" §2.1;
//   - nearest-rank percentile of |X| for static calibration, the page on choosing
//     quantization precision ("大语言模型轻量化与量化精度") §3.2 (percentile 99.99);
//   - row sums of the int8 weight (zero-point correction of asymmetric activations,
//     "量化基础与INT8" 非对称量化).
// All of them are HBM-bound passes over bf16 / int8 matrices with 16-byte loads; the
// reductions that feed a floating-point decision are summed in fp64 in a fixed order, so
// every result is deterministic run to run.
#include "sq_internal.h"
#include "sq_ptx.cuh"
#include "sq_rows.cuh"

#include <algorithm>
#include <atomic>

namespace sq {
namespace {

using namespace rows;

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// ------------------------------------------------------------------ smoothing factors
// One CTA: smax = max_j s_j, then s_j <- max((s_j / smax) * 127, 1e-5), inv_s_j = 1/s_j.
__global__ void __launch_bounds__(1024) normalize_scale_kernel(float* __restrict__ s, float* __restrict__ inv_s,
                                                               int64_t K) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float red[32];
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) m = fmaxf(m, s[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float smax = red[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) smax = fmaxf(smax, red[w]);
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
    const float t = fmaxf(__fmul_rn(__fdiv_rn(s[j], smax), 127.0f), 1e-5f);
    s[j] = t;
    inv_s[j] = __fdiv_rn(1.0f, t);
  }
}

// ------------------------------------------------------------------ weight row sums
// One warp per row: rowsum[n] = sum_k Wq[n,k] (16-byte loads, dp4a against ones).
__global__ void __launch_bounds__(256) row_sums_kernel(const int8_t* __restrict__ Wq, int64_t N, int64_t K,
                                                       int32_t* __restrict__ rowsum) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += warps) {
    const int4* row = reinterpret_cast<const int4*>(Wq + n * K);
    int acc = 0;
    for (int64_t v = lane; v < K / 16; v += 32) {
      const int4 w = __ldg(row + v);
      acc = __dp4a(w.x, 0x01010101, acc);
      acc = __dp4a(w.y, 0x01010101, acc);
      acc = __dp4a(w.z, 0x01010101, acc);
      acc = __dp4a(w.w, 0x01010101, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) rowsum[n] = acc;
  }
}

// ------------------------------------------------------------------ fused normalisation
// Row groups of TPR threads walk the rows with a grid stride (as the row quantization
// kernel does); a thread owns 16 consecutive columns per chunk and keeps its row values in
// registers between the statistics, the absmax and the quantization, and prefetches its
// next row. With one chunk per thread its slices of gamma, beta and inv_s stay in
// registers for all its rows; with two they are re-read per row (L1 hits) to keep the
// register count within the launch bound.
template <int TPR, int CHUNKS>
__global__ void __launch_bounds__(TPR > kCta ? TPR : kCta)
norm_quant_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int norm,
                  const uint16_t* __restrict__ gamma, const uint16_t* __restrict__ beta, float eps,
                  const float* __restrict__ vec, int8_t* __restrict__ q, float* __restrict__ scale,
                  float* __restrict__ mean_rstd) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  constexpr int kGroups = kThreads / TPR;
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float redf[kThreads / 32];
  __shared__ double2 redd[kThreads / 32];
  const int g = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int64_t step = static_cast<int64_t>(TPR) * 16;
  const int64_t row_stride = static_cast<int64_t>(gridDim.x) * kGroups;
  const bool layer = (norm == 0);
  const bool has_beta = beta != nullptr;
  const bool has_vec = vec != nullptr;

  constexpr bool kResident = CHUNKS == 1;
  // gamma, beta (0 when absent) and inv_s (1 when absent) of columns k..k+15; columns past
  // K get gamma = 0, so their y is 0 and they do not enter the absmax
  auto load_vectors = [&](int64_t k, float (&g16)[16], float (&b16)[16], float (&v16)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      g16[i] = 0.0f;
      b16[i] = 0.0f;
      v16[i] = 1.0f;
    }
    if (k < K) {
      uint4 r[2];
      raw16(gamma + k, r);
      widen16(r, g16);
      if (has_beta) {
        raw16(beta + k, r);
        widen16(r, b16);
      }
      if (has_vec) {
        const float4* p4 = reinterpret_cast<const float4*>(vec + k);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 f = __ldg(p4 + i);
          v16[4 * i] = f.x;
          v16[4 * i + 1] = f.y;
          v16[4 * i + 2] = f.z;
          v16[4 * i + 3] = f.w;
        }
      }
    }
  };
  float gs[1][16], bs[1][16], vs[1][16];  // this thread's chunk (the only one when resident)
  if constexpr (kResident) load_vectors(t * 16, gs[0], bs[0], vs[0]);

  uint4 raw[CHUNKS][2];
  int64_t row = static_cast<int64_t>(blockIdx.x) * kGroups + g;
  if (row < rows) {
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int64_t k = c * step + t * 16;
      if (k < K) raw16(src + row * ld + k, raw[c]);
    }
  }

  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kGroups; base < rows; base += row_stride, row += row_stride) {
    const bool row_ok = row < rows;
    float x[CHUNKS][16];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int64_t k = c * step + t * 16;
      if (row_ok && k < K) {
        widen16(raw[c], x[c]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[c][i] = 0.0f;
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
    // row statistics in one pass: sum and sum of squares in fp64 (the square of a bf16
    // value is exact in fp64), four independent chains per thread, one group reduction;
    // var = E[x^2] - mean^2 (the fp64 headroom keeps it within rounding of the two-pass form
    // for any input a bf16 row can hold relative to fp32 resolution). Absent columns hold 0.
    double s1a = 0.0, s1b = 0.0, s2a = 0.0, s2b = 0.0;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c)
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const double xa = static_cast<double>(x[c][i]);
        const double xb = static_cast<double>(x[c][i + 1]);
        s1a = __dadd_rn(s1a, xa);
        s1b = __dadd_rn(s1b, xb);
        s2a = __fma_rn(xa, xa, s2a);
        s2b = __fma_rn(xb, xb, s2b);
      }
    double s1 = __dadd_rn(s1a, s1b), s2 = __dadd_rn(s2a, s2b);
    group_sum2<TPR>(s1, s2, redd);
    const double kd = static_cast<double>(K);
    float mean_f = 0.0f;
    double m2 = __ddiv_rn(s2, kd);
    if (layer) {
      const double mean = __ddiv_rn(s1, kd);
      mean_f = __double2float_rn(mean);
      m2 = fmax(__dsub_rn(m2, __dmul_rn(mean, mean)), 0.0);
    }
    const float rstd_f = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(m2, static_cast<double>(eps)))));
    // y = ((x - mean) * rstd) * gamma + beta, x' = y * inv_s, absmax
    float a = 0.0f;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      if constexpr (!kResident) load_vectors(c * step + t * 16, gs[0], bs[0], vs[0]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float y = layer ? __fmul_rn(__fsub_rn(x[c][i], mean_f), rstd_f) : __fmul_rn(x[c][i], rstd_f);
        y = __fmul_rn(y, gs[0][i]);
        if (has_beta) y = __fadd_rn(y, bs[0][i]);
        if (has_vec) y = __fmul_rn(y, vs[0][i]);
        x[c][i] = y;
        a = fmaxf(a, fabsf(y));
      }
    }
    a = group_max<TPR>(a, redf);
    const float r = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    if (row_ok) {
      if (t == 0) {
        scale[row] = __fdiv_rn(a, 127.0f);
        if (mean_rstd != nullptr) {
          mean_rstd[2 * row] = mean_f;
          mean_rstd[2 * row + 1] = rstd_f;
        }
      }
      int8_t* qrow = q + row * K;
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int64_t k = c * step + t * 16;
        if (k < K && SQ_GUARD(k + 16 <= K)) store_q16_own_max(qrow + k, x[c], r);
      }
    }
  }
}

constexpr int kNormMaxSlots = 6;
constexpr int kNormSmem = 192 * 1024;  // row ring per CTA

// Row groups for long rows (see launch_norm_quant): G groups of GT threads per CTA, one
// persistent CTA per SM. Each group streams its rows (row0 + j * stride) through a ring of
// `slots` shared-memory row buffers filled by cp.async.bulk (one thread issues a whole row,
// completion on the slot's mbarrier), so the bytes in flight do not depend on the registers
// the arithmetic needs. A thread owns the 8-column chunks t, t + GT, ... of every row. Each
// pass of the group's loop works on two rows:
//   1. the statistics of row j from the warps' partial sums (every warp finishes them itself:
//      no broadcast, no extra barrier), then row j read from its slot into the normalised,
//      smoothed values y (kept in registers) and the warp's partial absmax;
//   2. row j+1 read from its slot into its fp64 partial sums;
//   3. one group barrier, after which row j's slot goes back to the copy engine, its absmax is
//      known and its codes are stored.
// One barrier per row, and the statistics of one row overlap the arithmetic of the previous
// one; reading each row twice from shared memory keeps no raw row in registers across the
// barrier. The per-row finish uses a multiply by 1/K and the fp64 reciprocal square root (each
// within a few fp64 ulps of the divisions and square root written out, far below the fp32
// rounding of mean_f and rstd_f). Where both operands of an operation are pairs, the fp32 steps
// use sm_100's packed f32x2 instructions (two IEEE round-to-nearest operations each); the
// multiply that the beta add follows stays scalar, so that no packed multiply feeds an add (such
// a pair was observed to execute as one fused multiply-add). The codes use scalar multiplies and
// adds, each rounded.
template <int GT, int CH, int G, bool LAYER, bool BETA, bool VEC>
__global__ void __launch_bounds__(GT * G, 1)
norm_quant_pipe_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                       const uint16_t* __restrict__ gamma, const uint16_t* __restrict__ beta, float eps,
                       const float* __restrict__ vec, int8_t* __restrict__ q, float* __restrict__ scale,
                       float* __restrict__ mean_rstd, int slots, unsigned int* status, uint64_t wait_limit_ns) {
  constexpr int kWarps = GT / 32;
  extern __shared__ __align__(128) uint8_t ring_all[];
  __shared__ uint64_t full_all[G][kNormMaxSlots];
  __shared__ double2 red2[G][2][kWarps];  // partial (sum x, sum x^2) per warp, by row parity
  __shared__ float redm[G][2][kWarps];    // partial absmax per warp, by row parity
  const int g = threadIdx.x / GT;
  const int t = threadIdx.x % GT;
  const int lane = threadIdx.x & 31;
  const int wg = t >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  uint8_t* ring = ring_all + static_cast<size_t>(g) * slots * row_bytes;
  uint64_t* full = full_all[g];
  if (t == 0) {
    for (int i = 0; i < slots; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  const int nch = static_cast<int>(K / 8);
  const int64_t stride = static_cast<int64_t>(G) * gridDim.x;
  const int64_t row0 = blockIdx.x + static_cast<int64_t>(g) * gridDim.x;
  const int64_t nrows = row0 < rows ? (rows - 1 - row0) / stride + 1 : 0;  // this group's rows
  const double inv_k = 1.0 / static_cast<double>(K);
  int64_t issued = 0;
  if (t == 0) {
    for (int i = 0; i < slots && i < nrows; ++i) {
      mbar_arrive_expect_tx(full + i, row_bytes);
      bulk_load(ring + static_cast<size_t>(i) * row_bytes, src + (row0 + i * stride) * ld, row_bytes, full + i);
      ++issued;
    }
  }

  int64_t pending = 0;  // the row whose slot was waited for last
  bool failed = false;  // this thread's wait for a slot gave up
  auto slot_row = [&](int64_t i) {
    return reinterpret_cast<const uint4*>(ring + static_cast<size_t>(i % slots) * row_bytes);
  };
  // Row i of the group: wait for its slot, read this thread's chunks, leave the warp's partial
  // sums in red2[g][i & 1]. A thread whose wait gives up still reaches the next group barrier,
  // which ORs `failed` over the group, so that the whole group stops there together.
  auto load_stats = [&](int64_t i) {
    pending = i;
    if (!mbar_wait_bounded(full + static_cast<int>(i % slots), static_cast<uint32_t>((i / slots) & 1),
                           wait_limit_ns)) {
      atomicOr(status, kErrProducerWait);
      failed = true;
    }
    const uint4* srow = slot_row(i);
    double s1a = 0.0, s1b = 0.0, s2a = 0.0, s2b = 0.0;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int idx = t + c * GT;
      const uint4 rc = idx < nch ? srow[idx] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {rc.x, rc.y, rc.z, rc.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double xa = static_cast<double>(__uint_as_float(w[k] << 16));
        const double xb = static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u));
        if constexpr (LAYER) {
          s1a = __dadd_rn(s1a, xa);
          s1b = __dadd_rn(s1b, xb);
        }
        s2a = __fma_rn(xa, xa, s2a);
        s2b = __fma_rn(xb, xb, s2b);
      }
    }
    double s1 = __dadd_rn(s1a, s1b), s2 = __dadd_rn(s2a, s2b);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      if constexpr (LAYER) s1 = __dadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, o));
      s2 = __dadd_rn(s2, __shfl_xor_sync(0xffffffffu, s2, o));
    }
    if (lane == 0) red2[g][i & 1][wg] = make_double2(s1, s2);
  };
  // After the group barrier that follows the last read of row i, its slot takes row i + slots.
  auto refill = [&](int64_t i) {
    if (t == 0 && i + slots < nrows) {
      const int slot = static_cast<int>(i % slots);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(full + slot, row_bytes);
      bulk_load(ring + static_cast<size_t>(slot) * row_bytes, src + (row0 + (i + slots) * stride) * ld, row_bytes,
                full + slot);
      ++issued;
    }
  };

  bool aborted = false;
  if (nrows > 0) {
    load_stats(0);
    aborted = named_bar_sync_or(1 + g, GT, failed);
  }
  for (int64_t j = 0; j < nrows && !aborted; ++j) {
    const int p = static_cast<int>(j & 1);
    // 1. statistics of row j (the same fixed order of the warps' partials in every warp)
    double s1 = 0.0, s2 = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const double2 v = red2[g][p][w];
      if constexpr (LAYER) s1 = __dadd_rn(s1, v.x);
      s2 = __dadd_rn(s2, v.y);
    }
    float mean_f = 0.0f;
    double m2 = __dmul_rn(s2, inv_k);
    if constexpr (LAYER) {
      const double mean = __dmul_rn(s1, inv_k);
      mean_f = __double2float_rn(mean);
      m2 = fmax(__dsub_rn(m2, __dmul_rn(mean, mean)), 0.0);
    }
    const float rstd_f = __double2float_rn(rsqrt(__dadd_rn(m2, static_cast<double>(eps))));
    const uint64_t mean2 = f2_pack(mean_f, mean_f);
    const uint64_t rstd2 = f2_pack(rstd_f, rstd_f);
    // y = ((x - mean) * rstd) * gamma + beta, x' = y * inv_s; absmax
    const uint4* srow = slot_row(j);
    float y[CH][8];
    float a = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int idx = t + c * GT;
      if (idx < nch) {
        const uint4 rc = srow[idx];
        const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gamma) + idx);
        const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
        uint32_t bw[4] = {0u, 0u, 0u, 0u};
        if constexpr (BETA) {
          const uint4 b4 = __ldg(reinterpret_cast<const uint4*>(beta) + idx);
          bw[0] = b4.x; bw[1] = b4.y; bw[2] = b4.z; bw[3] = b4.w;
        }
        uint64_t vv[4] = {0u, 0u, 0u, 0u};
        if constexpr (VEC) {
          const ulonglong2 v0 = __ldg(reinterpret_cast<const ulonglong2*>(vec) + 2 * idx);
          const ulonglong2 v1 = __ldg(reinterpret_cast<const ulonglong2*>(vec) + 2 * idx + 1);
          vv[0] = v0.x; vv[1] = v0.y; vv[2] = v1.x; vv[3] = v1.y;
        }
        const uint32_t xw[4] = {rc.x, rc.y, rc.z, rc.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint64_t v2 = f2_pack(__uint_as_float(xw[k] << 16), __uint_as_float(xw[k] & 0xFFFF0000u));
          if constexpr (LAYER) v2 = f2_sub(v2, mean2);
          v2 = f2_mul(v2, rstd2);
          float y0, y1;
          if constexpr (BETA) {
            f2_unpack(v2, y0, y1);
            y0 = __fadd_rn(__fmul_rn(y0, __uint_as_float(gw[k] << 16)), __uint_as_float(bw[k] << 16));
            y1 = __fadd_rn(__fmul_rn(y1, __uint_as_float(gw[k] & 0xFFFF0000u)), __uint_as_float(bw[k] & 0xFFFF0000u));
            if constexpr (VEC) f2_unpack(f2_mul(f2_pack(y0, y1), vv[k]), y0, y1);
          } else {
            v2 = f2_mul(v2, f2_pack(__uint_as_float(gw[k] << 16), __uint_as_float(gw[k] & 0xFFFF0000u)));
            if constexpr (VEC) v2 = f2_mul(v2, vv[k]);
            f2_unpack(v2, y0, y1);
          }
          y[c][2 * k] = y0;
          y[c][2 * k + 1] = y1;
          a = fmaxf(a, fmaxf(fabsf(y0), fabsf(y1)));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) y[c][k] = 0.0f;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) redm[g][p][wg] = a;
    // 2. the next row
    if (j + 1 < nrows) load_stats(j + 1);
    // 3. one barrier: row j's partial maxima and row j+1's partial sums are in, row j's slot
    //    has been read for the last time by every thread
    aborted = named_bar_sync_or(1 + g, GT, failed);
    if (aborted) break;
    refill(j);
    a = redm[g][p][0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) a = fmaxf(a, redm[g][p][w]);
    const float r = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    const int64_t row = row0 + j * stride;
    if (t == 0) {
      scale[row] = __fdiv_rn(a, 127.0f);
      if (mean_rstd != nullptr) {
        mean_rstd[2 * row] = mean_f;
        mean_rstd[2 * row + 1] = rstd_f;
      }
    }
    // codes: a row scaled by its own maximum needs no clamp unless r overflowed
    int8_t* qrow = q + row * K;
    const bool clamp = !(r <= 3.402823466e38f);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int idx = t + c * GT;
      if (idx < nch && SQ_GUARD(idx * 8 + 8 <= K)) {
        int qv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float tq = __fmul_rn(y[c][k], r);
          if (clamp) tq = fminf(fmaxf(tq, -128.0f), 127.0f);
          qv[k] = __float_as_int(__fadd_rn(tq, 12582912.0f));
        }
        *reinterpret_cast<uint2*>(qrow + idx * 8) =
            make_uint2(pack4(qv[0], qv[1], qv[2], qv[3]), pack4(qv[4], qv[5], qv[6], qv[7]));
      }
    }
  }
  // copies issued for rows this group did not consume (after a timed-out wait) land before exit
  if (t == 0 && aborted) {
    for (int64_t k = pending; k < issued; ++k) {
      if (!mbar_wait_bounded(full + static_cast<int>(k % slots), static_cast<uint32_t>((k / slots) & 1),
                             wait_limit_ns))
        atomicOr(status, kErrTeardownWait);
    }
  }
}

template <int GT, int CH, int G, bool LAYER, bool BETA, bool VEC>
cudaError_t launch_norm_pipe_t(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, const uint16_t* gamma,
                               const uint16_t* beta, float eps, const float* vec, int8_t* q, float* scale,
                               float* mean_rstd, cudaStream_t stream) {
  auto kernel = norm_quant_pipe_kernel<GT, CH, G, LAYER, BETA, VEC>;
  const int64_t row_bytes = K * 2;
  const int slots = static_cast<int>(std::min<int64_t>(kNormMaxSlots, kNormSmem / (G * row_bytes)));
  // a group holds two rows at once (row j being normalised, row j+1 being summed)
  if (slots < 2 || K > static_cast<int64_t>(GT) * CH * 8) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(G) * slots * row_bytes;
  static std::atomic<uint64_t> attr_done{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kNormSmem);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  unsigned int* status = device_status_word();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  const int64_t blocks = std::min<int64_t>(sm_count(), (rows + G - 1) / G);
  return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(GT * G), smem, stream, false, src, rows, K,
                       ld, gamma, beta, eps, vec, q, scale, mean_rstd, slots, status, kDefaultWaitLimitNs);
}

// The norm kind and the presence of beta and of the smoothing vector are compile-time flags.
template <int GT, int CH, int G>
cudaError_t launch_norm_pipe(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, int norm,
                             const uint16_t* gamma, const uint16_t* beta, float eps, const float* vec, int8_t* q,
                             float* scale, float* mean_rstd, cudaStream_t stream) {
#define SQ_PIPE(L, B, V) \
  launch_norm_pipe_t<GT, CH, G, L, B, V>(src, rows, K, ld, gamma, beta, eps, vec, q, scale, mean_rstd, stream)
  const bool b = beta != nullptr, v = vec != nullptr;
  if (norm == 0) {
    if (b) return v ? SQ_PIPE(true, true, true) : SQ_PIPE(true, true, false);
    return v ? SQ_PIPE(true, false, true) : SQ_PIPE(true, false, false);
  }
  if (b) return v ? SQ_PIPE(false, true, true) : SQ_PIPE(false, true, false);
  return v ? SQ_PIPE(false, false, true) : SQ_PIPE(false, false, false);
#undef SQ_PIPE
}

template <int TPR, int CHUNKS>
cudaError_t launch_norm_t(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, int norm, const uint16_t* gamma,
                          const uint16_t* beta, float eps, const float* vec, int8_t* q, float* scale,
                          float* mean_rstd, cudaStream_t stream) {
  constexpr int kThreads = TPR > kCta ? TPR : kCta;
  constexpr int kGroups = kThreads / TPR;
  auto kernel = norm_quant_kernel<TPR, CHUNKS>;
  static int per_sm = 0;
  if (per_sm <= 0) {
    int v = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, kThreads, 0) != cudaSuccess || v < 1) v = 1;
    per_sm = v;
  }
  const int64_t groups = (rows + kGroups - 1) / kGroups;
  const int64_t blocks = std::min<int64_t>(groups, static_cast<int64_t>(sm_count()) * per_sm);
  return launch_kernel(kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, stream, false, src, rows, K,
                       ld, norm, gamma, beta, eps, vec, q, scale, mean_rstd);
}

// ------------------------------------------------------------------ mean / std threshold
constexpr int kStatThreads = 256;
constexpr int kStatUnroll = 4;

// part1[b], part2[b] = sum and sum of squares of the elements of CTA b's rows (fp64, four
// independent chains per thread, then a fixed-order CTA reduction). Each thread keeps
// kStatUnroll 16-byte loads in flight ahead of the conversions and sums.
__global__ void __launch_bounds__(kStatThreads)
sum_partials_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int64_t rows_per_cta,
                    double* __restrict__ part1, double* __restrict__ part2) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double2 red[kStatThreads / 32];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
  const int64_t r1 = min(rows, r0 + rows_per_cta);
  const int64_t vecs = K / 8;
  double s1a = 0.0, s1b = 0.0, s2a = 0.0, s2b = 0.0;
  for (int64_t r = r0; r < r1; ++r) {
    const uint4* p = reinterpret_cast<const uint4*>(src + r * ld);
    for (int64_t v0 = threadIdx.x; v0 < vecs; v0 += kStatThreads * kStatUnroll) {
      uint4 w[kStatUnroll];
#pragma unroll
      for (int j = 0; j < kStatUnroll; ++j) {
        const int64_t v = v0 + j * kStatThreads;
        w[j] = v < vecs ? __ldg(p + v) : make_uint4(0u, 0u, 0u, 0u);  // zeros add nothing
      }
#pragma unroll
      for (int j = 0; j < kStatUnroll; ++j) {
        const uint32_t u[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double lo = static_cast<double>(__uint_as_float(u[i] << 16));
          const double hi = static_cast<double>(__uint_as_float(u[i] & 0xFFFF0000u));
          s1a = __dadd_rn(s1a, lo);
          s1b = __dadd_rn(s1b, hi);
          s2a = __fma_rn(lo, lo, s2a);
          s2b = __fma_rn(hi, hi, s2b);
        }
      }
    }
  }
  double s1 = __dadd_rn(s1a, s1b), s2 = __dadd_rn(s2a, s2b);
  group_sum2<kStatThreads>(s1, s2, red);
  if (threadIdx.x == 0) {
    part1[blockIdx.x] = s1;
    part2[blockIdx.x] = s2;
  }
}

// One CTA: totals of the G partials in a fixed order, mean = S1/n, unbiased
// var = (S2 - S1*mean)/(n - 1), threshold = fp32(mean + k*sqrt(var)).
__global__ void __launch_bounds__(kStatThreads)
finish_threshold_kernel(const double* __restrict__ part1, const double* __restrict__ part2, int G, double n,
                        double k, float* __restrict__ threshold, double* __restrict__ mean_std) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double2 red[kStatThreads / 32];
  double s1 = 0.0, s2 = 0.0;
  for (int i = threadIdx.x; i < G; i += kStatThreads) {
    s1 = __dadd_rn(s1, part1[i]);
    s2 = __dadd_rn(s2, part2[i]);
  }
  group_sum2<kStatThreads>(s1, s2, red);
  if (threadIdx.x == 0) {
    const double mean = __ddiv_rn(s1, n);
    const double var = n > 1.0 ? fmax(__ddiv_rn(__dsub_rn(s2, __dmul_rn(s1, mean)), n - 1.0), 0.0) : 0.0;
    const double sd = __dsqrt_rn(var);
    *threshold = __double2float_rn(__dadd_rn(mean, __dmul_rn(k, sd)));
    if (mean_std != nullptr) {
      mean_std[0] = mean;
      mean_std[1] = sd;
    }
  }
}

// ------------------------------------------------------------------ percentile
constexpr int kBins = 1 << 15;  // bf16 magnitudes (sign dropped)
constexpr int kHistThreads = 1024;

// Per-CTA histogram of |x| bit patterns in shared memory, added into the global one. Each
// thread keeps kHistUnroll 16-byte loads in flight before their shared-memory atomics (one
// load per thread left the pass short of bytes in flight).
constexpr int kHistUnroll = 4;

__global__ void __launch_bounds__(kHistThreads)
abs_hist_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                unsigned long long* __restrict__ hist) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t sh[];
  for (int b = threadIdx.x; b < kBins; b += kHistThreads) sh[b] = 0u;
  __syncthreads();
  const int64_t vecs_per_row = K / 8;
  const int64_t total = rows * vecs_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kHistThreads;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kHistThreads + threadIdx.x; v0 < total;
       v0 += stride * kHistUnroll) {
    uint4 w[kHistUnroll];
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      const int64_t v = v0 + u * stride;
      if (v < total) {
        const int64_t r = v / vecs_per_row;
        const int64_t c = v - r * vecs_per_row;
        w[u] = __ldg(reinterpret_cast<const uint4*>(src + r * ld) + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      if (v0 + u * stride < total) {
        const uint32_t q[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          atomicAdd(&sh[q[i] & 0x7FFFu], 1u);
          atomicAdd(&sh[(q[i] >> 16) & 0x7FFFu], 1u);
        }
      }
    }
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += kHistThreads)
    if (sh[b] != 0u) atomicAdd(hist + b, static_cast<unsigned long long>(sh[b]));
}

// One CTA of 32 warps; warp w owns the 1024 consecutive bins [1024 w, 1024 w + 1024). The
// warps' totals (coalesced reads) locate the warp whose bins hold the element of 1-based rank
// `rank`; that warp walks its bins 32 at a time with an inclusive warp scan and the first bin
// whose cumulative count reaches the rank gives the value (the bin is the value's bit pattern).
__global__ void __launch_bounds__(kHistThreads)
select_rank_kernel(const unsigned long long* __restrict__ hist, unsigned long long rank, float* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int kWarps = kHistThreads / 32;
  constexpr int kPerWarp = kBins / kWarps;
  __shared__ unsigned long long wsum[kWarps];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const unsigned long long* h = hist + static_cast<int64_t>(warp) * kPerWarp;
  unsigned long long s = 0;
  for (int i = lane; i < kPerWarp; i += 32) s += h[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) wsum[warp] = s;
  __syncthreads();
  unsigned long long run = 0;  // count in the bins before this warp's
  for (int w = 0; w < warp; ++w) run += wsum[w];
  if (!(run < rank && run + wsum[warp] >= rank)) return;  // warp-uniform
  for (int i0 = 0; i0 < kPerWarp; i0 += 32) {
    unsigned long long inc = h[i0 + lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, run + inc >= rank);
    if (hit != 0u) {
      const int first = __ffs(hit) - 1;
      const int bin = warp * kPerWarp + i0 + first;
      if (lane == first && SQ_GUARD(bin < kBins)) *out = __uint_as_float(static_cast<uint32_t>(bin) << 16);
      break;
    }
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
}

}  // namespace

cudaError_t launch_normalize_scale(float* s, float* inv_s, int64_t K, cudaStream_t stream) {
  return launch_kernel(normalize_scale_kernel, dim3(1), dim3(1024), 0, stream, false, s, inv_s, K);
}

cudaError_t launch_row_sums(const int8_t* Wq, int64_t N, int64_t K, int32_t* rowsum, cudaStream_t stream) {
  const int64_t blocks = std::min<int64_t>((N + 7) / 8, static_cast<int64_t>(sm_count()) * 8);
  return launch_kernel(row_sums_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, false, Wq, N, K,
                       rowsum);
}

cudaError_t launch_norm_quant(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, int norm,
                              const uint16_t* gamma, const uint16_t* beta, float eps, const float* vec, int8_t* q,
                              float* scale, float* mean_rstd, cudaStream_t stream) {
#define SQ_NORM_ARGS src, rows, K, ld, norm, gamma, beta, eps, vec, q, scale, mean_rstd, stream
  // Measured on X [M, K] with M = 2048..8192 (graph-timed, one B200): the pipelined row groups
  // win for K > 4096 (LayerNorm / RMSNorm 87 / 78 us at 8192 x 8192 against 99 / 82 us for the
  // best earlier forms, 86 / 80 us against 106 / 82 us at 4096 x 16384); at K <= 4096 they are
  // no faster than the register rows (13.6 vs 13.7 us at 2048 x 4096).
  if (K <= 512) return launch_norm_t<32, 1>(SQ_NORM_ARGS);
  if (K <= 1024) return launch_norm_t<64, 1>(SQ_NORM_ARGS);
  if (K <= 2048) return launch_norm_t<128, 1>(SQ_NORM_ARGS);
  if (K <= 4096) return launch_norm_t<256, 1>(SQ_NORM_ARGS);
  if (K <= 8192) return launch_norm_pipe<128, 8, 4>(SQ_NORM_ARGS);
  return launch_norm_pipe<256, 8, 2>(SQ_NORM_ARGS);
#undef SQ_NORM_ARGS
}

int64_t mean_std_ctas(int64_t rows) { return std::min<int64_t>(rows, 1024); }

size_t mean_std_workspace_bytes(int64_t rows) {
  // the two partial arrays of G doubles
  return sizeof(double) * 2 * static_cast<size_t>(mean_std_ctas(rows));
}

cudaError_t launch_mean_std_threshold(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, double k,
                                      float* threshold, double* mean_std, void* ws, cudaStream_t stream) {
  const int64_t G = mean_std_ctas(rows);
  const int64_t rpc = (rows + G - 1) / G;
  const int64_t ctas = (rows + rpc - 1) / rpc;
  double* part1 = static_cast<double*>(ws);
  double* part2 = part1 + G;
  const double n = static_cast<double>(rows) * static_cast<double>(K);
  cudaError_t e = launch_kernel(sum_partials_kernel, dim3(static_cast<unsigned>(ctas)), dim3(kStatThreads), 0,
                                stream, false, src, rows, K, ld, rpc, part1, part2);
  if (e == cudaSuccess)
    e = launch_kernel(finish_threshold_kernel, dim3(1), dim3(kStatThreads), 0, stream, false,
                      static_cast<const double*>(part1), static_cast<const double*>(part2), static_cast<int>(ctas), n,
                      k, threshold, mean_std);
  return e;
}

size_t abs_percentile_workspace_bytes() { return sizeof(unsigned long long) * kBins; }

cudaError_t launch_abs_percentile(const uint16_t* src, int64_t rows, int64_t K, int64_t ld, uint64_t rank,
                                  float* out, void* ws, cudaStream_t stream) {
  unsigned long long* hist = static_cast<unsigned long long*>(ws);
  cudaError_t e = launch_zero_words(reinterpret_cast<uint32_t*>(hist), 2 * static_cast<int64_t>(kBins), stream);
  static std::atomic<uint64_t> attr_done{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  const size_t smem = sizeof(uint32_t) * kBins;
  if (e == cudaSuccess && !(attr_done.load() & bit)) {
    e = cudaFuncSetAttribute(abs_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) attr_done.fetch_or(bit);
  }
  if (e == cudaSuccess) {
    const int64_t vecs = rows * (K / 8);
    const int64_t blocks =
        std::max<int64_t>(1, std::min<int64_t>(sm_count(), (vecs + kHistThreads - 1) / kHistThreads));
    e = launch_kernel(abs_hist_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kHistThreads), smem, stream, false,
                      src, rows, K, ld, hist);
  }
  if (e == cudaSuccess)
    e = launch_kernel(select_rank_kernel, dim3(1), dim3(kHistThreads), 0, stream, false,
                      static_cast<const unsigned long long*>(hist), static_cast<unsigned long long>(rank), out);
  return e;
}

}  // namespace sq
