// INT8 x INT8 -> INT32 GEMM on the sm_100a tensor cores (tcgen05.mma kind::i8) with a
// fused dequantization / bias / bf16 epilogue, and the LLM.int8() outlier product
// (tcgen05.mma kind::f16 on bf16 operands) accumulated into a second TMEM accumulator of
// the same output tile and added in the same epilogue.
//
// "量化基础与INT8" INT8推理流程 (INT8 (M,K) x (K,N) -> INT32 accumulate, INT32 -> 16-bit output)
//   and 量化流程示例 (Y = Y_int32 * X_scale * W_scale);
// "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §3.4 (out * (x_scale*w_scale) + bias);
// "LLM.int8()技术解析：8位量化如何优化大语言模型计算" §3.1 (normal columns in an INT8 GEMM,
//   outlier columns in a 16-bit GEMM, results merged).
//
// Structure (one persistent CTA per SM, 6 warps):
//   warp 0     TMA producer: 128x128-byte A tiles and BNx128-byte B tiles into a ring of
//              shared-memory stages (128-byte swizzle), completion on `full` mbarriers;
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (4 x K=32 bytes per stage) into
//              a double-buffered accumulator and frees stages with tcgen05.commit;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one output row per
//              thread), y = (float(acc) * d_m) * e_n (+ o) (+ bias) -> bf16, global stores;
//              overlaps the next tile's main loop through the second TMEM buffer.
// Every mbarrier wait is bounded; on timeout the kernel records an error bit in the
// device status word, drains its own TMA loads and MMAs, frees TMEM and returns.
#include "sq_internal.h"
#include "sq_ptx.cuh"

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

namespace sq {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // bytes of K per stage row: 128 int8 or 64 bf16
constexpr int kThreads = 192;

template <int BN, bool OUTLIERS>
struct Cfg {
  static constexpr int kStageA = kBM * kBK;
  static constexpr int kStageB = BN * kBK;
  static constexpr int kStageBytes = kStageA + kStageB;
  static constexpr int kStages = (200 * 1024) / kStageBytes;
  static constexpr int kAccCols = OUTLIERS ? 2 * BN : BN;  // per buffer: int32 acc (+ fp32 acc)
  static constexpr int kTmemCols = 2 * kAccCols;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM columns");
  static_assert(kStages >= 3, "pipeline depth");
};

struct Params {
  const float* x_scale;
  const float* w_scale;
  int w_per_channel;
  const uint16_t* bias;
  uint16_t* Y;
  int32_t* acc_out;
  int64_t M, N;
  int num_m_tiles, num_n_tiles, num_kb;
  const int32_t* o_count;
  unsigned int* status;
  uint64_t wait_limit_ns;
  int fault;
};

struct Abort {
  volatile int* flag;
  __device__ void raise(unsigned int* status, unsigned int bit) const {
    atomicOr(status, bit);
    *flag = 1;
  }
};

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

template <int BN, bool OUTLIERS>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                 const Params p) {
  using C = Cfg<BN, OUTLIERS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tmem_full = bars + 2 * C::kStages;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* teardown = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const Abort ab{abort_flag};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tmem_full + b, 1);
      mbar_init(tmem_empty + b, 4);
    }
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (OUTLIERS) {
      tma_prefetch_desc(&tmXo);
      tma_prefetch_desc(&tmWo);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.num_m_tiles * p.num_n_tiles;
  const int kb_i8 = p.num_kb;
  int kb_o = 0;
  if constexpr (OUTLIERS) kb_o = (__ldg(p.o_count) + 63) / 64;
  const int kb_total = kb_i8 + kb_o;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;      // stages that received at least one load
      uint32_t issued_parity = 0;    // parity of the last load issued into each stage
      bool withheld = false;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const int m0 = (tile % p.num_m_tiles) * kBM;
        const int n0 = (tile / p.num_m_tiles) * BN;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!wait_or_abort(empty + stage, phase ^ 1, p.wait_limit_ns, abort_flag)) {
            if (!*abort_flag) ab.raise(p.status, kErrProducerWait);
            break;
          }
          if (p.fault == 1 && !withheld) {
            withheld = true;  // test hook: this stage never gets its loads nor its arrival
          } else {
            uint8_t* sa = stage_base + stage * C::kStageBytes;
            uint8_t* sb = sa + C::kStageA;
            mbar_arrive_expect_tx(full + stage, C::kStageBytes);
            if (kb < kb_i8) {
              tma_load_2d(sa, &tmA, full + stage, kb * kBK, m0, kEvictNormal);
              tma_load_2d(sb, &tmB, full + stage, kb * kBK, n0, kEvictNormal);
            } else {
              const int ko = (kb - kb_i8) * (kBK / 2);
              tma_load_2d(sa, &tmXo, full + stage, ko, m0, kEvictNormal);
              tma_load_2d(sb, &tmWo, full + stage, ko, n0, kEvictNormal);
            }
            issued_mask |= 1u << stage;
            issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: every load this thread issued must have landed before the CTA exits
      for (int s = 0; s < C::kStages; ++s) {
        if ((issued_mask >> s) & 1u) {
          if (!mbar_wait_bounded(full + s, (issued_parity >> s) & 1u, p.wait_limit_ns))
            ab.raise(p.status, kErrTeardownWait);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescI8 = idesc_i8_s32(kBM, BN);
      constexpr uint32_t kIdescBf16 = idesc_bf16_f32(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!wait_or_abort(tmem_empty + buf, acc_phase ^ 1, p.wait_limit_ns, abort_flag)) {
          if (!*abort_flag) ab.raise(p.status, kErrMmaWait);
          break;
        }
        tc_fence_after();
        const uint32_t d_i32 = tmem_base + buf * C::kAccCols;
        const uint32_t d_f32 = d_i32 + BN;
        bool ok = true;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!wait_or_abort(full + stage, phase, p.wait_limit_ns, abort_flag)) {
            if (!*abort_flag) ab.raise(p.status, kErrMmaWait);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stage_base + stage * C::kStageBytes);
          const uint32_t b_addr = a_addr + C::kStageA;
          if (kb < kb_i8) {
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_i8(d_i32, smem_desc_k128(a_addr + 32 * k), smem_desc_k128(b_addr + 32 * k), kIdescI8,
                     (kb | k) != 0);
          } else {
            const int ko = kb - kb_i8;
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_f16(d_f32, smem_desc_k128(a_addr + 32 * k), smem_desc_k128(b_addr + 32 * k), kIdescBf16,
                      (ko | k) != 0);
          }
          mma_commit(empty + stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(tmem_full + buf);
      }
      // all MMAs issued by this thread complete before TMEM is released
      mma_commit(teardown);
      if (!mbar_wait_bounded(teardown, 0, p.wait_limit_ns)) ab.raise(p.status, kErrTeardownWait);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
    const int row = quad * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // lane 0 waits and the warp follows its verdict, so the warp stays converged
      int ok = 0;
      if (lane == 0) {
        ok = wait_or_abort(tmem_full + buf, acc_phase, p.wait_limit_ns, abort_flag) ? 1 : 0;
        if (!ok && !*abort_flag) ab.raise(p.status, kErrEpilogueWait);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int64_t m = static_cast<int64_t>(tile % p.num_m_tiles) * kBM + row;
      const int64_t n_tile0 = static_cast<int64_t>(tile / p.num_m_tiles) * BN;
      const bool m_ok = m < p.M;
      const float d_m = m_ok ? __ldg(p.x_scale + m) : 0.0f;
      const float e_all = p.w_per_channel ? 0.0f : __ldg(p.w_scale);
      const uint32_t t_i32 = tmem_base + buf * C::kAccCols + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        __syncwarp();
        uint32_t acc[32];
        uint32_t of[32];
        tmem_ld_32x32b_x32(t_i32 + c * 32, acc);
        if constexpr (OUTLIERS) {
          if (kb_o > 0) tmem_ld_32x32b_x32(t_i32 + BN + c * 32, of);
        }
        tmem_wait_ld();
        const int64_t n0 = n_tile0 + c * 32;
        if (m_ok && n0 < p.N) {
          const int nvalid = (p.N - n0) < 32 ? static_cast<int>(p.N - n0) : 32;  // a multiple of 8
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 e4 = make_float4(e_all, e_all, e_all, e_all);
            if (p.w_per_channel && j < nvalid) e4 = __ldg(reinterpret_cast<const float4*>(p.w_scale + n0 + j));
            const float e[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float v = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(acc[j + u])), d_m), e[u]);
              if constexpr (OUTLIERS) {
                if (kb_o > 0) v = __fadd_rn(v, __uint_as_float(of[j + u]));
              }
              y[j + u] = v;
            }
          }
          if (p.bias != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              if (j < nvalid) {
                const uint4 b = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + j));
                const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  y[j + 2 * u] = __fadd_rn(y[j + 2 * u], __uint_as_float(w[u] << 16));
                  y[j + 2 * u + 1] = __fadd_rn(y[j + 2 * u + 1], __uint_as_float(w[u] & 0xFFFF0000u));
                }
              }
            }
          }
          uint16_t* yrow = p.Y + m * p.N + n0;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            if (j < nvalid) {
              uint4 o;
              o.x = pack_bf16x2(y[j + 0], y[j + 1]);
              o.y = pack_bf16x2(y[j + 2], y[j + 3]);
              o.z = pack_bf16x2(y[j + 4], y[j + 5]);
              o.w = pack_bf16x2(y[j + 6], y[j + 7]);
              *reinterpret_cast<uint4*>(yrow + j) = o;
            }
          }
          if (p.acc_out != nullptr) {
            int32_t* arow = p.acc_out + m * p.N + n0;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              if (j < nvalid)
                *reinterpret_cast<uint4*>(arow + j) = make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty + buf);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D K-major map: inner extent `inner` elements (contiguous), `outer` rows, row pitch
// `pitch_bytes`; box = 128 bytes of K x box_rows rows, 128-byte swizzle, zero OOB fill.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
              uint64_t outer, uint64_t pitch_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK / elem_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int BN, bool OUTLIERS>
cudaError_t run(const GemmArgs& a, cudaStream_t stream, const char** why) {
  using C = Cfg<BN, OUTLIERS>;
  CUtensorMap tmA{}, tmB{}, tmXo{}, tmWo{};
  const uint64_t K = static_cast<uint64_t>(a.K);
  if (!make_map(&tmA, a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, a.M, K, kBM) ||
      !make_map(&tmB, a.Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, a.N, K, BN)) {
    *why = "cuTensorMapEncodeTiled failed for the int8 operands";
    return cudaErrorInvalidValue;
  }
  if (OUTLIERS) {
    const uint64_t ldo = static_cast<uint64_t>(a.ld_o);
    if (!make_map(&tmXo, a.Xo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ldo, a.M, ldo * 2, kBM) ||
        !make_map(&tmWo, a.Wo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ldo, a.N, ldo * 2, BN)) {
      *why = "cuTensorMapEncodeTiled failed for the outlier operands";
      return cudaErrorInvalidValue;
    }
  } else {
    tmXo = tmA;
    tmWo = tmB;
  }
  static std::atomic<uint64_t> attr_done{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(w8a8_gemm_kernel<BN, OUTLIERS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    attr_done.fetch_or(bit);
  }
  Params p{};
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.w_per_channel = a.w_per_channel ? 1 : 0;
  p.bias = a.bias;
  p.Y = a.Y;
  p.acc_out = a.acc_out;
  p.M = a.M;
  p.N = a.N;
  p.num_m_tiles = static_cast<int>((a.M + kBM - 1) / kBM);
  p.num_n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.num_kb = static_cast<int>((a.K + kBK - 1) / kBK);
  p.o_count = a.o_count;
  p.status = device_status_word();
  p.wait_limit_ns = a.wait_limit_ns;
  p.fault = a.fault;
  const int tiles = p.num_m_tiles * p.num_n_tiles;
  const int grid = std::min(tiles, num_sms());
  note_launch();
  w8a8_gemm_kernel<BN, OUTLIERS><<<grid, kThreads, C::kSmemBytes, stream>>>(tmA, tmB, tmXo, tmWo, p);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t, bool) { return 0; }

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream, const char** why) {
  const int sms = num_sms();
  const int64_t m_tiles = (a.M + kBM - 1) / kBM;
  auto tiles = [&](int bn) { return m_tiles * ((a.N + bn - 1) / bn); };
  if (a.Xo != nullptr) {
    if (tiles(128) >= sms) return run<128, true>(a, stream, why);
    return run<64, true>(a, stream, why);
  }
  if (tiles(256) >= sms) return run<256, false>(a, stream, why);
  if (tiles(128) >= sms) return run<128, false>(a, stream, why);
  return run<64, false>(a, stream, why);
}

}  // namespace sq
