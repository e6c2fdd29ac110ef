// INT8 x INT8 -> INT32 GEMM on the sm_100a tensor cores (tcgen05.mma kind::i8) with a
// fused dequantization / bias / bf16 epilogue, and the LLM.int8() outlier product
// (tcgen05.mma kind::f16 on bf16 operands) added by the tensor cores onto the dequantized
// fp32 values of the same output tile, which the epilogue writes back into TMEM.
//
// "量化基础与INT8" INT8推理流程 (INT8 (M,K) x (K,N) -> INT32 accumulate, INT32 -> 16-bit output)
//   and 量化流程示例 (Y = Y_int32 * X_scale * W_scale);
// "SmoothQuant量化实战：W8A8推理部署与单节点530B模型落地" §3.4 (out * (x_scale*w_scale) + bias);
// "LLM.int8()技术解析：8位量化如何优化大语言模型计算" §3.1 (normal columns in an INT8 GEMM,
//   outlier columns in a 16-bit GEMM, results merged).
//
// Up to 4 tokens (no outlier product) take the CUDA-core product of sq_gemv.cu instead.
//
// Structure (one persistent CTA per SM, 10 warps):
//   warp 0     TMA producer: 128x128-byte A tiles and BNx128-byte B tiles into a ring of
//              shared-memory stages (128-byte swizzle), completion on `full` mbarriers;
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (4 x K=32 bytes per stage) into
//              a double-buffered accumulator and frees stages with tcgen05.commit;
//   warps 2-9  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one output row per
//              thread, two column halves), y = (float(acc) * d_m) * e_n (+ bias) -> bf16,
//              TMA stores through shared-memory staging; overlaps the next tile's main loop
//              through the second TMEM buffer.
// For a few tokens (M <= 64) the operands swap roles: the weight supplies the 128-row MMA
// operand (output channels on TMEM lanes) and the tokens the N dimension, so no MMA row
// and no weight byte is spent on padding; the epilogue then applies the per-token scale
// per column and the per-channel scale and bias per row, and stores transposed boxes.
// LLM.int8 (outlier operands): per tile the epilogue turns the int32 accumulator into
// (float(acc) * d_m) * e_n + bias_n in place (tcgen05.st), the MMA warp then adds the bf16
// outlier k-blocks onto it (fp32 accumulation), and the epilogue stores the sum; the outlier
// k-blocks of tile i are issued after the first kOutlierLag int8 k-blocks of tile i+1, so the
// accumulator stays double-buffered and neither product waits for the other.
// Large shapes run on CTA pairs (clusters of 2): each pair computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 issued by the even CTA; each CTA stages its own 128 rows of A
// and 128 rows of B, the loads of both CTAs complete on the even CTA's barriers, and each
// CTA's epilogue drains its own 128 accumulator rows.
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
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kStageTileBytes = 32 * 32 * 2;  // one 32-row x 32-column bf16 output box
constexpr int kEpiBufs = 2;                   // per epilogue warp
constexpr int kEpiSmem = kEpiWarps * kEpiBufs * kStageTileBytes;

// PAIR: a CTA pair computes one 256 x BN tile; each CTA stages its 128 rows of A and half
// of the BN rows of B, so a stage holds 32 KB instead of 48 at BN = 256 and the ring gets
// 6 stages.
// TMEM: ACC_BUFS = 2 accumulators of BN columns each (columns [b*BN, (b+1)*BN)), so the
// epilogue of tile i overlaps the main loop of tile i+1. With OUTLIERS (LLM.int8) the same
// buffer serves both products of a tile: the int8 MMAs accumulate int32 there; the epilogue
// converts it to the dequantized fp32 value (float(acc) * d_m) * e_n + bias_n and writes that
// back into the same columns; the bf16 MMAs of the outlier columns then add their product onto
// it (fp32 accumulation on the tensor cores), and the epilogue reads the sum and stores it as
// bf16. The outlier MMAs of tile i are issued after the first kOutlierLag int8 k-blocks of
// tile i+1, by which time the epilogue has written tile i back, so neither product waits for
// the other in the common case.
constexpr int pow2_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }
// Bytes of one K-split unit's int32 partial in the workspace: every epilogue warp's 32 rows x 32
// columns for each chunk of its column half (the larger half when BN / 32 is odd).
constexpr int64_t split_slot_bytes(int bn) {
  return static_cast<int64_t>(kEpiWarps) * ((bn / 32 + 1) / 2) * 32 * 32 * 4;
}
constexpr int kOutlierLag = 8;
template <int BN, bool OUTLIERS, int ACC_BUFS, bool PAIR = false>
struct Cfg {
  static constexpr int kBN = BN;
  static constexpr int kStageA = kBM * kBK;
  static constexpr int kStageB = (PAIR ? BN / 2 : BN) * kBK;
  static constexpr int kStageBytes = kStageA + kStageB;
  static constexpr int kStages = (192 * 1024) / kStageBytes;
  static constexpr int kUsedCols = ACC_BUFS * BN;
  static constexpr int kTmemCols = pow2_cols(kUsedCols);  // allocations are powers of two
  static constexpr int kChunksTotal = BN / 32;             // 32-column chunks of a tile
  static constexpr int kChunks = (kChunksTotal + 1) / 2;   // per epilogue column half (at most)
  static constexpr int kBarOffset = kStages * kStageBytes + kEpiSmem;
  static constexpr int kSmemBytes = kBarOffset + 256 /*barriers*/ + 1024 /*alignment slack*/;
  static_assert(ACC_BUFS == 2, "double-buffered int32 accumulator");
  static_assert(kUsedCols <= 512, "TMEM columns");
  static_assert(kStages >= 3, "pipeline depth");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kStageB % 1024 == 0, "B tile of whole 128-byte swizzle atoms");
  static_assert(BN % 32 == 0, "epilogue chunks of 32 columns");
  static_assert(2 * kStages + 4 * ACC_BUFS + 1 <= 30, "barrier area");
};

struct Params {
  const float* x_scale;
  int x_per_token;           // x_scale has M entries (else 1)
  const int32_t* x_zero;     // asymmetric activations: per-token zero points [M], or nullptr
  const int32_t* w_rowsum;   // sum_k Wq[n,k] [N] (with x_zero)
  const float* w_scale;
  int w_per_channel;
  const uint16_t* bias;
  int32_t* acc_out;
  int64_t M, N;
  // Tile space: `rows` along the 128-row MMA operand, `cols` along the BN-column one
  // (M and N, or N and M when the operands are swapped).
  int64_t rows, cols;
  int num_m_tiles, num_n_tiles, num_kb;
  // Work units: units [0, num_full) are whole output tiles (tile index = unit); the tiles
  // after them ("tail" tiles) are split along K into `splits` units of kb_per_split k-blocks,
  // whose exact int32 partials meet in the workspace.
  int num_full;
  int num_units;
  int splits;
  int kb_per_split;
  int32_t* partials;   // [tail tiles * splits][kEpiWarps][BN/64 chunks][8][32 lanes] int4 (int32 x4)
  int32_t* counters;   // [tail tiles * kEpiWarps] arrival counters, zero between calls
  int64_t partial_int4;  // int4 elements of the partials region (bounds guard)
  const int32_t* o_count;
  // short (programmatic) launches: the weight tiles of the CTA's first work unit are
  // prefetched into L2 before the wait on the previous kernel (the weight does not depend
  // on it in a decode step; a prefetch is only a hint, so it is safe even when it does)
  int prefetch_weight;
  unsigned int* status;
  uint64_t wait_limit_ns;
  int fault;
};

struct Abort {
  volatile int* flag;
  uint32_t peer_flag;  // the other CTA's flag (shared::cluster address) in a CTA pair, else 0
  __device__ void raise(unsigned int* status, unsigned int bit) const {
    atomicOr(status, bit);
    *flag = 1;
    if (peer_flag != 0) st_cluster_u32(peer_flag, 1u);
  }
};

struct Unit {
  int tile_mn;  // output tile (m fastest)
  int split;    // part of a split tail tile (0 for whole tiles)
  int kb0, kb1; // int8 k-block range
  bool is_split;
};

__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit w;
  if (u < p.num_full) {
    w.tile_mn = u;
    w.split = 0;
    w.kb0 = 0;
    w.kb1 = p.num_kb;
    w.is_split = false;
  } else {
    const int v = u - p.num_full;
    w.tile_mn = p.num_full + v / p.splits;
    w.split = v % p.splits;
    w.kb0 = w.split * p.kb_per_split;
    w.kb1 = min(p.num_kb, w.kb0 + p.kb_per_split);
    w.is_split = true;
  }
  return w;
}

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

// bf16_rne(lo) in the low half, bf16_rne(hi) in the high half (one conversion instruction).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Swapped operands (tokens on the columns): per-warp token constants of a 32-column chunk,
// spread over the lanes: lane l holds the per-token scales of columns 4*(l%8)..4*(l%8)+3 of
// chunk l/8 (and their zero points with asymmetric activations), so a warp covers 4 chunks
// (128 tokens). Loaded before the accumulator is ready. x_scale / x_zero have no alignment
// contract and M need not be a multiple of 4: scalar loads.
struct TokenConsts {
  float4 d;
  int4 z;  // asymmetric activations: the token's zero point
};

template <bool ASYM>
__device__ __forceinline__ TokenConsts load_token_consts(const Params& p, int64_t n_half0, int lane, int chunks) {
  TokenConsts tc;
  const int c = lane >> 3;
  const int64_t n = n_half0 + c * 32 + (lane & 7) * 4;
  const bool ok = c < chunks && n < p.cols;
  float v[4];
  int zz[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool in = ok && n + i < p.cols;
    v[i] = in ? __ldg(p.x_scale + (p.x_per_token ? n + i : 0)) : 0.0f;
    zz[i] = (ASYM && in) ? __ldg(p.x_zero + n + i) : 0;
  }
  tc.d = make_float4(v[0], v[1], v[2], v[3]);
  tc.z = make_int4(zz[0], zz[1], zz[2], zz[3]);
  return tc;
}

// Swapped operands: y[j] = (float(acc[j]) * d_m) * e_n for the 32 tokens m of chunk c of
// output channel n (the thread's row): d_m comes from the lanes' token constants (shuffled),
// e_n is the row constant. With asymmetric activations acc is first corrected in 64-bit
// integers, acc - z_m * rowsum_n (rowsum_n is the row's integer factor).
template <bool ASYM>
__device__ __forceinline__ void dequant32_tokens(const uint32_t (&acc)[32], float row_scale, int row_int,
                                                 const TokenConsts& tc, int c, float (&y)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const int src = c * 8 + j / 4;
    const float d[4] = {__shfl_sync(0xffffffffu, tc.d.x, src), __shfl_sync(0xffffffffu, tc.d.y, src),
                        __shfl_sync(0xffffffffu, tc.d.z, src), __shfl_sync(0xffffffffu, tc.d.w, src)};
    int zc[4] = {0, 0, 0, 0};
    if constexpr (ASYM) {
      zc[0] = __shfl_sync(0xffffffffu, tc.z.x, src);
      zc[1] = __shfl_sync(0xffffffffu, tc.z.y, src);
      zc[2] = __shfl_sync(0xffffffffu, tc.z.z, src);
      zc[3] = __shfl_sync(0xffffffffu, tc.z.w, src);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float a;
      if constexpr (ASYM) {
        const long long t = static_cast<long long>(static_cast<int32_t>(acc[j + u])) -
                            static_cast<long long>(row_int) * static_cast<long long>(zc[u]);
        a = __ll2float_rn(t);
      } else {
        a = static_cast<float>(static_cast<int32_t>(acc[j + u]));
      }
      y[j + u] = __fmul_rn(__fmul_rn(a, d[u]), row_scale);
    }
  }
}

// Swapped operands: y[j] += the row's (output channel's) bias when there is one, then pack
// to bf16 pairs.
__device__ __forceinline__ void bias_pack32_tokens(float (&y)[32], bool has_bias, float row_bias,
                                                   uint32_t (&out)[16]) {
  if (has_bias) {
#pragma unroll
    for (int j = 0; j < 32; ++j) y[j] = __fadd_rn(y[j], row_bias);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) out[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
}

// Operands not swapped (output channels on the columns): y[j] = (float(acc[j]) * d_m) * e_n
// with d_m the row constant, then + bias_n and bf16 packing; the column constants of columns
// n0..n0+31 are read by every lane from the same addresses (one broadcast load per 4 scales,
// per 8 biases): fewer instructions than spreading them over the lanes and shuffling. With
// asymmetric activations acc is first corrected in 64-bit integers, acc - z_m * rowsum_n.
// N is a multiple of 8 and w_scale / bias are 16-byte aligned, so each vector load lies
// wholly inside or wholly past the end of its array (then it is skipped).
template <bool ASYM>
__device__ __forceinline__ void dequant32_cols(const Params& p, const uint32_t (&acc)[32], float row_scale,
                                               int row_int, int64_t n0, float (&y)[32]) {
  const float e_t = p.w_per_channel ? 0.0f : __ldg(p.w_scale);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const int64_t n = n0 + j;
    const bool in = n < p.cols;
    float4 e4 = make_float4(e_t, e_t, e_t, e_t);
    if (p.w_per_channel)
      e4 = in ? __ldg(reinterpret_cast<const float4*>(p.w_scale + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float e[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float a;
      if constexpr (ASYM) {
        const int rs = in ? __ldg(p.w_rowsum + n + u) : 0;
        const long long t = static_cast<long long>(static_cast<int32_t>(acc[j + u])) -
                            static_cast<long long>(row_int) * static_cast<long long>(rs);
        a = __ll2float_rn(t);
      } else {
        a = static_cast<float>(static_cast<int32_t>(acc[j + u]));
      }
      y[j + u] = __fmul_rn(__fmul_rn(a, row_scale), e[u]);
    }
  }
}

__device__ __forceinline__ void add_bias32_cols(const Params& p, float (&y)[32], bool has_bias, int64_t n0) {
  if (has_bias) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const int64_t n = n0 + j;
      const uint4 b4 = n < p.cols ? __ldg(reinterpret_cast<const uint4*>(p.bias + n)) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t b[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        y[j + 2 * u] = __fadd_rn(y[j + 2 * u], __uint_as_float(b[u] << 16));
        y[j + 2 * u + 1] = __fadd_rn(y[j + 2 * u + 1], __uint_as_float(b[u] & 0xFFFF0000u));
      }
    }
  }
}

__device__ __forceinline__ void bias_pack32_cols(const Params& p, float (&y)[32], bool has_bias, int64_t n0,
                                                 uint32_t (&out)[16]) {
  add_bias32_cols(p, y, has_bias, n0);
#pragma unroll
  for (int j = 0; j < 16; ++j) out[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
}

// Debug copy of the int32 accumulators of one 32-column chunk (nvalid valid columns) of
// tile row r; with swapped operands the row is output channel r and the columns tokens.
template <bool SWAP>
__device__ __forceinline__ void store_acc32(const Params& p, const uint32_t (&acc)[32], int64_t r, int64_t n0,
                                            int nvalid) {
  if constexpr (SWAP) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) p.acc_out[(n0 + j) * p.N + r] = static_cast<int32_t>(acc[j]);
  } else {
    int32_t* arow = p.acc_out + r * p.N + n0;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      if (j < nvalid) *reinterpret_cast<uint4*>(arow + j) = make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
  }
}

// One 32x32 bf16 box through the warp's staging buffer to a TMA store. Each lane holds
// 32 values of its tile row. Normally the row is an output row: the box is stored at
// (column n0, row row0) with one staging row per lane. With swapped operands the lane's
// row is an output channel, so lane l writes staging column l of 32 token rows and the
// box goes to (channel row0, token n0).
template <bool SWAP>
__device__ __forceinline__ void store_box(const uint32_t (&v)[16], uint8_t* stage_tiles, int& ebuf, int lane,
                                          const CUtensorMap* tmY, int64_t n0, int64_t row0) {
  // staging buffer `ebuf` was last read by the TMA store issued two boxes ago
  if (lane == 0) bulk_wait_group_read<kEpiBufs - 1>();
  __syncwarp();
  uint8_t* tile = stage_tiles + ebuf * kStageTileBytes;
  if constexpr (SWAP) {
    uint16_t* st = reinterpret_cast<uint16_t*>(tile) + lane;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      st[(2 * j) * 32] = static_cast<uint16_t>(v[j] & 0xFFFFu);
      st[(2 * j + 1) * 32] = static_cast<uint16_t>(v[j] >> 16);
    }
  } else {
    // the output map uses the 64-byte swizzle: 16-byte granule j of staging row l sits at
    // granule j ^ ((l >> 1) & 3) (the tile is 2048-byte aligned), so the 32 lanes' stores
    // spread over all eight 16-byte bank groups (4 wavefronts per instruction, not 16)
    uint4* st = reinterpret_cast<uint4*>(tile + lane * 64);
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) st[j ^ sw] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if constexpr (SWAP)
      tma_store_2d(tmY, tile, static_cast<int32_t>(row0), static_cast<int32_t>(n0));
    else
      tma_store_2d(tmY, tile, static_cast<int32_t>(n0), static_cast<int32_t>(row0));
    bulk_commit_group();
  }
  ebuf ^= 1;
}

// The single-thread roles walk the ring of shared-memory stages in the same order.
struct Ring {
  int stage;
  uint32_t phase;
  uint32_t issued_mask;    // producer: stages that received at least one load
  uint32_t issued_parity;  // producer: parity of the last load issued into each stage
  bool withheld;           // producer: the test hook's withheld stage
};

struct LoadCtx {
  const Params* p;
  const Abort* ab;
  volatile int* abort_flag;
  uint64_t* full;
  uint64_t* empty;
  uint8_t* stage_base;
  bool leader;
};

// TMA producer: `count` k-blocks, block i at column x0 + i * x_step of map_a (rows ya) and
// map_b (rows yb), each into the next stage once the MMAs have freed it.
template <class C, bool PAIR>
__device__ __forceinline__ bool load_blocks(Ring& r, const LoadCtx& c, const CUtensorMap* map_a,
                                            const CUtensorMap* map_b, int x0, int x_step, int count, int ya,
                                            int yb) {
  const Params& p = *c.p;
  for (int i = 0; i < count; ++i) {
    if (!wait_or_abort(c.empty + r.stage, r.phase ^ 1, p.wait_limit_ns, c.abort_flag)) {
      if (!*c.abort_flag) c.ab->raise(p.status, kErrProducerWait);
      return false;
    }
    if (p.fault == 1 && !r.withheld) {
      r.withheld = true;  // test hook: this stage never gets its loads nor its arrival
    } else {
      uint8_t* sa = c.stage_base + r.stage * C::kStageBytes;
      uint8_t* sb = sa + C::kStageA;
      const int x = x0 + i * x_step;
      if constexpr (PAIR) {
        // both CTAs' halves complete on the even CTA's barrier, which expects them all
        if (c.leader) mbar_arrive_expect_tx(c.full + r.stage, 2 * C::kStageBytes);
        const uint32_t fb = mapa_shared(c.full + r.stage, 0);
        tma_load_2d_pair(sa, map_a, fb, x, ya, kEvictNormal);
        tma_load_2d_pair(sb, map_b, fb, x, yb, kEvictNormal);
      } else {
        mbar_arrive_expect_tx(c.full + r.stage, C::kStageBytes);
        tma_load_2d(sa, map_a, c.full + r.stage, x, ya, kEvictNormal);
        tma_load_2d(sb, map_b, c.full + r.stage, x, yb, kEvictNormal);
      }
      r.issued_mask |= 1u << r.stage;
      r.issued_parity = (r.issued_parity & ~(1u << r.stage)) | (r.phase << r.stage);
    }
    if (++r.stage == C::kStages) {
      r.stage = 0;
      r.phase ^= 1;
    }
  }
  return true;
}

struct MmaCtx {
  const Params* p;
  const Abort* ab;
  volatile int* abort_flag;
  uint64_t* full;
  uint64_t* empty;
  uint8_t* stage_base;
  uint32_t empty_c0, empty_c1;  // a pair's stage barriers in each CTA (shared::cluster)
};

// MMA issuer: `count` stages into the accumulator at d, int8 x int8 -> int32 (the first
// instruction starts the accumulation when `start`), or with BF16 the outlier columns,
// bf16 x bf16 added onto the fp32 values d holds. Each stage is freed by a commit.
template <class C, bool PAIR, bool BF16>
__device__ __forceinline__ bool mma_blocks(Ring& r, const MmaCtx& c, uint32_t d, int count, bool start) {
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  constexpr uint32_t kIdesc = BF16 ? idesc_bf16_f32(kTileM, C::kBN) : idesc_i8_s32(kTileM, C::kBN);
  const Params& p = *c.p;
  for (int i = 0; i < count; ++i) {
    if (!wait_or_abort(c.full + r.stage, r.phase, p.wait_limit_ns, c.abort_flag)) {
      if (!*c.abort_flag) c.ab->raise(p.status, kErrMmaWait);
      return false;
    }
    tc_fence_after();
    const uint32_t a_addr = smem_u32(c.stage_base + r.stage * C::kStageBytes);
    const uint32_t b_addr = a_addr + C::kStageA;
#pragma unroll
    for (int k = 0; k < kBK / 32; ++k) {
      const uint32_t acc = (BF16 || !start || i != 0 || k != 0) ? 1u : 0u;
      const uint64_t da = smem_desc_k128(a_addr + 32 * k), db = smem_desc_k128(b_addr + 32 * k);
      if constexpr (PAIR) {
        if constexpr (BF16)
          mma_f16_pair(d, da, db, kIdesc, acc);
        else
          mma_i8_pair(d, da, db, kIdesc, acc);
      } else {
        if constexpr (BF16)
          mma_f16(d, da, db, kIdesc, acc);
        else
          mma_i8(d, da, db, kIdesc, acc);
      }
    }
    if constexpr (PAIR) {
      mma_commit_pair(c.empty_c0 + 8u * r.stage);
      mma_commit_pair(c.empty_c1 + 8u * r.stage);
    } else {
      mma_commit(c.empty + r.stage);
    }
    if (++r.stage == C::kStages) {
      r.stage = 0;
      r.phase ^= 1;
    }
  }
  return true;
}

template <int BN, bool OUTLIERS, int ACC_BUFS, bool SWAP, bool ASYM, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                 const __grid_constant__ CUtensorMap tmY, const Params p) {
  using C = Cfg<BN, OUTLIERS, ACC_BUFS, PAIR>;
  static_assert(!PAIR || (!SWAP && BN == 256), "CTA pairs: 256 x 256 tiles, operands not swapped");
  // rows of A per output tile: one CTA's 128, or a pair's 256 (this CTA's half at rank * 128)
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + C::kStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tmem_full = bars + 2 * C::kStages;
  uint64_t* tmem_empty = tmem_full + ACC_BUFS;
  uint64_t* y_ready = tmem_empty + ACC_BUFS;    // outlier form: dequantized values written back
  uint64_t* tmem_full2 = y_ready + ACC_BUFS;    // outlier form: outlier product added
  uint64_t* teardown = tmem_full2 + ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;  // the pair's MMA issuer (always true for a single CTA)
  const Abort ab{abort_flag, PAIR ? mapa_shared(const_cast<int*>(abort_flag), rank ^ 1u) : 0u};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // work units of this CTA (a pair walks them together)
  const int u_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int u_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      mbar_init(tmem_full + b, 1);
      mbar_init(tmem_empty + b, PAIR ? 2 * kEpiWarps : kEpiWarps);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      mbar_init(y_ready + b, PAIR ? 2 * kEpiWarps : kEpiWarps);
      mbar_init(tmem_full2 + b, 1);
    }
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
    if (OUTLIERS) {
      tma_prefetch_desc(&tmXo);
      tma_prefetch_desc(&tmWo);
    }
    if (p.prefetch_weight && u_first < p.num_units) {
      // the weight is the 128-row operand A when the operands are swapped, else B
      const Unit w = unit_of(p, u_first);
      const int y = SWAP ? (w.tile_mn % p.num_m_tiles) * kTileM + static_cast<int>(rank) * kBM
                         : (w.tile_mn / p.num_m_tiles) * BN + (PAIR ? static_cast<int>(rank) * (BN / 2) : 0);
      for (int kb = w.kb0; kb < w.kb1; ++kb) tma_prefetch_l2_2d(SWAP ? &tmA : &tmB, kb * kBK, y);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync();  // both CTAs' barriers initialised before any remote arrive or copy
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up done: from here on global memory written by the previous kernel is read
  griddep_wait();
  griddep_launch_dependents();

  const int num_units = p.num_units;
  int kb_o = 0;
  if constexpr (OUTLIERS) kb_o = (__ldg(p.o_count) + 63) / 64;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      Ring ring{};
      const LoadCtx lc{&p, &ab, abort_flag, full, empty, stage_base, leader};
      if (!OUTLIERS || kb_o == 0) {
        // plain form: each unit's k-blocks in order
        for (int u = u_first; u < num_units && !*abort_flag; u += u_step) {
          const Unit w = unit_of(p, u);
          const int m0 = (w.tile_mn % p.num_m_tiles) * kTileM + static_cast<int>(rank) * kBM;
          const int n0 = (w.tile_mn / p.num_m_tiles) * BN + (PAIR ? static_cast<int>(rank) * (BN / 2) : 0);
          if (!load_blocks<C, PAIR>(ring, lc, &tmA, &tmB, w.kb0 * kBK, kBK, w.kb1 - w.kb0, m0, n0)) break;
        }
      } else {
        // outlier form: the previous unit's outlier k-blocks (bf16, 64 columns = 128 bytes
        // per row: the same stage geometry) after the first kOutlierLag int8 k-blocks of
        // each unit, and the last unit's after the last unit
        bool ok = true;
        int j = 0, prev_m0 = 0, prev_n0 = 0;
        for (int u = u_first; u < num_units && !*abort_flag; u += u_step, ++j) {
          const Unit w = unit_of(p, u);
          const int m0 = (w.tile_mn % p.num_m_tiles) * kTileM + static_cast<int>(rank) * kBM;
          const int n0 = (w.tile_mn / p.num_m_tiles) * BN + (PAIR ? static_cast<int>(rank) * (BN / 2) : 0);
          const int nk = w.kb1 - w.kb0;
          const int ins = min(kOutlierLag, nk);
          ok = load_blocks<C, PAIR>(ring, lc, &tmA, &tmB, w.kb0 * kBK, kBK, ins, m0, n0);
          if (ok && j > 0) ok = load_blocks<C, PAIR>(ring, lc, &tmXo, &tmWo, 0, kBK / 2, kb_o, prev_m0, prev_n0);
          if (ok) ok = load_blocks<C, PAIR>(ring, lc, &tmA, &tmB, (w.kb0 + ins) * kBK, kBK, nk - ins, m0, n0);
          if (!ok) break;
          prev_m0 = m0;
          prev_n0 = n0;
        }
        if (ok && j > 0 && !*abort_flag)
          load_blocks<C, PAIR>(ring, lc, &tmXo, &tmWo, 0, kBK / 2, kb_o, prev_m0, prev_n0);
      }
      // drain: every load this thread issued must have landed before the CTA exits (a
      // pair's odd CTA counts its copies on the even CTA's barriers, which the even CTA
      // drains before the final cluster barrier)
      for (int s = 0; s < C::kStages; ++s) {
        if (leader && ((ring.issued_mask >> s) & 1u)) {
          if (!mbar_wait_bounded(full + s, (ring.issued_parity >> s) & 1u, p.wait_limit_ns))
            ab.raise(p.status, kErrTeardownWait);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      // a pair's commits go to the barrier in each CTA (shared::cluster addresses)
      const uint32_t tfull_c0 = PAIR ? mapa_shared(tmem_full, 0) : 0u;
      const uint32_t tfull_c1 = PAIR ? mapa_shared(tmem_full, 1) : 0u;
      const uint32_t tfull2_c0 = PAIR ? mapa_shared(tmem_full2, 0) : 0u;
      const uint32_t tfull2_c1 = PAIR ? mapa_shared(tmem_full2, 1) : 0u;
      Ring ring{};
      const MmaCtx mc{&p, &ab, abort_flag, full, empty, stage_base, PAIR ? mapa_shared(empty, 0) : 0u,
                      PAIR ? mapa_shared(empty, 1) : 0u};
      auto commit_to = [&](uint64_t* bar, uint32_t c0, uint32_t c1, int b) {
        if constexpr (PAIR) {
          mma_commit_pair(c0 + 8u * b);
          mma_commit_pair(c1 + 8u * b);
        } else {
          mma_commit(bar + b);
        }
      };
      bool ok = true;
      int it = 0;
      for (int u = u_first; u < num_units && !*abort_flag; u += u_step, ++it) {
        const int buf = it % ACC_BUFS;
        const uint32_t acc_phase = (it / ACC_BUFS) & 1;
        if (!wait_or_abort(tmem_empty + buf, acc_phase ^ 1, p.wait_limit_ns, abort_flag)) {
          if (!*abort_flag) ab.raise(p.status, kErrMmaWait);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_i32 = tmem_base + buf * BN;
        const Unit w = unit_of(p, u);
        const int nk = w.kb1 - w.kb0;
        if (!OUTLIERS || kb_o == 0) {
          ok = mma_blocks<C, PAIR, false>(ring, mc, d_i32, nk, true);
        } else {
          const int ins = min(kOutlierLag, nk);
          ok = mma_blocks<C, PAIR, false>(ring, mc, d_i32, ins, true);
          if (ok && it > 0) {
            // the previous unit's outlier product starts once the epilogue has written its
            // dequantized fp32 values back into its buffer
            const int pit = it - 1;
            ok = wait_or_abort(y_ready + pit % ACC_BUFS, (pit / ACC_BUFS) & 1, p.wait_limit_ns, abort_flag);
            if (!ok && !*abort_flag) ab.raise(p.status, kErrMmaWait);
            if (ok) {
              tc_fence_after();
              ok = mma_blocks<C, PAIR, true>(ring, mc, tmem_base + (pit % ACC_BUFS) * BN, kb_o, false);
            }
            if (ok) commit_to(tmem_full2, tfull2_c0, tfull2_c1, pit % ACC_BUFS);
          }
          if (ok) ok = mma_blocks<C, PAIR, false>(ring, mc, d_i32, nk - ins, false);
        }
        if (!ok) break;
        commit_to(tmem_full, tfull_c0, tfull_c1, buf);
      }
      // the last unit's outlier product
      if (OUTLIERS && kb_o > 0 && ok && it > 0 && !*abort_flag) {
        const int pit = it - 1;
        ok = wait_or_abort(y_ready + pit % ACC_BUFS, (pit / ACC_BUFS) & 1, p.wait_limit_ns, abort_flag);
        if (!ok && !*abort_flag) ab.raise(p.status, kErrMmaWait);
        if (ok) {
          tc_fence_after();
          ok = mma_blocks<C, PAIR, true>(ring, mc, tmem_base + (pit % ACC_BUFS) * BN, kb_o, false);
        }
        if (ok) commit_to(tmem_full2, tfull2_c0, tfull2_c1, pit % ACC_BUFS);
      }
      // all MMAs issued by this thread complete before TMEM is released (in both CTAs of a
      // pair: the odd CTA frees its TMEM only after the final cluster barrier)
      if constexpr (PAIR)
        mma_commit_pair(smem_u32(teardown));
      else
        mma_commit(teardown);
      if (!mbar_wait_bounded(teardown, 0, p.wait_limit_ns)) ab.raise(p.status, kErrTeardownWait);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // 8 warps: warp w reads TMEM lanes [32*(w%4), +32) (one output row per thread) and
    // the column half (w-2)/4 of the tile, 32 columns at a time (half 0 takes the first
    // kChunks chunks, half 1 the rest: 4 + 4 at BN = 256, 3 + 2 at BN = 160). The whole
    // half-row is dequantized into registers (packed bf16) first, so the accumulators are
    // handed back to the MMA warp before the stores; each 32x32 bf16 box then goes through
    // this warp's staging buffer in shared memory to a TMA store.
    constexpr int kChunks = C::kChunks;  // 32-column chunks per warp (at most)
    static_assert(!(SWAP && OUTLIERS) && !(ASYM && OUTLIERS), "no outlier product with these forms");
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int my_chunks = half == 0 ? kChunks : C::kChunksTotal - kChunks;
    const int row = quad * 32 + lane;
    uint8_t* stage_tiles = epi_base + (warp - 2) * kEpiBufs * kStageTileBytes;
    int ebuf = 0;
    int it = 0;
    // a pair's odd CTA hands the accumulators back on the even CTA's barriers
    const uint32_t tempty_c0 = PAIR ? mapa_shared(tmem_empty, 0) : 0u;
    const uint32_t yready_c0 = PAIR ? mapa_shared(y_ready, 0) : 0u;
    for (int u = u_first; u < num_units; u += u_step, ++it) {
      const int buf = it % ACC_BUFS;
      const uint32_t acc_phase = (it / ACC_BUFS) & 1;
      // everything that does not need the accumulator is fetched before waiting for it
      const Unit w = unit_of(p, u);
      const int tile_mn = w.tile_mn;
      const int split = w.split;
      const int64_t m_tile0 = static_cast<int64_t>(tile_mn % p.num_m_tiles) * kTileM + rank * kBM;
      const int64_t r = m_tile0 + row;  // this thread's tile row (output row, or channel if swapped)
      const int64_t box_row0 = m_tile0 + quad * 32;
      const bool rows_live = box_row0 < p.rows;  // uniform across the warp
      const int64_t n_half0 = static_cast<int64_t>(tile_mn / p.num_m_tiles) * BN + half * (kChunks * 32);
      const bool r_ok = r < p.rows;
      float row_scale = 0.0f, row_bias = 0.0f;
      int row_int = 0;
      if constexpr (SWAP) {
        if (r_ok) {
          row_scale = __ldg(p.w_scale + (p.w_per_channel ? r : 0));
          if (p.bias != nullptr) row_bias = __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + r)) << 16);
          if constexpr (ASYM) row_int = __ldg(p.w_rowsum + r);
        }
      } else {
        if (r_ok) {
          row_scale = __ldg(p.x_scale + (p.x_per_token ? r : 0));
          if constexpr (ASYM) row_int = __ldg(p.x_zero + r);
        }
      }
      // swapped operands spread the per-token column constants over the lanes; otherwise
      // the column constants are broadcast loads inside the chunk loop
      TokenConsts tc{};
      if constexpr (SWAP) tc = load_token_consts<ASYM>(p, n_half0, lane, my_chunks);
      const bool has_bias = p.bias != nullptr;
      // lane 0 waits and the warp follows its verdict, so the warp stays converged
      int ok = 0;
      if (lane == 0) {
        ok = wait_or_abort(tmem_full + buf, acc_phase, p.wait_limit_ns, abort_flag) ? 1 : 0;
        if (!ok && !*abort_flag) ab.raise(p.status, kErrEpilogueWait);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
      const uint32_t t_row = tmem_base + buf * BN + lane_off + half * (kChunks * 32);
      if constexpr (OUTLIERS) {
        // LLM.int8 form (tiles are never split). With outlier columns, pass 1 turns the int8
        // product into its dequantized fp32 value (+ bias) in place and hands it to the MMA
        // warp, whose bf16 MMAs add the outlier product onto it.
        if (kb_o > 0) {
#pragma unroll 1
          for (int c = 0; c < my_chunks; ++c) {
            const int64_t n0 = n_half0 + c * 32;
            if (n0 >= p.cols) break;  // uniform across the warp
            __syncwarp();
            uint32_t acc[32];
            tmem_ld_32x32b_x32(t_row + c * 32, acc);
            tmem_wait_ld();
            const int nvalid = (p.cols - n0) < 32 ? static_cast<int>(p.cols - n0) : 32;
            if (p.acc_out != nullptr && r_ok) store_acc32<false>(p, acc, r, n0, nvalid);
            float y[32];
            dequant32_cols<false>(p, acc, row_scale, 0, n0, y);
            add_bias32_cols(p, y, has_bias, n0);
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = __float_as_uint(y[j]);
            tmem_st_32x32b_x32(t_row + c * 32, acc);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR)
              mbar_arrive_remote(yready_c0 + 8u * buf);
            else
              mbar_arrive(y_ready + buf);
          }
          int ok2 = 0;
          if (lane == 0) {
            ok2 = wait_or_abort(tmem_full2 + buf, acc_phase, p.wait_limit_ns, abort_flag) ? 1 : 0;
            if (!ok2 && !*abort_flag) ab.raise(p.status, kErrEpilogueWait);
          }
          ok2 = __shfl_sync(0xffffffffu, ok2, 0);
          if (!ok2) break;
          tc_fence_after();
        }
        // last pass: the sum with the outlier product (or, with no outlier column, the int8
        // product dequantized here) -> packed bf16 in registers; the buffer is handed back
        // before the stores
        uint32_t packed[kChunks][16];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int64_t n0 = n_half0 + c * 32;
          if (c < my_chunks && n0 < p.cols) {  // uniform across the warp
            __syncwarp();
            uint32_t v[32];
            tmem_ld_32x32b_x32(t_row + c * 32, v);
            tmem_wait_ld();
            if (kb_o > 0) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                packed[c][j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            } else {
              const int nvalid = (p.cols - n0) < 32 ? static_cast<int>(p.cols - n0) : 32;
              if (p.acc_out != nullptr && r_ok) store_acc32<false>(p, v, r, n0, nvalid);
              float y[32];
              dequant32_cols<false>(p, v, row_scale, 0, n0, y);
              bias_pack32_cols(p, y, has_bias, n0, packed[c]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR)
            mbar_arrive_remote(tempty_c0 + 8u * buf);
          else
            mbar_arrive(tmem_empty + buf);
        }
        if (rows_live) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const int64_t n0 = n_half0 + c * 32;
            if (c < my_chunks && n0 < p.cols) store_box<false>(packed[c], stage_tiles, ebuf, lane, &tmY, n0, box_row0);
          }
        }
      } else if (!w.is_split) {
        uint32_t packed[kChunks][16];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int64_t n0 = n_half0 + c * 32;
          if (c < my_chunks && n0 < p.cols) {  // uniform across the warp
            __syncwarp();
            uint32_t acc[32];
            tmem_ld_32x32b_x32(t_row + c * 32, acc);
            tmem_wait_ld();
            const int nvalid = (p.cols - n0) < 32 ? static_cast<int>(p.cols - n0) : 32;
            float y[32];
            if constexpr (SWAP)
              dequant32_tokens<ASYM>(acc, row_scale, row_int, tc, c, y);
            else
              dequant32_cols<ASYM>(p, acc, row_scale, row_int, n0, y);
            if (p.acc_out != nullptr && r_ok) store_acc32<SWAP>(p, acc, r, n0, nvalid);
            if constexpr (SWAP)
              bias_pack32_tokens(y, has_bias, row_bias, packed[c]);
            else
              bias_pack32_cols(p, y, has_bias, n0, packed[c]);
          }
        }
        // the accumulator is no longer needed: hand it back before storing
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR)
            mbar_arrive_remote(tempty_c0 + 8u * buf);
          else
            mbar_arrive(tmem_empty + buf);
        }
        if (rows_live) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const int64_t n0 = n_half0 + c * 32;
            if (c < my_chunks && n0 < p.cols) store_box<SWAP>(packed[c], stage_tiles, ebuf, lane, &tmY, n0, box_row0);
          }
        }
      } else {
        // K split: this split's int32 partial goes to the workspace; the warp that brings
        // the last split of its 32-row x BN/2 sub-tile sums all partials (exact) and stores Y.
        // Partials are stored warp-contiguous (lane-minor), so every access moves 512 bytes.
        const int64_t tail = tile_mn - p.num_full;
        constexpr int64_t kSlotInt4 = split_slot_bytes(BN) / 16;
        static_assert(kSlotInt4 == static_cast<int64_t>(kEpiWarps) * kChunks * 8 * 32, "slot layout");
        auto part_ptr = [&](int sidx, int c) {
          return reinterpret_cast<int4*>(p.partials) + (tail * p.splits + sidx) * kSlotInt4 +
                 ((static_cast<int64_t>(warp - 2) * kChunks + c) * 8) * 32 + lane;
        };
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int64_t n0 = n_half0 + c * 32;
          if (c < my_chunks && n0 < p.cols) {
            __syncwarp();
            uint32_t acc[32];
            tmem_ld_32x32b_x32(t_row + c * 32, acc);
            tmem_wait_ld();
            int4* dst = part_ptr(split, c);
            const int64_t off = dst - reinterpret_cast<int4*>(p.partials);
            if (SQ_GUARD(off >= 0 && off + 7 * 32 < p.partial_int4)) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(dst + j * 32, make_int4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_empty + buf);
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          int32_t* ctr = p.counters + tail * kEpiWarps + (warp - 2);
          if (atomicAdd(ctr, 1) == p.splits - 1) {
            last = 1;
            atomicExch(ctr, 0);  // leave the counter at zero for the next call
          }
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last && rows_live) {
          __threadfence();
#pragma unroll 1
          for (int c = 0; c < my_chunks; ++c) {
            const int64_t n0 = n_half0 + c * 32;
            if (n0 >= p.cols) break;
            const int nvalid = (p.cols - n0) < 32 ? static_cast<int>(p.cols - n0) : 32;
            uint32_t acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0;
            for (int sidx = 0; sidx < p.splits; ++sidx) {
              const int4* src = part_ptr(sidx, c);
              const int64_t off = src - reinterpret_cast<const int4*>(p.partials);
              if (!SQ_GUARD(off >= 0 && off + 7 * 32 < p.partial_int4)) continue;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int4 v = __ldcg(src + j * 32);
                acc[4 * j] += static_cast<uint32_t>(v.x);
                acc[4 * j + 1] += static_cast<uint32_t>(v.y);
                acc[4 * j + 2] += static_cast<uint32_t>(v.z);
                acc[4 * j + 3] += static_cast<uint32_t>(v.w);
              }
            }
            float y[32];
            uint32_t packed[16];
            if constexpr (SWAP) {
              dequant32_tokens<ASYM>(acc, row_scale, row_int, tc, c, y);
              if (p.acc_out != nullptr && r_ok) store_acc32<SWAP>(p, acc, r, n0, nvalid);
              bias_pack32_tokens(y, has_bias, row_bias, packed);
            } else {
              dequant32_cols<ASYM>(p, acc, row_scale, row_int, n0, y);
              if (p.acc_out != nullptr && r_ok) store_acc32<SWAP>(p, acc, r, n0, nvalid);
              bias_pack32_cols(p, y, has_bias, n0, packed);
            }
            store_box<SWAP>(packed, stage_tiles, ebuf, lane, &tmY, n0, box_row0);
          }
        }
      }
    }
    // the output stores of this warp have completed before the CTA exits
    if (lane == 0) bulk_wait_group<0>();
  }

  __syncwarp();
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync();  // no copy, MMA or remote arrive into either CTA is outstanding past here
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
      tmem_dealloc(tmem_base, C::kTmemCols);
  }
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

// 2-D map: inner extent `inner` elements (contiguous), `outer` rows, row pitch `pitch_bytes`,
// box = box_inner x box_rows elements; zero fill out of range.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major operand map: 128 bytes of K x box_rows rows, 128-byte swizzle.
bool make_operand_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                      uint64_t outer, uint64_t pitch_bytes, uint32_t box_rows) {
  return make_map(map, base, dt, inner, outer, pitch_bytes, static_cast<uint32_t>(kBK / elem_bytes), box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

struct Plan {
  bool swap;         // weight rows on the 128-row MMA operand, tokens on the BN columns
  bool pair;         // CTA pairs on 256 x 256 tiles
  int bn;
  int num_full;      // whole-tile units
  int tail_tiles;    // tiles split along K
  int splits;        // parts per tail tile
  int kb_per_split;
};

constexpr int kPlanSms = 148;  // planning is device-independent so workspace sizes are too

constexpr int64_t kSwapMaxM = 64;  // token counts that fit one 64-column tile

// Operand roles: up to 64 tokens (and no outlier product) swap the operands, so the weight
// rows fill the 128-row MMA operand and the tokens one 32- or 64-column tile. Otherwise the tile
// width is the widest of 256/128/64 whose tile count covers the SMs; 256-wide tiles become
// 256 x 256 CTA-pair tiles when those still cover the SM pairs without padding rows (each
// CTA then stages two thirds of the bytes per k-block of a one-CTA 128 x 256 tile).
// Problems with fewer tiles than half the SMs (small M, or a swapped decode shape) split
// every tile along K into S parts whose exact int32 partials meet in the workspace.
// (Splitting only the tiles of a last partial wave was measured slower on the
// 2048 x 11008 x 4096 shape, so whole tiles are kept there.) LLM.int8 (outlier operands)
// tiles are never split.
Plan plan_gemm(int64_t M, int64_t N, int64_t K, bool outliers) {
  const bool swap = !outliers && M <= kSwapMaxM;
  const int64_t rows = swap ? N : M;
  const int64_t cols = swap ? M : N;
  const int64_t m_t = (rows + kBM - 1) / kBM;
  const int64_t kb = (K + kBK - 1) / kBK;
  auto tiles = [&](int bn) { return m_t * ((cols + bn - 1) / bn); };
  constexpr int wide = 256;
  Plan pl{swap, false, 64, 0, 0, 1, static_cast<int>(kb)};
  if (swap) {
    // up to 32 tokens stage a 32-row activation tile (4 KB per k-block instead of 8 KB of
    // mostly zero rows)
    pl.bn = cols <= 32 ? 32 : 64;
  } else if (tiles(wide) >= kPlanSms) {
    pl.bn = wide;
    // CTA pairs when the 256-row tiles still give every pair of SMs a tile and add no
    // padded rows (an even number of 128-row tiles) or few (at least 32 of them): with
    // 65..128 rows, say, the odd CTA of every pair would only compute padding
    const int64_t pair_tiles = ((rows + 2 * kBM - 1) / (2 * kBM)) * ((cols + wide - 1) / wide);
    const bool pair_rows = m_t % 2 == 0 || m_t >= 32;
    if (pair_rows && pair_tiles >= kPlanSms / 2) {
      pl.pair = true;
      pl.num_full = static_cast<int>(pair_tiles);
      return pl;
    }
  } else if (tiles(128) >= kPlanSms) {
    pl.bn = 128;
  }
  const int64_t T = tiles(pl.bn);
  pl.num_full = static_cast<int>(T);
  if (outliers || 2 * T > kPlanSms || kb < 4) return pl;
  const int64_t S = std::min<int64_t>({kPlanSms / T, kb / 2, 16});
  if (S < 2) return pl;
  const int64_t per = (kb + S - 1) / S;
  pl.splits = static_cast<int>((kb + per - 1) / per);
  pl.kb_per_split = static_cast<int>(per);
  pl.tail_tiles = static_cast<int>(T);
  pl.num_full = 0;
  return pl;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

template <int BN, bool OUTLIERS, int ACC_BUFS, bool SWAP, bool ASYM = false, bool PAIR = false>
cudaError_t run(const GemmArgs& a, const Plan& pl, cudaStream_t stream, const char** why) {
  using C = Cfg<BN, OUTLIERS, ACC_BUFS, PAIR>;
  auto kernel = w8a8_gemm_kernel<BN, OUTLIERS, ACC_BUFS, SWAP, ASYM, PAIR>;
  CUtensorMap tmA{}, tmB{}, tmXo{}, tmWo{}, tmY{};
  const uint64_t K = static_cast<uint64_t>(a.K);
  // A: the 128-row operand (Xq, or Wq when swapped); B: the BN-row operand
  const int8_t* a_ptr = SWAP ? a.Wq : a.Xq;
  const int8_t* b_ptr = SWAP ? a.Xq : a.Wq;
  const int64_t rows = SWAP ? a.N : a.M;
  const int64_t cols = SWAP ? a.M : a.N;
  if (!make_operand_map(&tmA, a_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, rows, K, kBM) ||
      !make_operand_map(&tmB, b_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, cols, K, PAIR ? BN / 2 : BN)) {
    *why = "cuTensorMapEncodeTiled failed for the int8 operands";
    return cudaErrorInvalidValue;
  }
  // 32 x 32 bf16 boxes (64-byte rows); row-major staging is swizzled (see store_box), the
  // transposed staging of swapped operands is written conflict-free as it is
  const CUtensorMapSwizzle y_swizzle = SWAP ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map(&tmY, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M),
                static_cast<uint64_t>(a.N) * 2, 32, 32, y_swizzle)) {
    *why = "cuTensorMapEncodeTiled failed for the output";
    return cudaErrorInvalidValue;
  }
  if (OUTLIERS) {
    const uint64_t ldo = static_cast<uint64_t>(a.ld_o);
    if (!make_operand_map(&tmXo, a.Xo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ldo, a.M, ldo * 2, kBM) ||
        !make_operand_map(&tmWo, a.Wo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ldo, a.N, ldo * 2, PAIR ? BN / 2 : BN)) {
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
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    attr_done.fetch_or(bit);
  }
  Params p{};
  p.x_scale = a.x_scale;
  p.x_per_token = a.x_per_token ? 1 : 0;
  p.x_zero = a.x_zero;
  p.w_rowsum = a.w_rowsum;
  p.w_scale = a.w_scale;
  p.w_per_channel = a.w_per_channel ? 1 : 0;
  p.bias = a.bias;
  p.acc_out = a.acc_out;
  p.M = a.M;
  p.N = a.N;
  p.rows = rows;
  p.cols = cols;
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  p.num_m_tiles = static_cast<int>((rows + kTileM - 1) / kTileM);
  p.num_n_tiles = static_cast<int>((cols + BN - 1) / BN);
  p.num_kb = static_cast<int>((a.K + kBK - 1) / kBK);
  p.num_full = pl.num_full;
  p.splits = pl.splits;
  p.kb_per_split = pl.kb_per_split;
  p.num_units = pl.num_full + pl.tail_tiles * pl.splits;
  p.partials = nullptr;
  p.counters = nullptr;
  p.partial_int4 = 0;
  if (pl.tail_tiles > 0) {
    p.partials = static_cast<int32_t*>(a.ws);
    p.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a.ws) +
                                            up256(static_cast<size_t>(pl.tail_tiles) * pl.splits * split_slot_bytes(BN)));
    p.partial_int4 = static_cast<int64_t>(pl.tail_tiles) * pl.splits * split_slot_bytes(BN) / 16;
  }
  p.o_count = a.o_count;
  p.status = device_status_word();
  p.prefetch_weight = (SWAP || pl.tail_tiles > 0) ? 1 : 0;
  p.wait_limit_ns = a.wait_limit_ns;
  p.fault = a.fault;
  // one persistent CTA per SM (a pair per two SMs)
  const int grid = PAIR ? 2 * std::min(p.num_units, num_sms() / 2) : std::min(p.num_units, num_sms());
  // every GEMM launch overlaps its set-up (barrier init, TMEM allocation, descriptor prefetch)
  // with the previous kernel's tail: measured on the SmoothQuant + LLM.int8 step
  // (2048 x 11008 x 4096), 0.2481-0.2499 ms against 0.2515-0.2526 ms with it on the short
  // (swapped or K-split) launches only
  const bool programmatic = true;
  return launch_kernel_clustered(kernel, dim3(grid), dim3(kThreads), C::kSmemBytes, stream, programmatic,
                                 PAIR ? 2u : 1u, tmA, tmB, tmXo, tmWo, tmY, p);
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, bool outliers) {
  if (gemv_applies(M, K, outliers)) return 0;
  const Plan pl = plan_gemm(M, N, K, outliers);
  if (pl.tail_tiles == 0) return 0;
  return up256(static_cast<size_t>(pl.tail_tiles) * pl.splits * split_slot_bytes(pl.bn)) +
         up256(sizeof(int32_t) * pl.tail_tiles * kEpiWarps);
}

void gemm_plan_numbers(int64_t M, int64_t N, int64_t K, bool outliers, int64_t* out) {
  if (gemv_applies(M, K, outliers)) {
    const int64_t kb = (K + kBK - 1) / kBK;
    const int64_t v[7] = {0, 0, 0, 0, 0, 1, kb};
    for (int i = 0; i < 7; ++i) out[i] = v[i];
    return;
  }
  const Plan pl = plan_gemm(M, N, K, outliers);
  const int64_t v[7] = {pl.pair ? 2 : 1, pl.swap ? 1 : 0, pl.bn, pl.num_full, pl.tail_tiles, pl.splits,
                        pl.kb_per_split};
  for (int i = 0; i < 7; ++i) out[i] = v[i];
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream, const char** why) {
  const bool outliers = a.Xo != nullptr;
  // up to 4 tokens: a weight stream on the CUDA cores (no tensor-core set-up, no K split)
  if (gemv_applies(a.M, a.K, outliers) && a.fault == 0) return launch_gemv(a, stream);
  const Plan pl = plan_gemm(a.M, a.N, a.K, outliers);
  if (outliers) {
    if (pl.pair) return run<256, true, 2, false, false, true>(a, pl, stream, why);
    if (pl.bn == 256) return run<256, true, 2, false>(a, pl, stream, why);
    if (pl.bn == 128) return run<128, true, 2, false>(a, pl, stream, why);
    return run<64, true, 2, false>(a, pl, stream, why);
  }
  if (pl.pair) {
    if (a.x_zero != nullptr) return run<256, false, 2, false, true, true>(a, pl, stream, why);
    return run<256, false, 2, false, false, true>(a, pl, stream, why);
  }
  if (a.x_zero != nullptr) {
    if (pl.swap)
      return pl.bn == 32 ? run<32, false, 2, true, true>(a, pl, stream, why)
                         : run<64, false, 2, true, true>(a, pl, stream, why);
    if (pl.bn == 256) return run<256, false, 2, false, true>(a, pl, stream, why);
    if (pl.bn == 128) return run<128, false, 2, false, true>(a, pl, stream, why);
    return run<64, false, 2, false, true>(a, pl, stream, why);
  }
  if (pl.swap)
    return pl.bn == 32 ? run<32, false, 2, true>(a, pl, stream, why) : run<64, false, 2, true>(a, pl, stream, why);
  if (pl.bn == 256) return run<256, false, 2, false>(a, pl, stream, why);
  if (pl.bn == 128) return run<128, false, 2, false>(a, pl, stream, why);
  return run<64, false, 2, false>(a, pl, stream, why);
}

}  // namespace sq
