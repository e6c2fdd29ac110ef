// Device helpers shared by the row kernels (quantization of rows, fused normalisation):
// 16-element bf16 loads, int8 packing with round-half-to-even, and reductions over the
// TPR threads that own one row.
#pragma once
#include <cstdint>

namespace sq {
namespace rows {

constexpr int kCta = 256;  // minimum CTA size of the row kernels

// The low bytes of a, b, c, d as one little-endian word (three byte permutes).
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t ab = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x0040u);
  const uint32_t cd = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x0040u);
  return __byte_perm(ab, cd, 0x5410u);
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: two IEEE round-to-nearest operations per
// instruction, each lane exactly the scalar result). Use them only where no packed multiply
// feeds a packed add: such a pair was observed to execute as one fused multiply-add.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// clamp(rne(x * r), -128, 127) of two values, each returned in the low byte (the upper bytes
// are not the code). The product is clamped first (the same result: every value in [127, 128)
// rounds to 127 or 128 and clamps to 127, likewise at -128), then rounded half to even by
// adding 1.5 * 2^23, whose fp32 sum keeps the integer in its low mantissa bits: no float->int
// conversion unit. With CLAMP the products and the rounding add are packed, and the clamp
// between them keeps the two from fusing. Without CLAMP the caller guarantees
// |x * r| < 127.5: a row scaled by r = 127/a with a its own absmax (|x| <= a, r finite) stays
// within 127 * (1 + 2^-24)^2, which rounds to a code in [-127, 127], so the clamp could not
// change a code; the products are then scalar multiplies with an explicit rounding mode, which
// are never contracted into the add (a fused multiply-add would round only once).
template <bool CLAMP>
__device__ __forceinline__ void q8x2(float x0, float x1, uint64_t r2, int& q0, int& q1) {
  float t0, t1;
  if constexpr (CLAMP) {
    f2_unpack(f2_mul(f2_pack(x0, x1), r2), t0, t1);
    t0 = fminf(fmaxf(t0, -128.0f), 127.0f);
    t1 = fminf(fmaxf(t1, -128.0f), 127.0f);
  } else {
    float r, r_hi;
    f2_unpack(r2, r, r_hi);
    t0 = __fmul_rn(x0, r);
    t1 = __fmul_rn(x1, r_hi);
  }
  f2_unpack(f2_add(f2_pack(t0, t1), f2_pack(12582912.0f, 12582912.0f)), t0, t1);
  q0 = __float_as_int(t0);
  q1 = __float_as_int(t1);
}

template <bool CLAMP = true>
__device__ __forceinline__ void store_q16(int8_t* dst, const float (&v)[16], float r) {
  const uint64_t r2 = f2_pack(r, r);
  int q[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) q8x2<CLAMP>(v[i], v[i + 1], r2, q[i], q[i + 1]);
  uint4 o;
  o.x = pack4(q[0], q[1], q[2], q[3]);
  o.y = pack4(q[4], q[5], q[6], q[7]);
  o.z = pack4(q[8], q[9], q[10], q[11]);
  o.w = pack4(q[12], q[13], q[14], q[15]);
  *reinterpret_cast<uint4*>(dst) = o;
}

// Codes of 16 values of a row quantized with its own absmax a (r = 127/a): the clamp is
// needed only when r overflowed to infinity (a < 127 / FLT_MAX), a branch uniform over the row.
__device__ __forceinline__ void store_q16_own_max(int8_t* dst, const float (&v)[16], float r) {
  if (r <= 3.402823466e38f)
    store_q16<false>(dst, v, r);
  else
    store_q16<true>(dst, v, r);
}

// Codes of 16 values with a zero point: clamp(rne(v * r) + z, -128, 127).
__device__ __forceinline__ int q8z(float x, float r, int z) {
  const int q = __float2int_rn(__fmul_rn(x, r)) + z;
  return min(127, max(-128, q));
}

__device__ __forceinline__ void store_q16z(int8_t* dst, const float (&v)[16], float r, int z) {
  uint4 o;
  o.x = pack4(q8z(v[0], r, z), q8z(v[1], r, z), q8z(v[2], r, z), q8z(v[3], r, z));
  o.y = pack4(q8z(v[4], r, z), q8z(v[5], r, z), q8z(v[6], r, z), q8z(v[7], r, z));
  o.z = pack4(q8z(v[8], r, z), q8z(v[9], r, z), q8z(v[10], r, z), q8z(v[11], r, z));
  o.w = pack4(q8z(v[12], r, z), q8z(v[13], r, z), q8z(v[14], r, z), q8z(v[15], r, z));
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

__device__ __forceinline__ void raw16(const uint16_t* p, uint4 (&r)[2]) {
  r[0] = __ldg(reinterpret_cast<const uint4*>(p));
  r[1] = __ldg(reinterpret_cast<const uint4*>(p + 8));
}

__device__ __forceinline__ void widen16(const uint4 (&r)[2], float (&v)[16]) {
  const uint32_t w[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Two fp64 sums over the TPR threads of one row group at once (one shared-memory round).
template <int TPR>
__device__ __forceinline__ void group_sum2(double& a, double& b, double2* red /* [CTA threads / 32] */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a = __dadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = __dadd_rn(b, __shfl_xor_sync(0xffffffffu, b, o));
  }
  if constexpr (TPR > 32) {
    constexpr int kWarpsPerGroup = TPR / 32;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g0 = (warp / kWarpsPerGroup) * kWarpsPerGroup;
    if (lane == 0) red[warp] = make_double2(a, b);
    __syncthreads();
    double2 t = red[g0];
#pragma unroll
    for (int w = 1; w < kWarpsPerGroup; ++w) {
      t.x = __dadd_rn(t.x, red[g0 + w].x);
      t.y = __dadd_rn(t.y, red[g0 + w].y);
    }
    __syncthreads();
    a = t.x;
    b = t.y;
  }
}

}  // namespace rows
}  // namespace sq
