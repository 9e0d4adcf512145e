// quant.cuh -- the integer-producing steps of the method, shared by every
// kernel that quantises: the outlier test, the absmax scale and the int8 code.
//
// 'LLM quantization, part 2' (hncyxsy.com) §2.1: an activation magnitude at or
// above the threshold marks its feature dim as an outlier.  '三、模型量化'
// (lowentro.cn) Q2 and '量化压缩实战' (tqpw.cn) §2.1: symmetric absmax int8,
// s = max|r| / 127, q = round(r / s), clipped.  Taken in binary32: |x| >= tau,
// s = amax / 127 (IEEE division), q = rint_even(fl(x / s)) clamped to
// [-127, 127], and q = 0 when s == 0.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "sm100.cuh"

namespace llmint8 {

// Symmetric absmax code of x under scale s.
__device__ __forceinline__ int8_t quant_code(float x, float s) {
  if (s == 0.0f) return 0;
  const float r = __fdiv_rn(x, s);
  int q = __float2int_rn(r);
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return static_cast<int8_t>(q);
}

// The same code without a division in the common case.  With inv = fl(1/s)
// (correctly rounded) and a = fl(x * inv):
//   |a - x/s| <= |x/s| (2^-24 + 2^-24 + 2^-48) <= 2^-16,  since |x/s| <= 127 (1 + 2^-24);
//   |fl(x/s) - x/s| <= 2^-18 (half an ulp below 128).
// So when a lies farther than 2^-12 from every half-integer k + 1/2, i.e. when
// |a - rint(a)| < 1/2 - 2^-12, the values a, x/s and fl(x/s) all sit strictly
// between the same two half-integers and round to the same integer, rint(a).
// Only inside that band (about one element in 2000) is fl(x/s) formed by the
// IEEE division.  A zero scale has inv = 0, so a = 0 and the code is 0.
__device__ __forceinline__ float scale_reciprocal(float s) { return s == 0.0f ? 0.0f : __frcp_rn(s); }

__device__ __forceinline__ int clamp127(int q) { return q > 127 ? 127 : (q < -127 ? -127 : q); }

// Eight halves packed in a uint4 -> their eight codes packed in a uint2.
// Lanes whose bit is set in `skip` get code 0.  The eight codes are formed
// independently (no branch per element); the rare near-tie elements are
// redone with the division afterwards.
__device__ __forceinline__ uint2 quant8(const uint4 v, float s, float inv, uint32_t skip) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float x[8];
  int q[8];
  uint32_t near = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[i] = half_bits_to_float(w[i >> 1] >> ((i & 1) * 16));
    const float a = x[i] * inv;
    const float r = rintf(a);
    near |= (fabsf(a - r) >= 0.5f - 0x1p-12f ? 1u : 0u) << i;
    q[i] = clamp127(__float2int_rn(r));
  }
  near &= ~skip;
  if (near) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((near >> i) & 1u) q[i] = quant_code(x[i], s);
  }
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int qi = ((skip >> i) & 1u) ? 0 : q[i];
    out[i >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << ((i & 3) * 8);
  }
  return make_uint2(out[0], out[1]);
}

// ---------------------------------------------------------------------------
// FP8 E4M3 codes ('量化压缩实战' (tqpw.cn) §3.6: 1 sign, 4 exponent, 3 mantissa
// bits, largest finite 448): the same absmax recipe with 448 in place of 127,
// s = amax / 448, code = e4m3(fl(x / s)), rounded to nearest even and
// saturated to +-448 by the hardware conversion; s == 0 gives code 0.
// ---------------------------------------------------------------------------
template <bool FP8>
__host__ __device__ constexpr float code_max() {
  return FP8 ? 448.0f : 127.0f;
}

__device__ __forceinline__ uint32_t e4m3_code(float v, float s) {
  if (s == 0.0f) return 0u;
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3));
}

// Eight halves -> eight E4M3 codes (lanes set in `skip` get 0).
__device__ __forceinline__ uint2 quant8_e4m3(const uint4 v, float s, uint32_t skip) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = ((skip >> i) & 1u) ? 0u : e4m3_code(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), s);
    out[i >> 2] |= c << ((i & 3) * 8);
  }
  return make_uint2(out[0], out[1]);
}

// Codes of either format; `inv` (= fl(1/s)) is used by the int8 codes only.
template <bool FP8>
__device__ __forceinline__ uint2 quant8_codes(const uint4 v, float s, float inv, uint32_t skip) {
  if constexpr (FP8)
    return quant8_e4m3(v, s, skip);
  else
    return quant8(v, s, inv, skip);
}

// max |x| over the lanes of eight halves whose bit is clear in `skip`.
__device__ __forceinline__ float absmax8(const uint4 v, uint32_t skip, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if ((skip >> i) & 1u) continue;
    m = fmaxf(m, fabsf(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16))));
  }
  return m;
}

// Bit i set iff |lane i| >= tau.
__device__ __forceinline__ uint32_t outlier_mask8(const uint4 v, float tau) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    m |= (fabsf(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16))) >= tau ? 1u : 0u) << i;
  return m;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace llmint8
