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
// (correctly rounded) and e = x * inv (the exact product):
//   |e - x/s| <= |x/s| 2^-24 < 2^-17,  since |x/s| <= 127 (1 + 2^-23);
//   |fl(x/s) - x/s| <= 2^-18 (half an ulp below 128).
// So when e lies farther than 2^-16 from every half-integer k + 1/2, the
// values e, x/s and fl(x/s) all sit strictly between the same two
// half-integers and round to the same integer, rint(e).  Three fused or exact
// steps give rint(e) and the distance to it (M = 1.5 * 2^23):
//   t = fl(e + M)       one rounding to an integer: M + rint_even(e) for
//                       |e| < 2^22; the low byte of t's bits is that integer
//                       as a two's-complement byte (t - 2^23 = 2^22 + q);
//   r = t - M           exact;
//   d = fl(e - r)       the product stays exact inside the fused multiply-add,
//                       so d is e - r rounded once (|error| <= 2^-25).
// An element with |d| < 1/2 - 2^-12 is at least 2^-12 - 2^-25 > 2^-16 away
// from every half-integer and takes the code of t.  The others (about one in
// 2000, and NaN) get the IEEE division.  A regular element satisfies |x| <=
// amax, hence |e| <= 127 (1 + 2^-23) and |rint(e)| <= 127: no clamp is needed
// on the fast path.  A zero scale has inv = 0, so t = M and the code is 0.
__device__ __forceinline__ float scale_reciprocal(float s) { return s == 0.0f ? 0.0f : __frcp_rn(s); }

__device__ __forceinline__ int clamp127(int q) { return q > 127 ? 127 : (q < -127 ? -127 : q); }

// Bytes whose bit is set in the low four bits of `bits` -> 0xFF, others 0.
__device__ __forceinline__ uint32_t byte_mask4(uint32_t bits) {
  return ((((bits & 0xFu) * 0x00204081u) & 0x01010101u) * 0xFFu);
}

// Eight halves packed in a uint4 -> their eight codes packed in a uint2.
// Lanes whose bit is set in `skip` get code 0.  The eight codes are formed
// independently (no branch per element); the rare near-tie elements are
// redone with the division afterwards.
__device__ __forceinline__ uint2 quant8(const uint4 v, float s, float inv, uint32_t skip) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float x[8];
  uint32_t tb[8];
  bool near = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = __fmaf_rn(x[i], inv, kMagic);
    const float d = __fmaf_rn(x[i], inv, -__fsub_rn(t, kMagic));
    near |= !(fabsf(d) < 0.5f - 0x1p-12f);
    tb[i] = __float_as_uint(t);
  }
  uint32_t lo = __byte_perm(__byte_perm(tb[0], tb[1], 0x0040), __byte_perm(tb[2], tb[3], 0x0040), 0x5410);
  uint32_t hi = __byte_perm(__byte_perm(tb[4], tb[5], 0x0040), __byte_perm(tb[6], tb[7], 0x0040), 0x5410);
  if (near) {
    // redo the near-tie lanes with the division
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float t = __uint_as_float(tb[i]);
      const float d = __fmaf_rn(x[i], inv, -__fsub_rn(t, kMagic));
      if (!((skip >> i) & 1u) && !(fabsf(d) < 0.5f - 0x1p-12f)) {
        const uint32_t q = static_cast<uint32_t>(quant_code(x[i], s)) & 0xFFu;
        const int sh = (i & 3) * 8;
        if (i < 4)
          lo = (lo & ~(0xFFu << sh)) | (q << sh);
        else
          hi = (hi & ~(0xFFu << sh)) | (q << sh);
      }
    }
  }
  if (skip) {
    lo &= ~byte_mask4(skip);
    hi &= ~byte_mask4(skip >> 4);
  }
  return make_uint2(lo, hi);
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

// Eight halves -> eight E4M3 codes (lanes set in `skip` get 0), without a
// division in the common case.  With inv = fl(1/s) and a = fl(x * inv):
//   |a - x/s| <= 2^-23 |x/s| (two roundings) and |fl(x/s) - x/s| <= 2^-24 |x/s|,
// so fl(x/s) lies strictly between fl(a (1 - 2^-20)) and fl(a (1 + 2^-20))
// (each still at least 2^-21 |a| away from a).  The conversion (round to
// nearest even, saturating) is monotonic, so when it gives one code for both
// ends it gives that code for fl(x/s) too; otherwise (a value next to a
// rounding point of E4M3) the lane takes the IEEE division.  Pairs of lanes
// go through the two-float conversion.
__device__ __forceinline__ uint2 quant8_e4m3(const uint4 v, float s, float inv, uint32_t skip) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  constexpr float kDown = 1.0f - 0x1p-20f, kUp = 1.0f + 0x1p-20f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t pair[4];
  uint32_t differ = 0;  // bit i: lane i's two ends convert differently
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    const float a0 = __fmul_rn(f.x, inv), a1 = __fmul_rn(f.y, inv);
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(a0, kDown), __fmul_rn(a1, kDown)),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(a0, kUp), __fmul_rn(a1, kUp)),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t d = lo ^ hi;
    differ |= ((d & 0xFFu) ? 1u : 0u) << (2 * j) | ((d & 0xFF00u) ? 1u : 0u) << (2 * j + 1);
    pair[j] = lo;
  }
  uint32_t lo32 = (pair[0] & 0xFFFFu) | (pair[1] << 16);
  uint32_t hi32 = (pair[2] & 0xFFFFu) | (pair[3] << 16);
  differ &= ~skip;
  if (differ) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (!((differ >> i) & 1u)) continue;
      const uint32_t c = e4m3_code(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), s);
      const int sh = (i & 3) * 8;
      if (i < 4)
        lo32 = (lo32 & ~(0xFFu << sh)) | (c << sh);
      else
        hi32 = (hi32 & ~(0xFFu << sh)) | (c << sh);
    }
  }
  if (skip) {
    lo32 &= ~byte_mask4(skip);
    hi32 &= ~byte_mask4(skip >> 4);
  }
  return make_uint2(lo32, hi32);
}

// Codes of either format (inv = fl(1/s), 0 for s == 0).
template <bool FP8>
__device__ __forceinline__ uint2 quant8_codes(const uint4 v, float s, float inv, uint32_t skip) {
  if constexpr (FP8)
    return quant8_e4m3(v, s, inv, skip);
  else
    return quant8(v, s, inv, skip);
}

// max |x| over the lanes of eight halves whose bit is clear in `skip`, merged
// into m.  The maximum of fp16 magnitudes is one of them, so it is taken in
// half2 (NaN lanes are ignored, as by fmaxf) and widened once.
__device__ __forceinline__ float absmax8(const uint4 v, uint32_t skip, float m) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (skip) {
    // a skipped lane becomes +0 (bits 0x0000)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b = (skip >> (2 * j)) & 3u;
      w[j] &= ((b & 1u) ? 0xFFFF0000u : 0xFFFFFFFFu) & ((b & 2u) ? 0x0000FFFFu : 0xFFFFFFFFu);
    }
  }
  const __half2 h0 = __hmax2(__habs2(*reinterpret_cast<const __half2*>(&w[0])),
                             __habs2(*reinterpret_cast<const __half2*>(&w[1])));
  const __half2 h1 = __hmax2(__habs2(*reinterpret_cast<const __half2*>(&w[2])),
                             __habs2(*reinterpret_cast<const __half2*>(&w[3])));
  const float2 f = __half22float2(__hmax2(h0, h1));
  return fmaxf(m, fmaxf(f.x, f.y));
}

// The smallest fp16 value >= tau (+inf above the largest finite half): for an
// fp16 x, |x| >= tau (binary32) exactly when |x| >= this value (fp16).
__device__ __forceinline__ __half2 tau_half2(float tau) {
  const __half h = __float2half_ru(tau);
  return __halves2half2(h, h);
}

// |x| >= tau for the eight halves, as four words of two 16-bit lane masks
// (0xFFFF where true; NaN never is).  OR-ing these over rows and turning the
// result into bits once (mask_bits) is the cheap way to detect over many rows.
struct Mask8 {
  uint32_t m[4];
};

__device__ __forceinline__ void outlier_mask8_or(const uint4 v, __half2 tau2, Mask8& acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) acc.m[j] |= __hge2_mask(__habs2(*reinterpret_cast<const __half2*>(&w[j])), tau2);
}

// Bit i set iff lane i of the masks is set.
__device__ __forceinline__ uint32_t mask_bits(const Mask8& a) {
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) r |= ((a.m[j] & 1u) << (2 * j)) | (((a.m[j] >> 16) & 1u) << (2 * j + 1));
  return r;
}

// Bit i set iff |lane i| >= tau.
__device__ __forceinline__ uint32_t outlier_mask8(const uint4 v, __half2 tau2) {
  Mask8 a = {{0u, 0u, 0u, 0u}};
  outlier_mask8_or(v, tau2, a);
  return mask_bits(a);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace llmint8
