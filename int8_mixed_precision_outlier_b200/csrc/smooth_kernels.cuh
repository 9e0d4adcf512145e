// smooth_kernels.cuh -- SmoothQuant W8A8 on the same int8 tensor-core path.
//
// 'LLM quantization, part 2' (hncyxsy.com) §5 and '三、模型量化' (lowentro.cn)
// Q9-Q10: Y = X W^T = (X diag(s)^-1)(W diag(s))^T holds exactly, so the
// activation channels that carry outliers can be divided by a per-channel
// factor s_j and the same weight columns multiplied by it; both sides are then
// quantised to int8 (per row of X, per output channel of W) and multiplied on
// the int8 tensor cores with no fp16 part.  The factor comes from the channel
// maxima of a calibration batch and of the weight, s_j = max|X_j|^a /
// max|W_j|^(1-a), a = migration strength (about 0.5); a channel that is zero
// on either side keeps s_j = 1.
//
// Kernels here: the channel maxima (HBM-bound column reduction), the factors
// (elementwise), the smoothed weight quantisation (offline, one CTA per output
// channel) and the smoothed activation quantisation (one CTA per row).  The
// product itself is the GEMV / GEMM of the LLM.int8() path with no outlier
// columns.  Decisions that produce integers are binary32 as stated:
// fl(x / s_j), fl(w * s_j), scale = amax / 127, code = rint_even(fl(v / scale)).
#pragma once
#include <cuda_fp16.h>
#include "quant.cuh"
#include "sm100.cuh"

namespace llmint8 {

constexpr int kColThreads = 256;
constexpr int kColCols = 512;  // columns per CTA (64 threads x 8)

// amax[k] = max(amax[k], max over rows r0.. of |A[r,k]|) for this CTA's 512
// columns and rows [blockIdx.y * rows_per_chunk, ...).  Thread (c = tid % 64,
// r = tid / 64) reads 16 bytes of every 4th row.  Non-negative binary32 values
// order like their bit patterns, so the merge is an integer atomicMax.
__global__ void __launch_bounds__(kColThreads) column_absmax_kernel(const uint16_t* __restrict__ A, int rows,
                                                                    int K, int rows_per_chunk,
                                                                    float* __restrict__ amax) {
  __shared__ float part[4][kColCols];
  const int c = threadIdx.x & 63, r = threadIdx.x >> 6;
  const int col0 = blockIdx.x * kColCols + c * 8;
  const int t0 = blockIdx.y * rows_per_chunk;
  const int t1 = min(rows, t0 + rows_per_chunk);
  pdl_launch_dependents();
  pdl_wait();
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  if (col0 < K) {
    const uint16_t* base = A + col0;
    for (int t = t0 + r; t < t1; t += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * K));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16))));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[r][c * 8 + i] = m[i];
  __syncthreads();
  for (int j = threadIdx.x; j < kColCols; j += kColThreads) {
    const int k = blockIdx.x * kColCols + j;
    if (k < K) {
      const float v = fmaxf(fmaxf(part[0][j], part[1][j]), fmaxf(part[2][j], part[3][j]));
      atomicMax(reinterpret_cast<unsigned int*>(amax) + k, __float_as_uint(v));
    }
  }
}

// p^a: exact or correctly rounded for a in {0, 1/2, 1}, powf otherwise.
__device__ __forceinline__ float smooth_pow(float p, float a) {
  if (a == 0.0f) return 1.0f;
  if (a == 1.0f) return p;
  if (a == 0.5f) return __fsqrt_rn(p);
  return powf(p, a);
}

// s[k] = ax[k]^alpha / aw[k]^(1 - alpha); 1 where either maximum is zero.
__global__ void smooth_factors_kernel(const float* __restrict__ ax, const float* __restrict__ aw, int K,
                                      float alpha, float* __restrict__ s) {
  pdl_launch_dependents();
  pdl_wait();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float x = ax[k], w = aw[k];
  const float beta = __fsub_rn(1.0f, alpha);
  s[k] = (x == 0.0f || w == 0.0f) ? 1.0f : __fdiv_rn(smooth_pow(x, alpha), smooth_pow(w, beta));
}

// Symmetric int8 code of a binary32 value v under scale s with inv = fl(1/s):
// rint(v * inv) unless that product lies within 2^-12 of a half-integer, where
// the IEEE quotient decides (the argument of quant8 in quant.cuh holds for any
// binary32 v with |v / s| <= 127 (1 + 2^-24)).
__device__ __forceinline__ int quant_code_value(float v, float s, float inv) {
  const float a = v * inv;
  const float r = rintf(a);
  if (fabsf(a - r) >= 0.5f - 0x1p-12f) return quant_code(v, s);
  return clamp127(__float2int_rn(r));
}

// Smoothed weight codes, one CTA per output channel n:
//   w~ = fl(W[n,k] * s[k]); sw[n] = max |w~| / 127; Wq[n,k] = code(w~).
__global__ void __launch_bounds__(kPrepThreads) smooth_quantize_weight_kernel(
    const uint16_t* __restrict__ W, int K, const float* __restrict__ s, int8_t* __restrict__ Wq,
    float* __restrict__ Wscale) {
  __shared__ float red[32];
  const int64_t n = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(W + n * K);
  const float4* s4 = reinterpret_cast<const float4*>(s);
  const int nchunk = K >> 3;
  float m = 0.0f;
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    const uint4 v = __ldg(row + c);
    const float4 sa = __ldg(s4 + 2 * c), sb = __ldg(s4 + 2 * c + 1);
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(__fmul_rn(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), sv[i])));
  }
  const float amax = block_max(m, red);
  const float sc = __fdiv_rn(amax, 127.0f);
  const float inv = scale_reciprocal(sc);
  if (threadIdx.x == 0) Wscale[n] = sc;
  uint2* out = reinterpret_cast<uint2*>(Wq + n * K);
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    const uint4 v = __ldg(row + c);
    const float4 sa = __ldg(s4 + 2 * c), sb = __ldg(s4 + 2 * c + 1);
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x = __fmul_rn(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), sv[i]);
      const int q = sc == 0.0f ? 0 : quant_code_value(x, sc, inv);
      o[i >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << ((i & 3) * 8);
    }
    out[c] = make_uint2(o[0], o[1]);
  }
}

// Smoothed activation codes, one CTA of 128 threads per row t:
//   x~ = fl(X[t,k] / s[k]); sx[t] = max |x~| / 127; Xq[t,k] = code(x~).
// The row is read twice (the second time from L1, where this CTA just put it).
constexpr int kSmoothThreads = 128;

__global__ void __launch_bounds__(kSmoothThreads) smooth_quantize_activations_kernel(
    const uint16_t* __restrict__ X, int K, const float* __restrict__ s, int8_t* __restrict__ Xq,
    float* __restrict__ sx) {
  __shared__ float red[4];
  pdl_launch_dependents();
  pdl_wait();  // X, and the workspace the previous call may still be reading
  const int64_t t = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(X + t * K);
  const float4* s4 = reinterpret_cast<const float4*>(s);
  const int nchunk = K >> 3;
  float m = 0.0f;
  for (int c = threadIdx.x; c < nchunk; c += kSmoothThreads) {
    const uint4 v = __ldg(row + c);
    const float4 sa = __ldg(s4 + 2 * c), sb = __ldg(s4 + 2 * c + 1);
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(__fdiv_rn(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), sv[i])));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  const float amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float sc = __fdiv_rn(amax, 127.0f);
  const float inv = scale_reciprocal(sc);
  if (threadIdx.x == 0) sx[t] = sc;
  uint2* out = reinterpret_cast<uint2*>(Xq + t * K);
  for (int c = threadIdx.x; c < nchunk; c += kSmoothThreads) {
    const uint4 v = __ldg(row + c);
    const float4 sa = __ldg(s4 + 2 * c), sb = __ldg(s4 + 2 * c + 1);
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x = __fdiv_rn(half_bits_to_float(w[i >> 1] >> ((i & 1) * 16)), sv[i]);
      const int q = sc == 0.0f ? 0 : quant_code_value(x, sc, inv);
      o[i >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << ((i & 3) * 8);
    }
    out[c] = make_uint2(o[0], o[1]);
  }
}

}  // namespace llmint8
