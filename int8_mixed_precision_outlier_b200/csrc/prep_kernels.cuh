// prep_kernels.cuh -- the HBM-bound stages of the LLM.int8() matmul:
//   a0 weight quantisation (offline), a1 outlier detection, a4 compaction and
//   gathers, a2+a3 per-row scale and int8 codes of X.
//
// Method: 'LLM quantization, part 2' (hncyxsy.com) §2.1 (vector-wise scales,
// threshold 6.0 on activation magnitude, outlier columns leave the int8
// product); '三、模型量化' (lowentro.cn) Q2 (q = round(r/s), s = max|r|/127).
//
// Integer-producing decisions are taken in binary32 exactly as stated:
// |x| >= tau, s = amax / 127 (IEEE division), q = rint_even(x / s) (IEEE
// division, then round half to even), clamp to [-127, 127], s == 0 -> 0.
#pragma once
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace llmint8 {

constexpr int kPrepThreads = 256;

// Symmetric absmax code of x under scale s.
__device__ __forceinline__ int8_t quant_code(float x, float s) {
  if (s == 0.0f) return 0;
  const float r = __fdiv_rn(x, s);
  int q = __float2int_rn(r);
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return static_cast<int8_t>(q);
}

// Eight halves packed in a uint4 -> their eight codes packed in a uint2.
// Lanes whose bit is set in `skip` get code 0.
__device__ __forceinline__ uint2 quant8(const uint4 v, float s, uint32_t skip) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float x = half_bits_to_float(w[i >> 1] >> ((i & 1) * 16));
    const int8_t q = ((skip >> i) & 1u) ? int8_t(0) : quant_code(x, s);
    out[i >> 2] |= (static_cast<uint32_t>(static_cast<uint8_t>(q))) << ((i & 3) * 8);
  }
  return make_uint2(out[0], out[1]);
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

// Block-wide max; `red` is shared scratch of >= 32 floats.
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < nwarps ? red[lane] : 0.0f;
    w = warp_max(w);
    if (lane == 0) red[0] = w;
  }
  __syncthreads();
  return red[0];
}

// Block-wide exclusive prefix sum of one int per thread; returns the prefix
// and writes the total to *total.  `scratch` is shared, >= 33 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    scratch[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  *total = scratch[32];
  return scratch[warp] + inc - v;
}

// ---------------------------------------------------------------------------
// a0: per-output-channel weight quantisation, one CTA per row of W.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPrepThreads) quantize_weight_kernel(
    const uint16_t* __restrict__ W, int K, int8_t* __restrict__ Wq, float* __restrict__ Wscale) {
  __shared__ float red[32];
  const int64_t n = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(W + n * K);
  const int nchunk = K >> 3;
  float m = 0.0f;
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) m = absmax8(__ldg(row + c), 0u, m);
  const float amax = block_max(m, red);
  const float s = __fdiv_rn(amax, 127.0f);
  if (threadIdx.x == 0) Wscale[n] = s;
  uint2* out = reinterpret_cast<uint2*>(Wq + n * K);
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) out[c] = quant8(__ldg(row + c), s, 0u);
}

// ---------------------------------------------------------------------------
// a1 (prefill): partial outlier flags.  CTA (strip, chunk) covers 512 columns
// x `rows_per_chunk` rows; thread (c = tid % 64, r = tid / 64) reads 16 B of
// every 4th row.  Result: part[chunk][word] bitmasks, bit k%32 of word k/32.
// ---------------------------------------------------------------------------
constexpr int kDetectCols = 512;

__global__ void __launch_bounds__(kPrepThreads) detect_partial_kernel(
    const uint16_t* __restrict__ X, int T, int K, float tau, int rows_per_chunk,
    uint32_t* __restrict__ part, int Kw) {
  __shared__ uint32_t words[4][kDetectCols / 32];
  const int c = threadIdx.x & 63, r = threadIdx.x >> 6;
  if (threadIdx.x < 4 * (kDetectCols / 32)) (&words[0][0])[threadIdx.x] = 0u;
  __syncthreads();
  pdl_launch_dependents();
  const int col0 = blockIdx.x * kDetectCols + c * 8;
  const int t0 = blockIdx.y * rows_per_chunk;
  const int t1 = min(T, t0 + rows_per_chunk);
  uint32_t mask = 0;
  if (col0 < K) {
    const uint16_t* base = X + col0;
    int t = t0 + r;
    for (; t + 12 < t1; t += 16) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)t * K));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(t + 4) * K));
      const uint4 v2 = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(t + 8) * K));
      const uint4 v3 = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(t + 12) * K));
      mask |= outlier_mask8(v0, tau) | outlier_mask8(v1, tau) | outlier_mask8(v2, tau) |
              outlier_mask8(v3, tau);
    }
    for (; t < t1; t += 4)
      mask |= outlier_mask8(__ldg(reinterpret_cast<const uint4*>(base + (int64_t)t * K)), tau);
  }
  if (mask) atomicOr(&words[r][c >> 2], mask << ((c & 3) * 8));
  __syncthreads();
  if (threadIdx.x < kDetectCols / 32) {
    const int w = blockIdx.x * (kDetectCols / 32) + threadIdx.x;
    if (w < Kw)
      part[(int64_t)blockIdx.y * Kw + w] =
          words[0][threadIdx.x] | words[1][threadIdx.x] | words[2][threadIdx.x] | words[3][threadIdx.x];
  }
}

// ---------------------------------------------------------------------------
// a4 (prefill): OR the partial flags, write the final bitmask and the
// ascending outlier index list and its length.  One CTA of 1024 threads;
// thread i owns words [i*wpt, (i+1)*wpt), so a prefix sum of per-thread
// counts orders the indices.
// ---------------------------------------------------------------------------
constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads) compact_kernel(
    const uint32_t* __restrict__ part, int R, int Kw, uint32_t* __restrict__ flags,
    int32_t* __restrict__ idx, int32_t* __restrict__ n_out) {
  __shared__ int scratch[33];
  pdl_wait();
  pdl_launch_dependents();
  const int wpt = (Kw + kCompactThreads - 1) / kCompactThreads;
  const int w0 = threadIdx.x * wpt;
  int count = 0;
  for (int i = 0; i < wpt; ++i) {
    const int w = w0 + i;
    if (w >= Kw) break;
    uint32_t f = 0;
    for (int r = 0; r < R; ++r) f |= part[(int64_t)r * Kw + w];
    flags[w] = f;
    count += __popc(f);
  }
  int total;
  int pos = block_exclusive_scan(count, scratch, &total);
  for (int i = 0; i < wpt; ++i) {
    const int w = w0 + i;
    if (w >= Kw) break;
    uint32_t f = flags[w];
    while (f) {
      const int b = __ffs(f) - 1;
      idx[pos++] = w * 32 + b;
      f &= f - 1;
    }
  }
  if (threadIdx.x == 0) *n_out = total;
}

// ---------------------------------------------------------------------------
// a2 + a3 + a4 gathers (prefill).  Blocks [0, T): one row of X each -> sx[t],
// Xq[t, :], Xo[t, 0:Opad) = X[t, idx] (zero past |O|).  Blocks [T, T + nwb):
// rows of W -> Wo[n, 0:Opad) = W[n, idx].  Opad = |O| rounded up to 64 (one
// 128-byte fp16 K block of the outlier GEMM).
// ---------------------------------------------------------------------------
constexpr int kWoRowsPerCta = 16;

__global__ void __launch_bounds__(kPrepThreads) quant_gather_kernel(
    const uint16_t* __restrict__ X, int T, int K, const uint16_t* __restrict__ W, int N,
    const uint32_t* __restrict__ flags, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ n_out, int8_t* __restrict__ Xq, float* __restrict__ sx,
    uint16_t* __restrict__ Xo, uint16_t* __restrict__ Wo, int ldo) {
  __shared__ float red[32];
  pdl_wait();
  pdl_launch_dependents();
  const int nO = *n_out;
  const int opad = (nO + 63) & ~63;
  if (static_cast<int>(blockIdx.x) < T) {
    const int64_t t = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(X + t * K);
    const uint8_t* fb = reinterpret_cast<const uint8_t*>(flags);
    const int nchunk = K >> 3;
    float m = 0.0f;
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) m = absmax8(row[c], fb[c], m);
    const float amax = block_max(m, red);
    const float s = __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0) sx[t] = s;
    uint2* out = reinterpret_cast<uint2*>(Xq + t * K);
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) out[c] = quant8(row[c], s, fb[c]);
    for (int j = threadIdx.x; j < opad; j += blockDim.x)
      Xo[t * ldo + j] = j < nO ? X[t * K + idx[j]] : uint16_t(0);
  } else {
    const int64_t n0 = (int64_t)(blockIdx.x - T) * kWoRowsPerCta;
    for (int rr = 0; rr < kWoRowsPerCta; ++rr) {
      const int64_t n = n0 + rr;
      if (n >= N) break;
      for (int j = threadIdx.x; j < opad; j += blockDim.x)
        Wo[n * ldo + j] = j < nO ? __ldg(W + n * K + idx[j]) : uint16_t(0);
    }
  }
}

// ---------------------------------------------------------------------------
// Decode (T <= 16): every activation stage in one CTA of 1024 threads --
// flags, ascending index list, per-row scales and codes -- and the reset of
// the GEMV's per-tile arrival counters.  Launched without a programmatic
// dependency, so the previous call on the stream has fully completed; it lets
// the GEMV launch at once so that the weight stream starts while this runs.
// Dynamic shared memory: K/8 bytes of per-chunk outlier masks.
// ---------------------------------------------------------------------------
constexpr int kDecodePrepThreads = 1024;

__global__ void __launch_bounds__(kDecodePrepThreads) decode_prep_kernel(
    const uint16_t* __restrict__ X, int T, int K, float tau, uint32_t* __restrict__ flags,
    int32_t* __restrict__ idx, int32_t* __restrict__ n_out, int8_t* __restrict__ Xq,
    float* __restrict__ sx, int32_t* __restrict__ counters, int ncounters) {
  extern __shared__ uint8_t fmask[];  // [K/8]
  __shared__ int scratch[33];
  pdl_launch_dependents();
  const int nchunk = K >> 3;
  for (int i = threadIdx.x; i < ncounters; i += blockDim.x) counters[i] = 0;
  // a1: flags of every 8-column chunk over the T rows
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    uint32_t m = 0;
    for (int t = 0; t < T; ++t)
      m |= outlier_mask8(__ldg(reinterpret_cast<const uint4*>(X + (int64_t)t * K) + c), tau);
    fmask[c] = static_cast<uint8_t>(m);
  }
  __syncthreads();
  const int Kw = (K + 31) >> 5;
  for (int w = threadIdx.x; w < Kw; w += blockDim.x) {
    uint32_t f = 0;
    for (int b = 0; b < 4; ++b)
      if (4 * w + b < nchunk) f |= static_cast<uint32_t>(fmask[4 * w + b]) << (8 * b);
    flags[w] = f;
  }
  // a4: ascending index list
  const int cpt = (nchunk + blockDim.x - 1) / blockDim.x;
  const int c0 = threadIdx.x * cpt;
  int count = 0;
  for (int i = 0; i < cpt; ++i)
    if (c0 + i < nchunk) count += __popc(static_cast<uint32_t>(fmask[c0 + i]));
  int total;
  int pos = block_exclusive_scan(count, scratch, &total);
  for (int i = 0; i < cpt; ++i) {
    const int c = c0 + i;
    if (c >= nchunk) break;
    uint32_t f = fmask[c];
    while (f) {
      const int b = __ffs(f) - 1;
      idx[pos++] = c * 8 + b;
      f &= f - 1;
    }
  }
  if (threadIdx.x == 0) *n_out = total;
  // a2 + a3: one warp per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < T; t += blockDim.x >> 5) {
    const uint4* row = reinterpret_cast<const uint4*>(X + (int64_t)t * K);
    float m = 0.0f;
    for (int c = lane; c < nchunk; c += 32) m = absmax8(__ldg(row + c), fmask[c], m);
    const float s = __fdiv_rn(warp_max(m), 127.0f);
    if (lane == 0) sx[t] = s;
    uint2* out = reinterpret_cast<uint2*>(Xq + (int64_t)t * K);
    for (int c = lane; c < nchunk; c += 32) out[c] = quant8(__ldg(row + c), s, fmask[c]);
  }
}

}  // namespace llmint8
