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
#include "quant.cuh"
#include "sm100.cuh"

namespace llmint8 {

constexpr int kPrepThreads = 256;

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
  const float inv = scale_reciprocal(s);
  if (threadIdx.x == 0) Wscale[n] = s;
  uint2* out = reinterpret_cast<uint2*>(Wq + n * K);
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) out[c] = quant8(__ldg(row + c), s, inv, 0u);
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
  pdl_wait();  // X, and the workspace the previous call may still be reading
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
  pdl_launch_dependents();
  pdl_wait();
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
  pdl_launch_dependents();
  pdl_wait();
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
    const float inv = scale_reciprocal(s);
    if (threadIdx.x == 0) sx[t] = s;
    uint2* out = reinterpret_cast<uint2*>(Xq + t * K);
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) out[c] = quant8(row[c], s, inv, fb[c]);
    for (int j = threadIdx.x; j < opad; j += blockDim.x)
      Xo[t * ldo + j] = j < nO ? X[t * K + idx[j]] : uint16_t(0);
  } else {
    // Wo rows: every (row, column) pair is an independent item, 4 loads in
    // flight per thread before their stores.
    const int64_t n0 = (int64_t)(blockIdx.x - T) * kWoRowsPerCta;
    const int64_t left = static_cast<int64_t>(N) - n0;
    const int rows = left < kWoRowsPerCta ? static_cast<int>(left) : kWoRowsPerCta;
    const int total = rows * opad;
    for (int base = threadIdx.x; base < total; base += 4 * blockDim.x) {
      uint16_t v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = base + u * blockDim.x;
        v[u] = 0;
        if (e < total) {
          const int rr = e / opad, j = e - rr * opad;
          if (j < nO) v[u] = __ldg(W + (n0 + rr) * K + idx[j]);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = base + u * blockDim.x;
        if (e < total) {
          const int rr = e / opad, j = e - rr * opad;
          Wo[(n0 + rr) * ldo + j] = v[u];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Decode (T <= 16): every activation stage in one CTA of 1024 threads, built
// for latency: a pass issues all its loads before using any.  Item e is
// (chunk c = e / TMAX, row t = e % TMAX) with TMAX = T rounded up to a power of
// two, so the TMAX rows of a chunk sit in adjacent lanes: its outlier mask is
// an OR across them, and each thread keeps one row's running absmax.
//   pass 1: masks -> shared mask bytes; per-row absmax over regular columns
//   reduce: sx[t] = max / 127, inv[t] = 1 / sx[t]
//   pass 2: codes (X re-read from L2) -> Xq
//   then the ascending outlier list, |O|, and zeroed GEMV tile counters.
// Waits for its predecessor before touching memory and lets the GEMV launch
// at once, so the GEMV streams weights while this runs.
// ---------------------------------------------------------------------------
constexpr int kDecodeThreads = 1024;
constexpr int kDecodeInFlight = 8;  // loads per thread per round

template <int TMAX>
__global__ void __launch_bounds__(kDecodeThreads) decode_prep_kernel(
    const uint16_t* __restrict__ X, int T, int K, float tau, int8_t* __restrict__ Xq,
    float* __restrict__ sx, int32_t* __restrict__ idx, int32_t* __restrict__ n_out,
    int32_t* __restrict__ counters, int ncounters) {
  __shared__ uint8_t fm[65536 / 8];
  __shared__ float red[kDecodeThreads / 32][TMAX];
  __shared__ float s_sx[TMAX], s_inv[TMAX];
  __shared__ int scratch[33];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nchunk = K >> 3;
  const int items = nchunk * TMAX;
  const int t = tid % TMAX;
  const uint16_t* xrow = X + static_cast<int64_t>(t) * K;
  for (int i = tid; i < ncounters; i += kDecodeThreads) counters[i] = 0;

  // pass 1
  // rounds are uniform across the block: the shuffles below need whole warps
  const int rounds = (items + kDecodeThreads * kDecodeInFlight - 1) / (kDecodeThreads * kDecodeInFlight);
  float m = 0.0f;
  for (int r = 0; r < rounds; ++r) {
    const int base = r * kDecodeThreads * kDecodeInFlight + tid;
    uint4 v[kDecodeInFlight];
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      v[u] = (e < items && t < T) ? __ldg(reinterpret_cast<const uint4*>(xrow) + e / TMAX)
                                  : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      uint32_t mask = outlier_mask8(v[u], tau) & (t < T ? 0xFFu : 0u);
#pragma unroll
      for (int o = 1; o < TMAX; o <<= 1) mask |= __shfl_xor_sync(0xffffffffu, mask, o);
      if (e < items && t == 0) fm[e / TMAX] = static_cast<uint8_t>(mask);
      m = absmax8(v[u], mask, m);
    }
  }
#pragma unroll
  for (int o = 16; o >= TMAX; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane < TMAX) red[warp][lane] = m;
  __syncthreads();
  if (tid < TMAX) {
    float mm = 0.0f;
    for (int w = 0; w < kDecodeThreads / 32; ++w) mm = fmaxf(mm, red[w][tid]);
    const float s = __fdiv_rn(mm, 127.0f);
    s_sx[tid] = s;
    s_inv[tid] = scale_reciprocal(s);
    if (tid < T) sx[tid] = s;
  }
  __syncthreads();

  // pass 2
  const float st = s_sx[t], it = s_inv[t];
  for (int r = 0; r < rounds; ++r) {
    const int base = r * kDecodeThreads * kDecodeInFlight + tid;
    uint4 v[kDecodeInFlight];
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      v[u] = (e < items && t < T) ? __ldg(reinterpret_cast<const uint4*>(xrow) + e / TMAX)
                                  : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      if (e < items && t < T) {
        const int c = e / TMAX;
        reinterpret_cast<uint2*>(Xq + static_cast<int64_t>(t) * K)[c] = quant8(v[u], st, it, fm[c]);
      }
    }
  }

  // ascending outlier list: thread i owns chunks [i*cpt, (i+1)*cpt)
  const int cpt = (nchunk + kDecodeThreads - 1) / kDecodeThreads;
  const int c0 = tid * cpt;
  int count = 0;
  for (int i = 0; i < cpt; ++i)
    if (c0 + i < nchunk) count += __popc(static_cast<uint32_t>(fm[c0 + i]));
  int total;
  int pos = block_exclusive_scan(count, scratch, &total);
  for (int i = 0; i < cpt; ++i) {
    const int c = c0 + i;
    if (c >= nchunk) break;
    uint32_t f = fm[c];
    while (f) {
      const int b = __ffs(f) - 1;
      idx[pos++] = c * 8 + b;
      f &= f - 1;
    }
  }
  if (tid == 0) *n_out = total;
}

}  // namespace llmint8
