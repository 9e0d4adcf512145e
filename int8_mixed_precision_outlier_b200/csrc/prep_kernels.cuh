// prep_kernels.cuh -- the HBM-bound stages of the LLM.int8() matmul:
//   a0 weight quantisation (offline), a1 outlier detection, a4 compaction and
//   gathers with a2+a3 per-row scale and int8 codes of X.
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
// FP8: the same with E4M3 codes and s = amax / 448.
template <bool FP8>
__global__ void __launch_bounds__(kPrepThreads) quantize_weight_kernel(
    const uint16_t* __restrict__ W, int K, int8_t* __restrict__ Wq, float* __restrict__ Wscale) {
  __shared__ float red[32];
  const int64_t n = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(W + n * K);
  const int nchunk = K >> 3;
  float m = 0.0f;
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) m = absmax8(__ldg(row + c), 0u, m);
  const float amax = block_max(m, red);
  const float s = __fdiv_rn(amax, code_max<FP8>());
  const float inv = scale_reciprocal(s);
  if (threadIdx.x == 0) Wscale[n] = s;
  uint2* out = reinterpret_cast<uint2*>(Wq + n * K);
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) out[c] = quant8_codes<FP8>(__ldg(row + c), s, inv, 0u);
}

// ---------------------------------------------------------------------------
// a1 (prefill): the outlier flags, bit k%32 of word k/32 set iff some row has
// |X[t,k]| >= tau, and the first half of a2: for every row t and 128-column
// strip s, the maximum |X[t,k]| over the strip's regular columns,
// rowmax[t * nstrips + s] (the row's absmax is the maximum of these).
// A cluster of kDetectCluster CTAs owns a strip; CTA r scans rows
// [r*rpc, (r+1)*rpc).  Thread (c = tid % 16, rr = tid / 16) reads the 16
// bytes of chunk c in every 16th row and ORs 16-bit lane masks (the bits are
// formed once at the end).  With KEEP > 0 a thread's rows (at most KEEP) are
// loaded all at once and stay in registers; with KEEP = 0 they are streamed
// 8 at a time and read again (from L1 / L2) for the second pass.  Every CTA
// sends its four words to every CTA of the cluster (distributed shared
// memory), so after one cluster barrier each holds the strip's final flags:
// the first CTA writes them, and every CTA takes its rows' maxima over the
// unflagged columns, reduced over the 16 lanes of a row.
// ---------------------------------------------------------------------------
constexpr int kDetectCols = 128;
constexpr int kDetectCluster = 8;
// KEEP > 0: each thread's rows (at most KEEP) stay in registers between the
// two passes; KEEP = 0 reads them again.
template <int KEEP>
__global__ void __launch_bounds__(kPrepThreads) detect_kernel(const uint16_t* __restrict__ X, int T, int K,
                                                              float tau, int rpc, uint32_t* __restrict__ flags,
                                                              int Kw, float* __restrict__ rowmax, int nstrips) {
  constexpr int NW = kDetectCols / 32;  // flag words per strip
  __shared__ uint32_t words[NW];
  __shared__ uint32_t cw[kDetectCluster][NW];  // every CTA's words (each CTA holds a copy)
  const int c = threadIdx.x & 15, rr = threadIdx.x >> 4;
  const uint32_t rank = cluster_ctarank();
  const int strip = blockIdx.x / kDetectCluster;
  if (threadIdx.x < NW) words[threadIdx.x] = 0u;
  pdl_launch_dependents();
  cluster_sync();  // every CTA of the cluster runs before any remote store; words cleared
  pdl_wait();      // X, and the workspace the previous call may still be reading
  const int col0 = strip * kDetectCols + c * 8;
  const int t0 = static_cast<int>(rank) * rpc;
  const int t1 = min(T, t0 + rpc);
  const bool live = col0 < K;
  const uint16_t* base = X + col0;
  constexpr int U = 8;
  const __half2 tau2 = tau_half2(tau);
  Mask8 acc = {{0u, 0u, 0u, 0u}};
  uint4 kv[KEEP > 0 ? KEEP : 1];  // this thread's rows t0 + rr + 16 i, all loads in flight at once
  if constexpr (KEEP > 0) {
#pragma unroll
    for (int i = 0; i < KEEP; ++i) {
      const int t = t0 + rr + 16 * i;
      kv[i] = (live && t < t1) ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * K))
                               : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < KEEP; ++i)  // only loaded rows (a zero fill passes |x| >= tau for tau <= 0)
      if (live && t0 + rr + 16 * i < t1) outlier_mask8_or(kv[i], tau2, acc);
  } else if (live) {
    int t = t0 + rr;
    for (; t + 16 * (U - 1) < t1; t += 16 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t + 16 * u) * K));
#pragma unroll
      for (int u = 0; u < U; ++u) outlier_mask8_or(v[u], tau2, acc);
    }
    for (; t < t1; t += 16) outlier_mask8_or(__ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * K)), tau2, acc);
  }
  const uint32_t bits = mask_bits(acc);
  if (bits) atomicOr(&words[c >> 2], bits << ((c & 3) * 8));
  __syncthreads();
  if (threadIdx.x < NW * kDetectCluster) {  // thread i: word i % NW to CTA i / NW
    const uint32_t w = threadIdx.x % NW, dst = threadIdx.x / NW;
    st_cluster_u32(map_shared_rank(&cw[rank][w], dst), words[w]);
  }
  cluster_sync();
  uint32_t fw = 0;  // the strip's final word holding this thread's chunk
#pragma unroll
  for (int r = 0; r < kDetectCluster; ++r) fw |= cw[r][c >> 2];
  if (rank == 0 && threadIdx.x < NW) {
    uint32_t f = 0;
#pragma unroll
    for (int r = 0; r < kDetectCluster; ++r) f |= cw[r][threadIdx.x];
    const int w = strip * NW + static_cast<int>(threadIdx.x);
    if (w < Kw) flags[w] = f;
  }
  // the strip maxima of this CTA's rows over the regular columns
  const uint32_t skip = live ? (fw >> ((c & 3) * 8)) & 0xFFu : 0xFFu;
  const int rounds = (t1 - t0 + 15) / 16;  // uniform over the CTA (the shuffles need whole half-warps)
  if constexpr (KEEP > 0) {
#pragma unroll
    for (int i = 0; i < KEEP; ++i) {
      float m = absmax8(kv[i], skip, 0.0f);
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int t = t0 + rr + 16 * i;
      if (c == 0 && i < rounds && t < t1) rowmax[static_cast<int64_t>(t) * nstrips + strip] = m;
    }
  } else {
    for (int i0 = 0; i0 < rounds; i0 += U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + rr + 16 * (i0 + u);
        v[u] = (live && i0 + u < rounds && t < t1)
                   ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * K))
                   : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float m = absmax8(v[u], skip, 0.0f);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int t = t0 + rr + 16 * (i0 + u);
        if (c == 0 && i0 + u < rounds && t < t1) rowmax[static_cast<int64_t>(t) * nstrips + strip] = m;
      }
    }
  }
}

constexpr int kMaxKw = 65536 / 32;

// ---------------------------------------------------------------------------
// a2 + a3 + a4 (prefill), CTAs of 128 threads.  Every CTA copies the Kw flag
// words to shared memory and ranks them (exclusive prefix of the set bits per
// word): outlier column j is the j-th set bit, |O| the total.  CTA 0 writes the
// ascending index list and |O|.  Blocks [0, gather_ctas): 16 rows of W each ->
// Wo[n, 0:Opad) = W[n, O] (zero past |O|), or 32 rows from a column store;
// listed first because their scattered loads take longest.  Blocks past
// those: one row t of X each, in one pass: sx[t] = (the maximum of the row's
// strip maxima) / 127, Xq[t, :] and Xo[t, 0:Opad) = X[t, O], the outlier
// values taken from the registers that hold the row.  The row's first loads
// are issued before the flag words are ranked.
// Opad = |O| rounded up to 64 (one 128-byte fp16 K block of the outlier GEMM).
// FP8: E4M3 codes with sx = amax / 448 instead of int8 codes with amax / 127.
// Dynamic shared memory: 8 * Kw bytes (flag words and their ranks).
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 128;
constexpr int kWoRowsPerCta = 16;
constexpr int kStoreRowsPerCta = 32;  // column-store gather: 32 rows x 64 columns per tile
constexpr int kGatherIdxCap = 1024;  // outlier indices listed in shared memory at a time

// Outlier columns of rank j in [j0, j1) -> si[j - j0].  Thread i owns the
// flag words [i * wpt, (i + 1) * wpt).
__device__ __forceinline__ void list_outliers(const uint32_t* sf, const int32_t* wpre, int Kw, int j0, int j1,
                                              int32_t* si) {
  const int wpt = (Kw + kQuantThreads - 1) / kQuantThreads;
  const int w0 = static_cast<int>(threadIdx.x) * wpt, w1 = min(Kw, w0 + wpt);
  for (int w = w0; w < w1; ++w) {
    int j = wpre[w];
    if (j >= j1) break;
    for (uint32_t f = sf[w]; f && j < j1; f &= f - 1, ++j)
      if (j >= j0) si[j - j0] = w * 32 + __ffs(f) - 1;
  }
}

// The flag words -> shared memory, ranked; returns |O|.  Thread i owns words
// [i * wpt, (i + 1) * wpt).  Ends with a CTA barrier.
__device__ __forceinline__ int rank_flags(const uint32_t* __restrict__ flags, int Kw, uint32_t* sf, int32_t* wpre,
                                          int* scratch) {
  const int wpt = (Kw + kQuantThreads - 1) / kQuantThreads;
  const int w0 = static_cast<int>(threadIdx.x) * wpt, w1 = min(Kw, w0 + wpt);
  int count = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t f = __ldg(flags + w);
    sf[w] = f;
    count += __popc(f);
  }
  int nO;
  int pos = block_exclusive_scan(count, scratch, &nO);
  for (int w = w0; w < w1; ++w) {
    wpre[w] = pos;
    pos += __popc(sf[w]);
  }
  __syncthreads();
  return nO;
}

// Outlier columns of this chunk (bits of `fbits`, chunk c = columns 8c..8c+7)
// -> Xo_row[rank]: the values are already in registers; ranks come from the
// ranked flag words.
__device__ __forceinline__ void emit_outliers(const uint4 v, int c, uint32_t fbits, const uint32_t* sf,
                                              const int32_t* wpre, uint16_t* xo_row) {
  const int w = c >> 2;
  int j = wpre[w] + __popc(sf[w] & ((1u << ((c & 3) * 8)) - 1u));
  for (uint32_t f = fbits; f; f &= f - 1) {
    const int i = __ffs(f) - 1;
    const uint32_t hw = i < 4 ? (i < 2 ? v.x : v.y) : (i < 6 ? v.z : v.w);
    xo_row[j++] = static_cast<uint16_t>(hw >> ((i & 1) * 16));
  }
}

// Outlier weights from a column store instead of the fp16 weight (W null,
// slot / Wst set): gather CTAs take 32 rows of Wo each and walk the outlier
// columns 64 at a time through a shared-memory tile: the tile's columns and
// store slots are staged first, then every thread has 16 independent loads in
// flight, reading 32 consecutive rows of a stored column (64 contiguous bytes)
// and writing 64 consecutive columns of Wo.  A column missing from the store
// gets fp16(fl(sw[n] * Wq[n,k])); CTA 0 counts those misses into *n_miss.
struct ColumnStore {
  const int32_t* slot = nullptr;   // [K]: row of Wst holding column k, or -1
  const uint16_t* Wst = nullptr;   // fp16 [n_store][N]
  const int8_t* Wq = nullptr;      // int8 codes [N][K]
  const float* sw = nullptr;       // weight scales [N]
  int32_t* n_miss = nullptr;       // optional
};

template <bool FP8>
__global__ void __launch_bounds__(kQuantThreads, 8) quant_gather_kernel(
    const uint16_t* __restrict__ X, int T, int K, const uint16_t* __restrict__ W, int N,
    const uint32_t* __restrict__ flags, int Kw, const float* __restrict__ rowmax, int nstrips,
    int32_t* __restrict__ idx, int32_t* __restrict__ n_out, int8_t* __restrict__ Xq, float* __restrict__ sx,
    uint16_t* __restrict__ Xo, uint16_t* __restrict__ Wo, int ldo, int gather_ctas, const ColumnStore cs) {
  extern __shared__ uint32_t sflags[];                          // [Kw] flag words, then [Kw] ranks
  int32_t* wpre = reinterpret_cast<int32_t*>(sflags + Kw);
  __shared__ int32_t si[kGatherIdxCap];
  __shared__ int scratch[33];
  __shared__ uint16_t tile[kStoreRowsPerCta][64 + 2];
  __shared__ int32_t tk[64], tslot[64];
  // The GEMM that follows may launch once every CTA of this grid has started:
  // its CTAs then take the SMs this grid's last CTAs leave and request their
  // first weight tiles while those finish.
  pdl_launch_dependents();
  pdl_wait();
  const int nchunk = K >> 3;
  const bool xrow = static_cast<int>(blockIdx.x) >= gather_ctas;
  // A row of X: its first round of loads goes out before the flags are ranked.
  constexpr int U = 4;  // loads in flight per thread
  constexpr int ROUND = kQuantThreads * U;
  const int64_t t = static_cast<int64_t>(blockIdx.x) - gather_ctas;
  const uint4* row = reinterpret_cast<const uint4*>(X + (xrow ? t : 0) * K);
  uint4 v0[U];
  float pm = 0.0f;
  if (xrow) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = static_cast<int>(threadIdx.x) + kQuantThreads * u;
      v0[u] = c < nchunk ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    // every warp reduces the row's strip maxima itself (no CTA barrier)
    for (int i = static_cast<int>(threadIdx.x & 31); i < nstrips; i += 32) pm = fmaxf(pm, __ldg(rowmax + t * nstrips + i));
  }
  const int nO = rank_flags(flags, Kw, sflags, wpre, scratch);
  if (blockIdx.x == 0) {  // the index list and |O|, for the caller and the next kernels
    const int wpt = (Kw + kQuantThreads - 1) / kQuantThreads;
    const int w0 = static_cast<int>(threadIdx.x) * wpt, w1 = min(Kw, w0 + wpt);
    for (int w = w0; w < w1; ++w) {
      int j = wpre[w];
      for (uint32_t f = sflags[w]; f; f &= f - 1) idx[j++] = w * 32 + __ffs(f) - 1;
    }
    if (threadIdx.x == 0) *n_out = nO;
    if (cs.n_miss) {  // outlier columns the column store does not hold
      __shared__ int miss_s;
      if (threadIdx.x == 0) miss_s = 0;
      __syncthreads();
      int miss = 0;
      for (int w = threadIdx.x; w < Kw; w += kQuantThreads)
        for (uint32_t f = sflags[w]; f; f &= f - 1) miss += cs.slot[w * 32 + __ffs(f) - 1] < 0 ? 1 : 0;
      miss = __reduce_add_sync(0xffffffffu, miss);
      if ((threadIdx.x & 31) == 0) atomicAdd(&miss_s, miss);
      __syncthreads();
      if (threadIdx.x == 0) *cs.n_miss = miss_s;
    }
  }
  const int opad = (nO + 63) & ~63;
  if (!xrow && !W) {
    // ---------------------------------------------------- column-store gather
    const int n0 = static_cast<int>(blockIdx.x) * kStoreRowsPerCta;
    const int rows = min(kStoreRowsPerCta, N - n0);
    constexpr int PER = kStoreRowsPerCta * 64 / kQuantThreads;  // 16 elements per thread
    for (int win = 0; win < opad; win += kGatherIdxCap) {
      __syncthreads();  // the previous window's indices have been read
      list_outliers(sflags, wpre, Kw, win, min(nO, win + kGatherIdxCap), si);
      for (int j0 = win; j0 < min(opad, win + kGatherIdxCap); j0 += 64) {
        __syncthreads();  // si is complete; the previous tile has been written out
        if (threadIdx.x < 64) {
          const int j = j0 + static_cast<int>(threadIdx.x);
          const int k = j < nO ? si[j - win] : 0;
          tk[threadIdx.x] = k;
          tslot[threadIdx.x] = j < nO ? cs.slot[k] : -2;  // -2: padding column, zeros
        }
        __syncthreads();
        uint16_t v[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = static_cast<int>(threadIdx.x) + kQuantThreads * u;
          const int jj = e / kStoreRowsPerCta, r = e % kStoreRowsPerCta, n = n0 + r;
          const int sl = tslot[jj];
          v[u] = 0;
          if (r < rows && sl != -2)
            v[u] = sl >= 0 ? __ldg(cs.Wst + static_cast<int64_t>(sl) * N + n)
                           : __half_as_ushort(__float2half_rn(__fmul_rn(
                                 __ldg(cs.sw + n), static_cast<float>(cs.Wq[static_cast<int64_t>(n) * K + tk[jj]]))));
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = static_cast<int>(threadIdx.x) + kQuantThreads * u;
          tile[e % kStoreRowsPerCta][e / kStoreRowsPerCta] = v[u];
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = static_cast<int>(threadIdx.x) + kQuantThreads * u;
          const int r = e / 64, jj = e % 64;
          if (r < rows) Wo[static_cast<int64_t>(n0 + r) * ldo + j0 + jj] = tile[r][jj];
        }
      }
    }
    return;
  }
  if (!xrow) {
    // ---------------------------------------------------- fp16 weight gather
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kWoRowsPerCta;
    const int64_t left = static_cast<int64_t>(N) - n0;
    const int rows = left < kWoRowsPerCta ? static_cast<int>(left) : kWoRowsPerCta;
    for (int win = 0; win < opad; win += kGatherIdxCap) {
      __syncthreads();  // the previous window's indices have been read
      list_outliers(sflags, wpre, Kw, win, min(nO, win + kGatherIdxCap), si);
      __syncthreads();
      // thread i takes column jj = i (+ 128 ...) of the window, 8 rows at a time
      const int width = min(opad - win, kGatherIdxCap);
      constexpr int UG = 8;
      for (int jj = static_cast<int>(threadIdx.x); jj < width; jj += kQuantThreads) {
        const bool real = win + jj < nO;  // past |O|: padding, zeros
        const int k = real ? si[jj] : 0;
        for (int r0 = 0; r0 < rows; r0 += UG) {
          uint16_t v[UG];
#pragma unroll
          for (int u = 0; u < UG; ++u)
            v[u] = (real && r0 + u < rows) ? __ldg(W + (n0 + r0 + u) * K + k) : uint16_t(0);
#pragma unroll
          for (int u = 0; u < UG; ++u)
            if (r0 + u < rows) Wo[(n0 + r0 + u) * ldo + win + jj] = v[u];
        }
      }
    }
    return;
  }
  // ------------------------------------------------------ one row of X, one pass
  pm = warp_max(pm);
  const float s = __fdiv_rn(pm, code_max<FP8>());
  const float inv = scale_reciprocal(s);
  if (threadIdx.x == 0) sx[t] = s;
  const uint8_t* fb = reinterpret_cast<const uint8_t*>(sflags);  // byte c: the flags of chunk c
  uint2* out = reinterpret_cast<uint2*>(Xq + t * K);
  uint16_t* xo_row = Xo + t * ldo;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = static_cast<int>(threadIdx.x) + kQuantThreads * u;
    if (c < nchunk) {
      const uint32_t f = fb[c];
      out[c] = quant8_codes<FP8>(v0[u], s, inv, f);
      if (f) emit_outliers(v0[u], c, f, sflags, wpre, xo_row);
    }
  }
  for (int c0 = static_cast<int>(threadIdx.x) + ROUND; c0 < nchunk; c0 += ROUND) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + kQuantThreads * u;
      v[u] = c < nchunk ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + kQuantThreads * u;
      if (c < nchunk) {
        const uint32_t f = fb[c];
        out[c] = quant8_codes<FP8>(v[u], s, inv, f);
        if (f) emit_outliers(v[u], c, f, sflags, wpre, xo_row);
      }
    }
  }
  for (int j = nO + static_cast<int>(threadIdx.x); j < opad; j += kQuantThreads) xo_row[j] = uint16_t(0);
}

// ---------------------------------------------------------------------------
// Decode (T <= 16): every activation stage in one cluster of 8 CTAs.  CTA r of
// the cluster owns a contiguous slice of 8-column chunks for all T rows.  Item
// e of a CTA is (chunk c = e / TMAX, row t = e % TMAX), TMAX = T rounded up to a
// power of two, so a chunk's rows sit in adjacent lanes: its outlier mask is an
// OR across them, and each thread keeps one row's running absmax.
//   pass 1: masks -> shared mask bytes; per-row absmax over regular columns
//   exchange: each CTA writes its per-row maxima and its outlier count into
//     every CTA's shared memory (distributed shared memory); after one
//     cluster barrier every CTA forms sx[t] = max / 127 and its offset in the
//     list from its own copies
//   then: this CTA's outlier indices; codes (values kept in registers, or X
//     re-read from L2) -> Xq
// FP8: E4M3 codes with sx = amax / 448 instead of int8 codes with amax / 127.
// 256 threads and at most 64 registers per CTA let a CTA share an SM with a
// GEMV CTA, so the cluster launches while the previous call's GEMV runs.  It
// waits for its predecessor before touching memory and lets the GEMV launch at
// once, so the GEMV streams weights while this runs.
// ---------------------------------------------------------------------------
constexpr int kDecodeCtas = 8;
constexpr int kDecodeThreads = 256;
constexpr int kDecodeInFlight = 4;   // loads per thread per round
constexpr int kDecodeMaxSlice = 65536 / 8 / kDecodeCtas;  // chunks per CTA at K = 65536

template <int TMAX, bool FP8>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_prep_kernel(
    const uint16_t* __restrict__ X, int T, int K, float tau, int8_t* __restrict__ Xq,
    float* __restrict__ sx, int32_t* __restrict__ idx, int32_t* __restrict__ n_out) {
  __shared__ uint8_t fm[kDecodeMaxSlice];
  __shared__ float red[kDecodeThreads / 32][TMAX];
  __shared__ float part[kDecodeCtas][TMAX];  // every CTA's row maxima (each CTA holds a copy)
  __shared__ int cnt[kDecodeCtas];           // every CTA's outlier count (each CTA holds a copy)
  __shared__ float s_sx[TMAX], s_inv[TMAX];
  __shared__ int s_off;
  __shared__ int scratch[33];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int nchunk = K >> 3;
  const int cpc = (nchunk + kDecodeCtas - 1) / kDecodeCtas;
  const int c_begin = static_cast<int>(rank) * cpc;
  const int myn = max(0, min(nchunk, c_begin + cpc) - c_begin);
  const int items = myn * TMAX;
  const int t = tid % TMAX;
  const uint4* xrow = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t) * K) + c_begin;
  // Ask L2 for this thread's lines of X before waiting for the previous
  // kernel: the loads after the wait then do not queue behind the GEMV's
  // weight stream at DRAM.  A prefetch only reads (L2 stays coherent with
  // any later write of X), so it is safe however X is produced.
  for (int e = tid; e < items; e += kDecodeThreads)
    if (t < T && (e / TMAX) % 8 == 0) prefetch_l2(xrow + e / TMAX);
  const __half2 tau2 = tau_half2(tau);
  cluster_sync();  // every CTA of the cluster has started before any remote access
  pdl_wait();

  // pass 1 (rounds are uniform across the CTA: the shuffles need whole warps)
  const int rounds = (items + kDecodeThreads * kDecodeInFlight - 1) / (kDecodeThreads * kDecodeInFlight);
  float m = 0.0f;
  uint4 keep[kDecodeInFlight];  // the slice's values when one round covers it
  for (int r = 0; r < rounds; ++r) {
    const int base = r * kDecodeThreads * kDecodeInFlight + tid;
    uint4 v[kDecodeInFlight];
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      v[u] = (e < items && t < T) ? __ldg(xrow + e / TMAX) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      uint32_t mask = outlier_mask8(v[u], tau2) & (t < T ? 0xFFu : 0u);
#pragma unroll
      for (int o = 1; o < TMAX; o <<= 1) mask |= __shfl_xor_sync(0xffffffffu, mask, o);
      if (e < items && t == 0) fm[e / TMAX] = static_cast<uint8_t>(mask);
      m = absmax8(v[u], mask, m);
      keep[u] = v[u];
    }
  }
#pragma unroll
  for (int o = 16; o >= TMAX; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane < TMAX) red[warp][lane] = m;
  __syncthreads();  // red and fm complete
  // This CTA's outlier positions, ascending: thread i owns chunks
  // [i*cpt, (i+1)*cpt); the scan gives its place among this CTA's outliers.
  const int cpt = (myn + kDecodeThreads - 1) / kDecodeThreads;
  const int c0 = tid * cpt;
  int count = 0;
  for (int i = 0; i < cpt; ++i)
    if (c0 + i < myn) count += __popc(static_cast<uint32_t>(fm[c0 + i]));
  int my_total;
  const int pos_local = block_exclusive_scan(count, scratch, &my_total);
  // Every CTA sends its row maxima and outlier count to every CTA of the
  // cluster, so that after one cluster barrier each reads its own copies
  // (and no CTA's shared memory is read after it may have exited).
  if (tid < TMAX * kDecodeCtas) {
    const int tt = tid % TMAX, dst = tid / TMAX;
    float pm = 0.0f;
#pragma unroll
    for (int w = 0; w < kDecodeThreads / 32; ++w) pm = fmaxf(pm, red[w][tt]);
    st_cluster_f32(map_shared_rank(&part[rank][tt], static_cast<uint32_t>(dst)), pm);
  }
  if (tid >= 224 && tid < 224 + kDecodeCtas)
    st_cluster_u32(map_shared_rank(&cnt[rank], static_cast<uint32_t>(tid - 224)), static_cast<uint32_t>(my_total));
  cluster_sync();

  if (tid < TMAX) {
    float mm = 0.0f;
#pragma unroll
    for (int r = 0; r < kDecodeCtas; ++r) mm = fmaxf(mm, part[r][tid]);
    const float s = __fdiv_rn(mm, code_max<FP8>());
    s_sx[tid] = s;
    s_inv[tid] = scale_reciprocal(s);
    if (rank == 0 && tid < T) sx[tid] = s;
  }
  if (tid == 32) {
    int off = 0, total = 0;
    for (int r = 0; r < kDecodeCtas; ++r) {
      const int c = cnt[r];
      off += r < static_cast<int>(rank) ? c : 0;
      total += c;
    }
    s_off = off;
    if (rank == 0) *n_out = total;
  }
  __syncthreads();  // s_sx, s_inv, s_off

  // outlier indices
  int pos = s_off + pos_local;
  for (int i = 0; i < cpt; ++i) {
    const int c = c0 + i;
    if (c >= myn) break;
    for (uint32_t f = fm[c]; f; f &= f - 1) idx[pos++] = (c_begin + c) * 8 + (__ffs(f) - 1);
  }

  // pass 2: codes
  const float st = s_sx[t], it = s_inv[t];
  for (int r = 0; r < rounds; ++r) {
    const int base = r * kDecodeThreads * kDecodeInFlight + tid;
    uint4 v[kDecodeInFlight];
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      v[u] = rounds == 1 ? keep[u]
             : (e < items && t < T) ? __ldg(xrow + e / TMAX) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDecodeInFlight; ++u) {
      const int e = base + u * kDecodeThreads;
      if (e < items && t < T) {
        const int c = e / TMAX;
        reinterpret_cast<uint2*>(Xq + static_cast<int64_t>(t) * K)[c_begin + c] =
            quant8_codes<FP8>(v[u], st, it, fm[c]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Column store build (offline): Wst[i][n] = W[n, cols[i]] and slot[cols[i]] = i
// (slot was set to -1 everywhere before).  A grid-stride loop over the
// n_cols * N elements, i-major; a column outside [0, K) is skipped (no access
// is made with it) and flagged in the error word.
// ---------------------------------------------------------------------------
__global__ void store_build_kernel(const uint16_t* __restrict__ W, int N, int K, const int32_t* __restrict__ cols,
                                   int n_cols, int32_t* __restrict__ slot, uint16_t* __restrict__ Wst) {
  const int64_t total = static_cast<int64_t>(n_cols) * N;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / N), n = static_cast<int>(e % N);
    const int k = cols[i];
    if (k < 0 || k >= K) {
      if (n == 0) atomicOr(&g_error_word, kErrBadColumn);
      continue;
    }
    if (n == 0) slot[k] = i;
    Wst[e] = W[static_cast<int64_t>(n) * K + k];
  }
}

}  // namespace llmint8
