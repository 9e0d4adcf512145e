// gemv_kernel.cuh -- decode-shaped LLM.int8() matmul (T <= 16 tokens).
//
// The int8 product acc = Xq * Wq^T is bound by reading Wq from HBM: decode
// reads every weight once per token batch ('三、模型量化' (lowentro.cn) Q15;
// 'LLM 量化' (llm-inference-handbook), why quantize).  So the kernel streams Wq
// with TMA, one 128 x 128-byte tile per stage, and multiplies on the tensor
// cores with the operands swapped: A = the Wq tile (MMA M = 128 output
// channels), B = the int8 codes of the T tokens padded to 16 (MMA N = 16),
// D = int32 in TMEM.  The codes, scales and outlier list come from
// decode_prep_kernel, which runs while this kernel already streams weights
// (programmatic dependent launch).
//
// Work split (stream-K): the N/128 x K/128 k-blocks are cut into one
// contiguous range per CTA, so every CTA streams the same number of weight
// bytes.  A range may start or end inside a tile; such partial int32 sums go to
// a per-CTA slot in the workspace and the last CTA to arrive at a tile (per-tile
// counter, no spinning) adds them -- exact in int32, so the order does not
// matter -- and writes
//   Y[t,n] = fp16( acc[t,n] * sx[t] * sw[n] + yo[t,n] ),
//   yo[t,n] = sum_{j<|O|} X[t,O_j] * W[n,O_j]   (fp32, ascending j)
// ('LLM quantization, part 2' (hncyxsy.com) §2.1: outlier columns in fp16,
// the rest in int8, the two results added; '三、模型量化' Q2: r' = s * q on
// each operand).
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA; warp 1 lane 0 issues
// tcgen05.mma and owns TMEM; warps 2-5 (128 threads = 128 TMEM lanes) compute
// the outlier products while the weights stream, then drain the accumulators.
// Two 16-column accumulators let the MMA of one segment overlap the epilogue
// of the previous one.  Every mbarrier wait is bounded.
#pragma once
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace llmint8 {
namespace gemv {

constexpr int BM = 128;                    // weight rows per tile = MMA M
constexpr int BK = 128;                    // K bytes per k-block (one 128 B swizzle row)
constexpr int NT = 16;                     // tokens per MMA (MMA N)
constexpr int STAGES = 11;
constexpr int A_BYTES = BM * BK;           // 16 KiB of Wq
constexpr int B_BYTES = NT * BK;           // 2 KiB of activation codes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 32;              // 2 accumulators x 16 columns
constexpr int XO_CHUNK = 64;               // outlier columns staged per epilogue pass
constexpr int MAX_CTAS = 256;              // partial-slot capacity of the workspace
constexpr int SLOT_INTS = BM * NT;         // one partial tile, int32 [128][16]
constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 256 +
                           NT * XO_CHUNK * 4 + XO_CHUNK * 4;

struct Params {
  int T, N, K;
  int KB;             // k-blocks per tile = ceil(K / BK)
  int num_tiles;      // ceil(N / BM)
  int units;          // num_tiles * KB
  int grid;           // CTAs (<= units, <= MAX_CTAS)
  const float* sx;
  const float* sw;
  const uint16_t* X;
  const uint16_t* W;
  const int32_t* idx;
  const int32_t* n_out;
  int32_t* counters;  // [num_tiles]: zeroed by the prep kernel, reset by each tile's last CTA
  int32_t* partials;  // [grid][2][BM][NT]
  uint16_t* Y;
  int32_t* acc_out;   // optional int32 [T][N]
  uint64_t wait_ns;
};

__device__ __forceinline__ int unit_begin(int c, const Params& p) {
  return static_cast<int>((static_cast<int64_t>(c) * p.units) / p.grid);
}

// CTA whose range holds unit u.
__device__ __forceinline__ int cta_of_unit(int u, const Params& p) {
  int c = static_cast<int>((static_cast<int64_t>(u) * p.grid) / p.units);
  while (c + 1 < p.grid && unit_begin(c + 1, p) <= u) ++c;
  while (c > 0 && unit_begin(c, p) > u) --c;
  return c;
}

// Outlier products of one tile row in each of two tiles (the two may be the
// same): for n = tile * BM + row,
//   yo[t] = sum_{j<|O|} X[t, O_j] * W[n, O_j]   (fp32, ascending j), t < TMAX.
// All 128 epilogue threads call this together.  Per 64 outlier columns: the
// indices go to shared memory, then the X values and both rows' W values are
// gathered with all loads in flight at once (two dependent round trips per
// chunk, whatever the number of tiles).
template <int TMAX>
__device__ __forceinline__ void outlier_products(const Params& p, int nO, int tile_a, int tile_b, int row,
                                                 int etid, float* xo_s, int32_t* idx_s, float (&ya)[TMAX],
                                                 float (&yb)[TMAX]) {
#pragma unroll
  for (int t = 0; t < TMAX; ++t) {
    ya[t] = 0.0f;
    yb[t] = 0.0f;
  }
  const int na = tile_a * BM + row, nb = tile_b * BM + row;
  const uint16_t* wa = p.W + static_cast<int64_t>(na < p.N ? na : 0) * p.K;
  const uint16_t* wb = p.W + static_cast<int64_t>(nb < p.N ? nb : 0) * p.K;
  for (int j0 = 0; j0 < nO; j0 += XO_CHUNK) {
    const int cnt = min(XO_CHUNK, nO - j0);
    named_barrier(1, 128);  // the previous chunk has been read
    if (etid < XO_CHUNK) idx_s[etid] = etid < cnt ? p.idx[j0 + etid] : 0;
    named_barrier(1, 128);
    constexpr int PER = (TMAX * XO_CHUNK + 127) / 128;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = etid + 128 * i;
      const int t = e / XO_CHUNK, jj = e % XO_CHUNK;
      v[i] = (t < p.T && jj < cnt)
                 ? half_bits_to_float(p.X[static_cast<int64_t>(t) * p.K + idx_s[jj]])
                 : 0.0f;
    }
    constexpr int G = 8;  // outlier columns per batch of weight loads
    uint16_t w_a[G], w_b[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int k = u < cnt ? idx_s[u] : 0;
      w_a[u] = u < cnt ? __ldg(wa + k) : uint16_t(0);
      w_b[u] = u < cnt ? __ldg(wb + k) : uint16_t(0);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (etid + 128 * i < TMAX * XO_CHUNK) xo_s[etid + 128 * i] = v[i];
    named_barrier(1, 128);
    for (int jj0 = 0; jj0 < cnt; jj0 += G) {
      if (jj0 > 0) {
#pragma unroll
        for (int u = 0; u < G; ++u) {
          const int k = jj0 + u < cnt ? idx_s[jj0 + u] : 0;
          w_a[u] = jj0 + u < cnt ? __ldg(wa + k) : uint16_t(0);
          w_b[u] = jj0 + u < cnt ? __ldg(wb + k) : uint16_t(0);
        }
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const float fa = half_bits_to_float(w_a[u]), fb = half_bits_to_float(w_b[u]);
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          const float x = xo_s[t * XO_CHUNK + jj0 + u];
          ya[t] = fmaf(x, fa, ya[t]);
          yb[t] = fmaf(x, fb, yb[t]);
        }
      }
    }
  }
}

// TMAX: T rounded up to a power of two (1, 2, 4, 8 or 16); the per-token
// registers and loops of the epilogue are sized by it.
template <int TMAX>
__global__ void __launch_bounds__(THREADS, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                const Params p) {
  static_assert(TMAX >= 1 && TMAX <= NT && (TMAX & (TMAX - 1)) == 0, "TMAX: 1, 2, 4, 8 or 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint64_t* done = tempty + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xo_s = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + 256);  // [NT][XO_CHUNK]
  int32_t* idx_s = reinterpret_cast<int32_t*>(xo_s + NT * XO_CHUNK);          // [XO_CHUNK]

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int cta = blockIdx.x;
  const int u0 = unit_begin(cta, p);
  const int u1 = unit_begin(cta + 1, p);

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_x);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  __syncwarp();  // warp 0 converged: the CTA barrier counts each warp once
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();  // the next call's kernels may launch and start prefetching

  auto stage_a = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int n_units = u1 - u0;
      const int pre = n_units < STAGES ? n_units : STAGES;
      // The weights do not depend on earlier kernels: stream them before
      // waiting for the activation codes.
      for (int i = 0; i < pre; ++i) {
        const int u = u0 + i;
        mbar_arrive_expect_tx(&full[i], STAGE_BYTES);
        tma_load_2d_hint(stage_a(i), &tmap_w, &full[i], (u % p.KB) * BK, (u / p.KB) * BM, pol);
      }
      // The rest of this CTA's weight range goes to L2 now, so that HBM keeps
      // streaming while the ring is full and the activation codes are made.
      for (int i = pre; i < n_units; ++i) {
        const int u = u0 + i;
        tma_prefetch_l2_2d(&tmap_w, (u % p.KB) * BK, (u / p.KB) * BM);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        const int u = u0 + i;
        tma_load_2d(stage_b(i), &tmap_x, &full[i], (u % p.KB) * BK, 0);
      }
      int issued = pre;
      for (int i = pre; i < n_units; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, p.wait_ns, kErrTimeoutProducer)) break;
        const int u = u0 + i;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d_hint(stage_a(s), &tmap_w, &full[s], (u % p.KB) * BK, (u / p.KB) * BM, pol);
        tma_load_2d(stage_b(s), &tmap_x, &full[s], (u % p.KB) * BK, 0);
        ++issued;
      }
      // Leave no copy in flight: wait for the last loads of every stage.
      for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.wait_ns, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8_s32(BM, NT);
      int i = 0, seg = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++seg) {
        const int tile = u / p.KB;
        const int seg_end = min(u1, (tile + 1) * p.KB);
        const int buf = seg & 1;
        if (seg >= 2) {
          ok = mbar_wait(&tempty[buf], ((seg >> 1) - 1) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * NT);
        const int seg_start = u;
        for (; u < seg_end; ++u, ++i) {
          const int s = i % STAGES;
          ok = mbar_wait(&full[s], (i / STAGES) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = smem_addr(stage_a(s));
          const uint32_t b0 = smem_addr(stage_b(s));
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_i8(d, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc,
                   (u > seg_start || k > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[buf]);
      }
      // All issued MMAs complete before TMEM is released.
      mma_commit(done);
      mbar_wait(done, 0, p.wait_ns, kErrTimeoutMma);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;           // tile row = TMEM lane
    const int etid = threadIdx.x - 64;       // 0..127
    const int nO = *p.n_out;
    const int T = p.T;
    // The outlier product of the (at most two) tiles this CTA shares with
    // other CTAs does not depend on the int8 accumulators: compute it now,
    // while the weights stream, so the tile's last CTA only has to combine.
    const int tile_first = u0 / p.KB, tile_last = (u1 - 1) / p.KB;
    float yo_first[TMAX], yo_last[TMAX];
    outlier_products<TMAX>(p, nO, tile_first, tile_last, row, etid, xo_s, idx_s, yo_first, yo_last);
    float sxr[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) sxr[t] = t < T ? p.sx[t] : 0.0f;
    int seg = 0;
    for (int u = u0; u < u1; ++seg) {
      const int tile = u / p.KB;
      const int kb_begin = u % p.KB;
      const int seg_end = min(u1, (tile + 1) * p.KB);
      const bool whole = (kb_begin == 0) && (seg_end == (tile + 1) * p.KB);
      u = seg_end;
      const int buf = seg & 1;
      // All 128 epilogue threads agree on the outcome before going on, so a
      // timeout can never leave some of them at a named barrier.
      const bool ok = mbar_wait(&tfull[buf], (seg >> 1) & 1, p.wait_ns, kErrTimeoutEpilogue);
      if (!named_barrier_and(2, 128, ok)) break;
      __syncwarp();
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * NT), r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      int32_t acc[TMAX];
#pragma unroll
      for (int t = 0; t < TMAX; ++t) acc[t] = static_cast<int32_t>(r[t]);

      if (!whole) {
        const int c_first = cta_of_unit(tile * p.KB, p);
        const int c_last = cta_of_unit((tile + 1) * p.KB - 1, p);
        const int slot = (tile == tile_first) ? 0 : 1;
        int32_t* mine = p.partials + (static_cast<int64_t>(cta) * 2 + slot) * SLOT_INTS + row * NT;
#pragma unroll
        for (int t = 0; t < TMAX; ++t) mine[t] = acc[t];
        // The barrier orders the 128 threads' stores before the signalling
        // thread's GPU-scope fence (cumulativity), which releases them all
        // with its counter update; the last arriver's fence acquires the
        // others' partials, and the second barrier passes that on.
        named_barrier(1, 128);
        if (etid == 0) {
          __threadfence();
          const int old = atomicAdd(&p.counters[tile], 1);
          __threadfence();
          const bool is_last = old == c_last - c_first;
          if (is_last) p.counters[tile] = 0;  // every contributor has arrived: leave it clean
          *last_flag = is_last ? 1 : 0;
        }
        named_barrier(1, 128);
        const bool last = *last_flag != 0;
        if (!last) continue;
        for (int c2 = c_first; c2 <= c_last; ++c2) {
          if (c2 == cta) continue;
          const int slot2 = (tile == unit_begin(c2, p) / p.KB) ? 0 : 1;
          const int32_t* other = p.partials + (static_cast<int64_t>(c2) * 2 + slot2) * SLOT_INTS + row * NT;
          int32_t o[TMAX];
#pragma unroll
          for (int t = 0; t < TMAX; ++t) o[t] = __ldcg(other + t);
#pragma unroll
          for (int t = 0; t < TMAX; ++t) acc[t] += o[t];
        }
      }

      // ---- finalize this tile: dequantisation + outlier product, fp16 store
      float yo[TMAX];
      if (tile == tile_first) {
#pragma unroll
        for (int t = 0; t < TMAX; ++t) yo[t] = yo_first[t];
      } else if (tile == tile_last) {
#pragma unroll
        for (int t = 0; t < TMAX; ++t) yo[t] = yo_last[t];
      } else {
        float unused[TMAX];
        outlier_products<TMAX>(p, nO, tile, tile, row, etid, xo_s, idx_s, yo, unused);  // a whole tile
      }
      const int n = tile * BM + row;
      if (n < p.N) {
        const float swn = p.sw[n];
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          if (t < T) {
            const float y = static_cast<float>(acc[t]) * sxr[t] * swn + yo[t];
            p.Y[static_cast<int64_t>(t) * p.N + n] = __half_as_ushort(__float2half_rn(y));
            if (p.acc_out) p.acc_out[static_cast<int64_t>(t) * p.N + n] = acc[t];
          }
        }
      }
    }
  }

  // Lane 0 of warps 0 and 1 ran a role loop alone: bring each warp back
  // together first, so the CTA barrier waits for every warp (an aligned
  // barrier reached twice by one diverged warp would count it twice).
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemv
}  // namespace llmint8
