// gemv_kernel.cuh -- decode-shaped LLM.int8() matmul (T <= 16 tokens).
//
// The int8 product acc = Xq * Wq^T is bound by reading Wq from HBM: decode
// reads every weight once per token batch ('三、模型量化' (lowentro.cn) Q15;
// 'LLM 量化' (llm-inference-handbook), why quantize).  So the kernel streams Wq
// with TMA and multiplies on the tensor cores with the operands swapped:
// A = a slab of Wq rows (MMA M = 128 lanes, of which the first H hold output
// channels), B = the int8 codes of the T tokens padded to 16 (MMA N = 16),
// D = int32 in TMEM.  The codes, scales and outlier list come from
// decode_prep_kernel; this kernel launches early (programmatic dependent
// launch) and requests its first weight stages before the prep is done.
//
// Work split: CTA c owns output rows [c * CH * H, (c + 1) * CH * H), as CH
// chunks of H <= 128 rows (a multiple of 8), each over all of K, with H and CH
// chosen on the host so that the grid fills the SMs and every CTA streams the
// same number of bytes.  One stage holds KPB k-blocks of the chunk's rows:
// with K % 128 == 0 a single 3-D TMA copy brings KPB * 128 contiguous bytes of
// each row (long runs of DRAM, few copies), as KPB swizzled tiles of
// H x 128 bytes; otherwise KPB = 1 and a 2-D copy brings one k-block.  No
// CTA shares a row with another, so no partial sums cross CTAs: each chunk
// ends in
//   Y[t,n] = fp16( acc[t,n] * sx[t] * sw[n] + yo[t,n] ),
//   yo[t,n] = sum_{j<|O|} X[t,O_j] * W[n,O_j]   (fp32, ascending j)
// ('LLM quantization, part 2' (hncyxsy.com) §2.1: outlier columns in fp16,
// the rest in int8, the two results added; '三、模型量化' Q2: r' = s * q on
// each operand).  The M = 128 product of a chunk with H < 128 rows computes
// lanes H..127 from stale shared memory; those lanes are never read.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA; warp 1 lane 0 issues
// tcgen05.mma and owns TMEM; warps 2-5 (128 threads = 128 TMEM lanes) compute
// a chunk's outlier products while its weights stream, then drain its
// accumulator.  The weight copies of the first PRE stages are issued before
// the prep kernel is done (they do not depend on it), the activation codes of
// those stages as soon as it is.  Two 16-column accumulators let the MMA of one
// chunk overlap the epilogue of the previous one.  Every wait is bounded.
#pragma once
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace llmint8 {
namespace gemv {

constexpr int BM = 128;                    // MMA M (TMEM lanes); a chunk holds H <= BM rows
constexpr int BK = 128;                    // K bytes per k-block (one 128 B swizzle row)
constexpr int NT = 16;                     // tokens per MMA (MMA N)
constexpr int KPB_MAX = 4;                 // k-blocks per stage
constexpr int STAGES = 4;
constexpr int PRE = STAGES;                // weight stages requested before the prep kernel is done
constexpr int A_BYTES = 40 * 1024;         // Wq: KPB tiles of H x 128 bytes (H * 128 * KPB <= 40 KiB)
constexpr int B_TILE = NT * BK;            // 2 KiB of activation codes per k-block
constexpr int B_BYTES = KPB_MAX * B_TILE;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;

// k-blocks per stage for chunks of h rows: as many as fit, at most KPB_MAX.
__host__ __device__ constexpr int kpb_for_rows(int h) {
  return A_BYTES / (h * BK) < KPB_MAX ? A_BYTES / (h * BK) : KPB_MAX;
}
static_assert(kpb_for_rows(BM) >= 2, "two k-blocks of 128 rows per stage");
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 32;              // 2 accumulators x 16 columns
constexpr int XO_CHUNK = 64;               // outlier columns staged per epilogue pass
constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 256 +
                           NT * XO_CHUNK * 4 + 2 * XO_CHUNK * 4;

struct Params {
  int T, N, K;
  int KB;             // k-blocks per chunk = ceil(K / BK)
  int H;              // rows per chunk (8..128, a multiple of 8)
  int CH;             // chunks per CTA
  int KPB;            // k-blocks per stage
  int NU;             // stages (units) per chunk = ceil(KB / KPB)
  int kpb3d;          // 1: 3-D tensor maps, KPB k-blocks per copy; 0: 2-D maps, KPB = 1
  const float* sx;
  const float* sw;
  const uint16_t* X;
  const uint16_t* W;       // fp16 weight, read at the outlier columns; null with a column store
  const int32_t* slot;     // column store: slot[k] = row of Wst holding column k, or -1
  const uint16_t* Wst;     // column store: fp16 [n_store][N], one column of W per row
  const int8_t* Wqr;       // the int8 codes, read for outlier columns missing from the store
  int32_t* n_miss;         // optional: outlier columns missing from the store (written by CTA 0)
  const int32_t* idx;
  const int32_t* n_out;
  uint16_t* Y;
  int32_t* acc_out;   // optional int32 [T][N] (FP8: the f32 accumulator's bits)
  uint64_t wait_ns;
};

// The fp16 weight W[n, k] of an outlier column: from the fp16 weight, or from
// the column store (slot >= 0: contiguous in n across the warp's lanes), or,
// for a column missing from the store, fp16(fl(sw[n] * Wq[n,k])) -- the fp16
// value of its int8 weight ('LLM quantization, part 2' (hncyxsy.com) §2.1
// keeps outlier weights in fp16; §2.2: only 8-bit weights are kept in memory).
__device__ __forceinline__ uint16_t outlier_weight(const Params& p, int n, int k, int slot, float swn) {
  if (p.W) return __ldg(p.W + static_cast<int64_t>(n) * p.K + k);
  if (slot >= 0) return __ldg(p.Wst + static_cast<int64_t>(slot) * p.N + n);
  const float q = static_cast<float>(p.Wqr[static_cast<int64_t>(n) * p.K + k]);
  return __half_as_ushort(__float2half_rn(__fmul_rn(swn, q)));
}

// Outlier products of output row n (all 128 epilogue threads call this
// together, each with its own n; n >= N gives zeros):
//   yo[t] = sum_{j<|O|} X[t, O_j] * W[n, O_j]   (fp32, ascending j), t < TMAX.
// Per 64 outlier columns: the indices (and their store slots) go to shared
// memory, then the X values and the row's W values are gathered with all
// loads in flight at once.
template <int TMAX>
__device__ __forceinline__ void outlier_products(const Params& p, int nO, int n, int etid, float* xo_s,
                                                 int32_t* idx_s, int32_t* slot_s, float (&yo)[TMAX]) {
#pragma unroll
  for (int t = 0; t < TMAX; ++t) yo[t] = 0.0f;
  const bool valid = n < p.N;
  const int nv = valid ? n : 0;
  // The scale is read only to rebuild weights a column store does not hold
  // (calls without outlier columns may pass no scales at all).
  const float swn = (nO > 0 && p.slot && valid) ? p.sw[nv] : 0.0f;
  for (int j0 = 0; j0 < nO; j0 += XO_CHUNK) {
    const int cnt = min(XO_CHUNK, nO - j0);
    named_barrier(1, 128);  // the previous chunk has been read
    if (etid < XO_CHUNK) {
      const int k = etid < cnt ? p.idx[j0 + etid] : 0;
      idx_s[etid] = k;
      slot_s[etid] = p.slot ? p.slot[k] : -1;
    }
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
    uint16_t w[G];
#pragma unroll
    for (int u = 0; u < G; ++u)
      w[u] = (valid && u < cnt) ? outlier_weight(p, nv, idx_s[u], slot_s[u], swn) : uint16_t(0);
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (etid + 128 * i < TMAX * XO_CHUNK) xo_s[etid + 128 * i] = v[i];
    named_barrier(1, 128);
    for (int jj0 = 0; jj0 < cnt; jj0 += G) {
      if (jj0 > 0) {
#pragma unroll
        for (int u = 0; u < G; ++u)
          w[u] = (valid && jj0 + u < cnt) ? outlier_weight(p, nv, idx_s[jj0 + u], slot_s[jj0 + u], swn)
                                          : uint16_t(0);
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const float f = half_bits_to_float(w[u]);
#pragma unroll
        for (int t = 0; t < TMAX; ++t) yo[t] = fmaf(xo_s[t * XO_CHUNK + jj0 + u], f, yo[t]);
      }
    }
  }
}

// TMAX: T rounded up to a power of two (1, 2, 4, 8 or 16); the per-token
// registers and loops of the epilogue are sized by it.  FP8: E4M3 codes, the
// product as kind::f8f6f4 into an f32 accumulator ('量化压缩实战' §3.6).
template <int TMAX, bool FP8>
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
  float* xo_s = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + 256);  // [NT][XO_CHUNK]
  int32_t* idx_s = reinterpret_cast<int32_t*>(xo_s + NT * XO_CHUNK);          // [XO_CHUNK]
  int32_t* slot_s = idx_s + XO_CHUNK;                                          // [XO_CHUNK]

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int row0 = blockIdx.x * p.CH * p.H;  // first output row of this CTA
  const int units = p.CH * p.NU;             // unit i: chunk i / NU, k-blocks KPB * (i % NU) ...

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
  pdl_launch_dependents();  // the next call's kernels may launch

  auto stage_a = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };
  // Bytes one stage receives: KPB k-blocks of H weight rows and of 16 code
  // rows (rows or k-blocks past the tensors' ends arrive as zeros and count
  // as well).
  const uint32_t stage_tx = static_cast<uint32_t>((p.H + NT) * BK * p.KPB);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      auto load_a = [&](int i, int s) {
        const int kb = (i % p.NU) * p.KPB, r = row0 + (i / p.NU) * p.H;
        if (p.kpb3d)
          tma_load_3d_hint(stage_a(s), &tmap_w, &full[s], 0, r, kb, pol);
        else
          tma_load_2d_hint(stage_a(s), &tmap_w, &full[s], kb * BK, r, pol);
      };
      auto load_b = [&](int i, int s) {
        const int kb = (i % p.NU) * p.KPB;
        if (p.kpb3d)
          tma_load_3d(stage_b(s), &tmap_x, &full[s], 0, 0, kb);
        else
          tma_load_2d(stage_b(s), &tmap_x, &full[s], kb * BK, 0);
      };
      // The weights do not depend on earlier kernels: the first PRE stages
      // are requested before waiting for them, their activation codes right
      // after.
      const int pre = units < PRE ? units : PRE;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], stage_tx);
        load_a(i, i);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) load_b(i, i);
      int issued = pre;
      for (int i = pre; i < units; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, p.wait_ns, kErrTimeoutProducer)) break;
        mbar_arrive_expect_tx(&full[s], stage_tx);
        load_a(i, s);
        load_b(i, s);
        ++issued;
      }
      // Leave no copy in flight: wait for the last loads of every stage.
      for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.wait_ns, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_codes<FP8>(BM, NT);
      int i = 0;
      bool ok = true;
      for (int c = 0; c < p.CH && ok; ++c) {
        const int buf = c & 1;
        if (c >= 2) {
          ok = mbar_wait(&tempty[buf], ((c >> 1) - 1) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * NT);
        for (int ku = 0; ku < p.NU; ++ku, ++i) {
          const int s = i % STAGES;
          ok = mbar_wait(&full[s], (i / STAGES) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          const int nkb = min(p.KPB, p.KB - ku * p.KPB);  // k-blocks of this stage inside K
          for (int j = 0; j < nkb; ++j) {
            // Tile j of the stage: H rows (a multiple of 8, so the tile stays
            // aligned to the 1024-byte swizzle pattern) of 128 bytes.
            const uint32_t a0 = smem_addr(stage_a(s)) + static_cast<uint32_t>(j * p.H * BK);
            const uint32_t b0 = smem_addr(stage_b(s)) + static_cast<uint32_t>(j * B_TILE);
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_codes<FP8>(d, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc,
                             (ku > 0 || j > 0 || k > 0) ? 1u : 0u);
          }
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
    const int row = q * 32 + lane;           // chunk row = TMEM lane
    const int etid = threadIdx.x - 64;       // 0..127
    const int nO = load_count(p.n_out);
    const int T = p.T;
    if (p.n_miss && blockIdx.x == 0) {  // the misses, counted by the 128 epilogue threads
      __shared__ int miss_s;
      if (etid == 0) miss_s = 0;
      named_barrier(1, 128);
      int miss = 0;
      for (int j = etid; j < nO; j += 128) miss += p.slot[p.idx[j]] < 0 ? 1 : 0;
      miss = __reduce_add_sync(0xffffffffu, miss);
      if (lane == 0) atomicAdd(&miss_s, miss);
      named_barrier(1, 128);
      if (etid == 0) *p.n_miss = miss_s;
    }
    float sxr[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) sxr[t] = (p.Y && t < T) ? p.sx[t] : 0.0f;
    for (int c = 0; c < p.CH; ++c) {
      // This row's output channel; lanes past the chunk's H rows hold none.
      const int n = row < p.H ? row0 + c * p.H + row : p.N;
      // The outlier product does not depend on the int8 accumulator: it is
      // computed while the chunk's weights stream.
      float yo[TMAX];
      outlier_products<TMAX>(p, nO, n, etid, xo_s, idx_s, slot_s, yo);
      const int buf = c & 1;
      // All 128 epilogue threads agree on the outcome before going on, so a
      // timeout can never leave some of them at a named barrier.
      const bool ok = mbar_wait(&tfull[buf], (c >> 1) & 1, p.wait_ns, kErrTimeoutEpilogue);
      if (!named_barrier_and(2, 128, ok)) break;
      __syncwarp();
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * NT), r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (n < p.N) {
        const float swn = p.Y ? p.sw[n] : 0.0f;
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          if (t < T) {
            const float y = acc_value<FP8>(r[t]) * sxr[t] * swn + yo[t];
            if (p.Y) p.Y[static_cast<int64_t>(t) * p.N + n] = __half_as_ushort(__float2half_rn(y));
            if (p.acc_out) p.acc_out[static_cast<int64_t>(t) * p.N + n] = static_cast<int32_t>(r[t]);
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
