// gemm_kernel.cuh -- prefill-shaped LLM.int8() matmul on the 5th-generation
// tensor cores: gemm_pair_kernel (further below) for T > 128, persistent 2-CTA
// clusters with tcgen05 cta_group::2; gemm_kernel for 17 <= T <= 128.
//
// Both compute tiles of Y = X * W^T; in gemm_kernel one CTA takes a BM x BN
// tile:
//   acc = Xq[m-tile, :] * Wq[n-tile, :]^T     tcgen05.mma kind::i8 -> int32 TMEM
//   yo  = Xo[m-tile, :] * Wo[n-tile, :]^T     tcgen05.mma kind::f16 -> fp32 TMEM
//   Y   = fp16( acc * sx[t] * sw[n] + yo )    epilogue (tcgen05.ld -> registers)
// where Xo / Wo are the outlier columns of X / W gathered into K-major fp16
// buffers, |O| rounded up to 64 with zeros ('LLM quantization, part 2'
// (hncyxsy.com) §2.1: outlier sub-matrices in fp16, the rest in int8, results
// added; '三、模型量化' (lowentro.cn) Q2/Q4: r' = s*q on both operands).
// |O| is read from device memory, so the host never waits for it.
//
// FP8 (template flag): the same kernels for E4M3 codes ('量化压缩实战' §3.6),
// the 8-bit product as tcgen05.mma kind::f8f6f4 into an f32 accumulator.
//
// Operands arrive by TMA (128-byte swizzle, one 128-byte K row per box row)
// into a STAGES-deep ring; warp 0 issues the copies, warp 1 issues the MMAs
// and owns TMEM, warps 2-5 run the epilogue.  Every mbarrier wait is bounded.
#pragma once
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace llmint8 {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                       // bytes of K per stage (128 int8 / 64 fp16)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;              // 16 KiB
constexpr int B_BYTES = BN * BK;              // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;                // int32 acc [0, BN) + fp32 yo [BN, 2 BN)
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256 + BN * 4;  // + barriers, + sw of the tile

struct Params {
  int T, N, K;
  int KB;            // int8 k-blocks = ceil(K / BK)
  int num_m;         // M tiles: ceil(T / BM), or ceil(T / (2 BM)) for the CTA-pair kernel
  int num_tiles;     // CTA-pair kernel: num_m * ceil(N / bn)
  int num_pairs;     // CTA-pair kernel: clusters in the grid
  int y_tma;         // CTA-pair kernel: 1 = Y written by TMA stores (N % 8 == 0)
  int bn;            // CTA-pair kernel: tile columns (128, 192 or 256)
  const float* sx;
  const float* sw;
  const int32_t* n_out;
  uint16_t* Y;
  int32_t* acc_out;  // optional int32 [T][N] (FP8: the f32 accumulator's bits)
  uint64_t wait_ns;
};

// Epilogue of one CTA's 128 x BN output block (rows m0.., columns n0..), run
// by the 4 epilogue warps (etid = 0..127); warp quadrant q reads TMEM lanes
// 32q..32q+31 = rows m0+32q+lane:
//   Y[row, n] = fp16( acc * sx[row] * sw[n] + yo )
// acc: int32 TMEM columns [0, BN); yo: fp32 columns [BN, 2 BN), read only when
// there are outlier columns.  The tile's sw values are staged in shared memory
// (sw_s, BN floats) while the MMAs still run, so that draining TMEM waits on
// no global load; then it waits (bounded) for `tfull`.
template <bool FP8>
__device__ __forceinline__ void epilogue_rows(const Params& p, uint32_t tmem_base, int q, int lane, int etid,
                                              int m0, int n0, uint64_t* tfull, float* sw_s) {
  for (int j = etid; j < BN; j += 128) sw_s[j] = (p.Y && n0 + j < p.N) ? __ldg(p.sw + n0 + j) : 0.0f;
  named_barrier(1, 128);
  const int row = m0 + q * 32 + lane;
  const int nO = load_count(p.n_out);
  const bool has_o = nO > 0;
  const float sxr = (p.Y && row < p.T) ? p.sx[row] : 0.0f;
  const bool ok = mbar_wait(tfull, 0, p.wait_ns, kErrTimeoutEpilogue);
  if (!__all_sync(0xffffffffu, ok)) return;  // warp-uniform before the .sync.aligned loads
  tc_fence_after();
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
  const bool vec_ok = (p.N % 8) == 0;
  for (int cc = 0; cc < BN; cc += 32) {
    if (n0 + cc >= p.N) break;
    uint32_t ra[32], rb[32];
    tmem_ld32(lane_addr + cc, ra);
    if (has_o) tmem_ld32(lane_addr + BN + cc, rb);
    tmem_ld_wait();
    if (row < p.T) {
      const int nbase = n0 + cc;
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float y[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float swn = sw_s[cc + j + h];
          y[h] = acc_value<FP8>(ra[j + h]) * sxr * swn + (has_o ? __uint_as_float(rb[j + h]) : 0.0f);
        }
        packed[j >> 1] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[0]))) |
                         (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[1]))) << 16);
      }
      if (p.Y) {
        uint16_t* yrow = p.Y + static_cast<int64_t>(row) * p.N + nbase;
        if (vec_ok && nbase + 32 <= p.N) {
          uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nbase + j < p.N) yrow[j] = static_cast<uint16_t>(packed[j >> 1] >> ((j & 1) * 16));
        }
      }
      if (p.acc_out) {
        int32_t* arow = p.acc_out + static_cast<int64_t>(row) * p.N + nbase;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (nbase + j < p.N) arow[j] = static_cast<int32_t>(ra[j]);
      }
    }
  }
}

template <bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_xq, const __grid_constant__ CUtensorMap tmap_wq,
                const __grid_constant__ CUtensorMap tmap_xo, const __grid_constant__ CUtensorMap tmap_wo,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* done = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int m_blk = blockIdx.x % p.num_m;
  const int n_blk = blockIdx.x / p.num_m;
  const int m0 = m_blk * BM, n0 = n_blk * BN;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_xq);
    prefetch_tensormap(&tmap_wq);
    prefetch_tensormap(&tmap_xo);
    prefetch_tensormap(&tmap_wo);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
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
  pdl_launch_dependents();  // the next call's kernels may launch and prefetch

  auto stage_a = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int KB = p.KB;
      const int pre = KB < STAGES ? KB : STAGES;
      // Wq does not depend on the preceding kernels: prefetch its first
      // stages before waiting for them.
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], STAGE_BYTES);
        tma_load_2d(stage_b(i), &tmap_wq, &full[i], i * BK, n0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) tma_load_2d(stage_a(i), &tmap_xq, &full[i], i * BK, m0);
      const int nO = load_count(p.n_out);
      const int OB = (nO + 63) / 64;
      const int total = KB + OB;
      int issued = pre;
      for (int i = pre; i < total; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, p.wait_ns, kErrTimeoutProducer)) break;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        if (i < KB) {
          tma_load_2d(stage_a(s), &tmap_xq, &full[s], i * BK, m0);
          tma_load_2d(stage_b(s), &tmap_wq, &full[s], i * BK, n0);
        } else {
          const int jb = i - KB;
          tma_load_2d(stage_a(s), &tmap_xo, &full[s], jb * 64, m0);
          tma_load_2d(stage_b(s), &tmap_wo, &full[s], jb * 64, n0);
        }
        ++issued;
      }
      for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.wait_ns, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      pdl_wait();
      const int nO = load_count(p.n_out);
      const int OB = (nO + 63) / 64;
      const int total = p.KB + OB;
      constexpr uint32_t idesc_i = idesc_codes<FP8>(BM, BN);
      constexpr uint32_t idesc_h = idesc_f16_f32(BM, BN);
      const uint32_t d_acc = tmem_base;
      const uint32_t d_yo = tmem_base + BN;
      bool ok = true;
      for (int i = 0; i < total; ++i) {
        const int s = i % STAGES;
        ok = mbar_wait(&full[s], (i / STAGES) & 1, p.wait_ns, kErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_addr(stage_a(s));
        const uint32_t b0 = smem_addr(stage_b(s));
        if (i < p.KB) {
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_codes<FP8>(d_acc, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc_i,
                           (i > 0 || k > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_f16(d_yo, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc_h,
                    (i > p.KB || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(tfull);
      mma_commit(done);
      mbar_wait(done, 0, p.wait_ns, kErrTimeoutMma);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    epilogue_rows<FP8>(p, tmem_base, warp & 3, lane, static_cast<int>(threadIdx.x) - 64, m0, n0, tfull,
                       reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + 256));
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


// ---------------------------------------------------------------------------
// CTA-pair kernel for T > BM.  A 2-CTA cluster computes 256 x bn tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = bn, bn = 128, 192 or 256, chosen by
// the host so that the tiles spread evenly over the resident pairs): CTA r of
// the pair loads rows m0 + 128 r .. +127 of Xq (A) and rows
// n0 + bn/2 r .. + bn/2 - 1 of Wq (its half of B), so at bn = 256 each SM
// stages 32 KiB per k-block for its 128 x 256 x 128 share of the products (a
// single CTA would stage 48 KiB).  The even CTA's thread
// issues the MMAs; both CTAs' copies complete on the even CTA's `full`
// barriers and each MMA commit arrives on the `empty` / `tfull` barriers of
// both CTAs.  TMEM (512 columns in each CTA) holds that CTA's 128 rows: int32
// acc in [0, bn), fp32 yo in [bn, 2 bn).
//
// Persistent: the grid holds as many pairs as fit on the GPU at once (the
// launch is 2-CTA clusters along x), and pair c takes tiles c, c + pairs, ...
// The copies of the next tile start while the epilogue drains the current
// one; its first MMA waits until both CTAs have read their accumulators out
// (`tempty`, one arrival per epilogue warp of both CTAs, on the even CTA).
// The epilogue runs in two sets of 4 warps; set s drains the 64-column groups
// g = s, s + 2, ... of the tile 32 columns at a time and writes Y through its
// own shared-memory staging box (128 x 64 fp16) and a TMA store when N is a
// multiple of 8, otherwise with plain stores.
// ---------------------------------------------------------------------------
constexpr int P_STAGES = 6;
constexpr int P_THREADS = 320;                       // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int P_EPI_WARPS = 8;                       // two sets of 4: one warp per TMEM lane quadrant each
constexpr int P_A_BYTES = BM * BK;                   // 16 KiB: this CTA's 128 rows of Xq
constexpr int P_B_BYTES = (BN / 2) * BK;             // 16 KiB: this CTA's half of the Wq tile
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_YCOLS = 64;                          // Y columns per store box (128 bytes)
constexpr int P_YBUF_BYTES = BM * P_YCOLS * 2;       // 16 KiB
constexpr int P_SMEM_BYTES = 1024 + P_STAGES * P_STAGE_BYTES + 2 * P_YBUF_BYTES + BN * 4 + 256;
static_assert(P_SMEM_BYTES <= 232448, "shared memory per CTA");

__device__ __forceinline__ void pair_tile(const Params& p, int tile, uint32_t rank, int* m0, int* n0) {
  *m0 = (tile % p.num_m) * (2 * BM) + static_cast<int>(rank) * BM;  // this CTA's rows of X / Y
  *n0 = (tile / p.num_m) * p.bn;                                    // the pair's columns of Y
}

// 32 outputs of one row: y = fp16(acc * sxr * sw + yo), packed in pairs.
template <bool FP8>
__device__ __forceinline__ void dequant32(const uint32_t (&ra)[32], const uint32_t (&rb)[32], bool has_o, float sxr,
                                          const float* sw32, uint32_t (&packed)[16]) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float y[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      y[h] = acc_value<FP8>(ra[j + h]) * sxr * sw32[j + h] + (has_o ? __uint_as_float(rb[j + h]) : 0.0f);
    const __half2 h2 = __floats2half2_rn(y[0], y[1]);  // y[0] in the low half
    packed[j >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
  }
}

template <bool FP8>
__global__ void __launch_bounds__(P_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_xq, const __grid_constant__ CUtensorMap tmap_wq,
                     const __grid_constant__ CUtensorMap tmap_xo, const __grid_constant__ CUtensorMap tmap_wo,
                     const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ybuf = smem + P_STAGES * P_STAGE_BYTES;                 // [2][128 rows][128 B], 1024-aligned
  float* sw_s = reinterpret_cast<float*>(ybuf + 2 * P_YBUF_BYTES);  // [BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(sw_s + BN);          // used in the even CTA
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 1;                                     // used in the even CTA
  uint64_t* done = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const int pair = blockIdx.x >> 1;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_xq);
    prefetch_tensormap(&tmap_wq);
    prefetch_tensormap(&tmap_xo);
    prefetch_tensormap(&tmap_wo);
    if (p.y_tma) prefetch_tensormap(&tmap_y);
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * P_EPI_WARPS);  // every epilogue warp of both CTAs
    mbar_init(done, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);  // collective with the other CTA's warp 1
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any copy or commit reaches them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();

  auto stage_a = [&](int s) { return smem + s * P_STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * P_STAGE_BYTES + P_A_BYTES; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0 && pair < p.num_tiles) {
      const bool lead = rank == 0;
      const int KB = p.KB;
      auto full_of = [&](int s) { return map_shared_rank(&full[s], 0); };
      int m0, n0;
      pair_tile(p, pair, rank, &m0, &n0);
      // Wq does not depend on the preceding kernels: the first tile's first
      // stages are requested before waiting for them.  The even CTA arms its
      // barrier for both CTAs' bytes; the odd CTA's copies may land before
      // that (the phase still waits for the arrival).
      const int pre = KB < P_STAGES ? KB : P_STAGES;
      const uint32_t stage_tx = 2u * static_cast<uint32_t>(P_A_BYTES + (p.bn / 2) * BK);  // both CTAs
      for (int i = 0; i < pre; ++i) {
        if (lead) mbar_arrive_expect_tx(&full[i], stage_tx);
        tma_load_2d_pair(stage_b(i), &tmap_wq, full_of(i), i * BK, n0 + static_cast<int>(rank) * (p.bn / 2));
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) tma_load_2d_pair(stage_a(i), &tmap_xq, full_of(i), i * BK, m0);
      const int total = KB + (load_count(p.n_out) + 63) / 64;
      int it = pre;  // k-blocks issued so far, over all tiles: stage it % P_STAGES
      int kb = pre;
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += p.num_pairs, kb = 0) {
        pair_tile(p, tile, rank, &m0, &n0);
        const int nb0 = n0 + static_cast<int>(rank) * (p.bn / 2);
        for (; kb < total; ++kb, ++it) {
          const int s = it % P_STAGES;
          if (it >= P_STAGES &&
              !mbar_wait(&empty[s], ((it / P_STAGES) & 1) ^ 1, p.wait_ns, kErrTimeoutProducer)) {
            ok = false;
            break;
          }
          if (lead) mbar_arrive_expect_tx(&full[s], stage_tx);
          if (kb < KB) {
            tma_load_2d_pair(stage_a(s), &tmap_xq, full_of(s), kb * BK, m0);
            tma_load_2d_pair(stage_b(s), &tmap_wq, full_of(s), kb * BK, nb0);
          } else {
            const int jb = kb - KB;
            tma_load_2d_pair(stage_a(s), &tmap_xo, full_of(s), jb * 64, m0);
            tma_load_2d_pair(stage_b(s), &tmap_wo, full_of(s), jb * 64, nb0);
          }
        }
      }
      // Every copy has landed once the MMAs that read it completed: the
      // `done` commit covers that on the normal path.
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      pdl_wait();
      const int total = p.KB + (load_count(p.n_out) + 63) / 64;
      const uint32_t idesc_i = idesc_codes<FP8>(2 * BM, p.bn);
      const uint32_t idesc_h = idesc_f16_f32(2 * BM, p.bn);
      const uint32_t d_acc = tmem_base;
      const uint32_t d_yo = tmem_base + static_cast<uint32_t>(p.bn);
      bool ok = true;
      int it = 0, tc = 0;
      for (int tile = pair; ok && tile < p.num_tiles; tile += p.num_pairs, ++tc) {
        if (tc > 0) {  // both CTAs have drained the previous tile's accumulators
          ok = mbar_wait_cluster(tempty, (tc - 1) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
        }
        tc_fence_after();
        for (int kb = 0; kb < total; ++kb, ++it) {
          const int s = it % P_STAGES;
          ok = mbar_wait(&full[s], (it / P_STAGES) & 1, p.wait_ns, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = smem_addr(stage_a(s));
          const uint32_t b0 = smem_addr(stage_b(s));
          if (kb < p.KB) {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_codes_pair<FP8>(d_acc, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32),
                                  idesc_i, (kb > 0 || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_f16_pair(d_yo, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc_h,
                           (kb > p.KB || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[s], 0x3);
        }
        if (ok) mma_commit_pair(tfull, 0x3);
      }
      mma_commit_pair(done, 0x3);
    }
    // Both CTAs: the pair's MMAs are complete before TMEM is released.
    if (lane == 0) mbar_wait(done, 0, p.wait_ns, kErrTimeoutMma);
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int set = (warp - 2) >> 2;                           // 0 or 1
    const int q = warp & 3;                                    // TMEM lane quadrant of this warp
    const int etid = static_cast<int>(threadIdx.x) - 64;       // 0..255
    const int stid = etid - 128 * set;                         // 0..127 within the set
    const uint32_t set_bar = 1u + 2u * static_cast<uint32_t>(set);  // named barriers 1 / 3
    const int r_loc = q * 32 + lane;                           // row within this CTA's 128
    uint8_t* yb = ybuf + set * P_YBUF_BYTES;                   // this set's staging box
    pdl_wait();
    const bool has_o = load_count(p.n_out) > 0;
    const uint32_t tempty_lead = map_shared_rank(tempty, 0);
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t yo_col = static_cast<uint32_t>(p.bn);
    const bool vec_ok = (p.N % 8) == 0;
    const int groups = p.bn / P_YCOLS;
    int tc = 0;
    for (int tile = pair; tile < p.num_tiles; tile += p.num_pairs, ++tc) {
      int m0, n0;
      pair_tile(p, tile, rank, &m0, &n0);
      named_barrier(5, 2 * 128);  // both sets are past the previous tile's reads of sw_s
      for (int j = etid; j < p.bn; j += 2 * 128)
        sw_s[j] = (p.Y && n0 + j < p.N) ? __ldg(p.sw + n0 + j) : 0.0f;
      named_barrier(5, 2 * 128);
      const int row = m0 + r_loc;
      const float sxr = (p.Y && row < p.T) ? p.sx[row] : 0.0f;
      const bool okw = mbar_wait(tfull, tc & 1, p.wait_ns, kErrTimeoutEpilogue);
      if (!named_barrier_and(2, 2 * 128, okw)) break;  // all 256 epilogue threads leave together
      tc_fence_after();
      for (int g = set; g < groups; g += 2) {
        const bool last_group = g + 2 >= groups;
        const bool active = n0 + g * P_YCOLS < p.N;        // uniform
        const bool staged = p.y_tma && active && m0 < p.T;  // uniform: a store with rows to write
        // The group's 64 columns of both accumulators go to registers first,
        // so that after the last group TMEM is released before any wait on a
        // store.
        uint32_t ra0[32], rb0[32], ra1[32], rb1[32];
        const uint32_t cg = static_cast<uint32_t>(g * P_YCOLS);
        tmem_ld32(lane_addr + cg, ra0);
        tmem_ld32(lane_addr + cg + 32, ra1);
        if (has_o) {
          tmem_ld32(lane_addr + yo_col + cg, rb0);
          tmem_ld32(lane_addr + yo_col + cg + 32, rb1);
        }
        tmem_ld_wait();
        tmem_regs_ready(ra0);
        tmem_regs_ready(ra1);
        tmem_regs_ready(rb0);
        tmem_regs_ready(rb1);
        if (last_group) {
          // This warp has read all of its accumulators: the next tile's MMAs
          // may overwrite them.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_lead);
        }
        if (!active) continue;
        if (staged) {
          if (stid == 0) bulk_wait_group_read<0>();  // this set's previous store is done with the box
          named_barrier(set_bar, 128);
        }
        // 32 columns starting at c0 = g * 64 + 32 h.
        auto half = [&](int h, const uint32_t (&ra)[32], const uint32_t (&rb)[32]) {
          const int c0 = g * P_YCOLS + h * 32;
          uint32_t packed[16];
          dequant32<FP8>(ra, rb, has_o, sxr, sw_s + c0, packed);
          if (staged) {
            // 128-byte swizzle, as the store's tensor map expects: 16-byte
            // chunk c of a row sits at chunk c ^ (row % 8).
            uint8_t* rowp = yb + r_loc * 128;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int c = h * 4 + v;
              *reinterpret_cast<uint4*>(rowp + ((c ^ (r_loc & 7)) << 4)) =
                  make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            }
          } else if (!p.y_tma && p.Y && row < p.T) {
            const int nbase = n0 + c0;
            uint16_t* yrow = p.Y + static_cast<int64_t>(row) * p.N + nbase;
            if (vec_ok && nbase + 32 <= p.N) {
              uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (nbase + j < p.N) yrow[j] = static_cast<uint16_t>(packed[j >> 1] >> ((j & 1) * 16));
            }
          }
          if (p.acc_out && row < p.T) {
            const int nbase = n0 + c0;
            int32_t* arow = p.acc_out + static_cast<int64_t>(row) * p.N + nbase;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nbase + j < p.N) arow[j] = static_cast<int32_t>(ra[j]);
          }
        };
        half(0, ra0, rb0);
        half(1, ra1, rb1);
        if (staged) {
          fence_proxy_async_shared();  // the staging writes, before the async-proxy store reads them
          named_barrier(set_bar, 128);
          if (stid == 0) {
            tma_store_2d(&tmap_y, yb, n0 + g * P_YCOLS, m0);
            bulk_commit_group();
          }
        }
      }
    }
    if (stid == 0) bulk_wait_group<0>();  // Y is written before the CTA ends
  }

  __syncwarp();
  tc_fence_before();
  // Neither CTA leaves while the other may still signal its barriers or, after
  // a timeout, copies of the pair may still be landing.
  if (threadIdx.x == 0 && ld_error_word() != 0) sleep_ns_bounded(20000);
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace llmint8
