// gemm_kernel.cuh -- prefill-shaped LLM.int8() matmul on the 5th-generation
// tensor cores.
//
// One CTA computes a BM x BN tile of Y = X * W^T:
//   acc = Xq[m-tile, :] * Wq[n-tile, :]^T     tcgen05.mma kind::i8 -> int32 TMEM
//   yo  = Xo[m-tile, :] * Wo[n-tile, :]^T     tcgen05.mma kind::f16 -> fp32 TMEM
//   Y   = fp16( acc * sx[t] * sw[n] + yo )    epilogue (tcgen05.ld -> registers)
// where Xo / Wo are the outlier columns of X / W gathered into K-major fp16
// buffers, |O| rounded up to 64 with zeros ('LLM quantization, part 2'
// (hncyxsy.com) §2.1: outlier sub-matrices in fp16, the rest in int8, results
// added; '三、模型量化' (lowentro.cn) Q2/Q4: r' = s*q on both operands).
// |O| is read from device memory, so the host never waits for it.
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
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;

struct Params {
  int T, N, K;
  int KB;            // int8 k-blocks = ceil(K / BK)
  int num_m;         // ceil(T / BM)
  const float* sx;
  const float* sw;
  const int32_t* n_out;
  uint16_t* Y;
  int32_t* acc_out;  // optional int32 [T][N]
  uint64_t wait_ns;
};

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
      const int nO = *p.n_out;
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
      const int nO = *p.n_out;
      const int OB = (nO + 63) / 64;
      const int total = p.KB + OB;
      constexpr uint32_t idesc_i = idesc_i8_s32(BM, BN);
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
            mma_i8(d_acc, make_sdesc_k_sw128(a0 + k * 32), make_sdesc_k_sw128(b0 + k * 32), idesc_i,
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
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    const int nO = *p.n_out;
    const bool has_o = nO > 0;
    const float sxr = row < p.T ? p.sx[row] : 0.0f;
    const bool ok = mbar_wait(tfull, 0, p.wait_ns, kErrTimeoutEpilogue);
    if (__all_sync(0xffffffffu, ok)) {  // warp-uniform before the .sync.aligned loads
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
              const int n = nbase + j + h;
              const float swn = n < p.N ? __ldg(p.sw + n) : 0.0f;
              y[h] = static_cast<float>(static_cast<int32_t>(ra[j + h])) * sxr * swn +
                     (has_o ? __uint_as_float(rb[j + h]) : 0.0f);
            }
            packed[j >> 1] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[0]))) |
                             (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(y[1]))) << 16);
          }
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
          if (p.acc_out) {
            int32_t* arow = p.acc_out + static_cast<int64_t>(row) * p.N + nbase;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nbase + j < p.N) arow[j] = static_cast<int32_t>(ra[j]);
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

}  // namespace gemm
}  // namespace llmint8
