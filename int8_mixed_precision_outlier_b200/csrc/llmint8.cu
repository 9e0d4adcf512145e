// llmint8.cu -- the C ABI (include/llmint8.h) over the sm_100a kernels.
//
// One translation unit: the kernels live in the .cuh files included below so
// that the per-device error word is a single __device__ symbol without
// relocatable device code.  Host code here only validates arguments, lays out
// the caller's workspace, encodes TMA tensor maps and launches; every step of
// the method runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "llmint8.h"

#include "gemm_kernel.cuh"
#include "gemv_kernel.cuh"
#include "prep_kernels.cuh"
#include "sm100.cuh"
#include "smooth_kernels.cuh"

namespace llmint8 {
namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = 65536;         // decode prep keeps K/8 mask bytes in shared memory
constexpr int64_t kMaxInt32Sum = 133143; // K * 127 * 127 < 2^31

std::atomic<uint64_t> g_wait_ns{2000000000ull};

// ------------------------------------------------------------ device facts
struct DeviceInfo {
  std::once_flag once;
  int status = LLMINT8_OK;
  int num_sms = 0;
  int max_pairs = 0;  // 2-CTA clusters of gemm_pair_kernel resident at once
};
DeviceInfo g_dev[kMaxDevices];

// Shared-memory limits and carveouts of every kernel of one code format.
template <bool FP8>
cudaError_t set_attributes() {
  cudaError_t e = cudaSuccess;
  auto big = [&](auto kern, int bytes) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  };
  // The decode prep kernel runs next to GEMV CTAs (its own call's, which
  // launch early, and the previous call's): with the largest shared memory
  // carveout on its SMs, a GEMV CTA fits beside it instead of waiting for it.
  auto carve = [&](auto kern) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  };
  big(gemm::gemm_kernel<FP8>, gemm::SMEM_BYTES);
  big(gemm::gemm_pair_kernel<FP8>, gemm::P_SMEM_BYTES);
  big(gemv::gemv_kernel<1, FP8>, gemv::SMEM_BYTES);
  big(gemv::gemv_kernel<2, FP8>, gemv::SMEM_BYTES);
  big(gemv::gemv_kernel<4, FP8>, gemv::SMEM_BYTES);
  big(gemv::gemv_kernel<8, FP8>, gemv::SMEM_BYTES);
  big(gemv::gemv_kernel<16, FP8>, gemv::SMEM_BYTES);
  carve(decode_prep_kernel<1, FP8>);
  carve(decode_prep_kernel<2, FP8>);
  carve(decode_prep_kernel<4, FP8>);
  carve(decode_prep_kernel<8, FP8>);
  carve(decode_prep_kernel<16, FP8>);
  return e;
}

int device_info(int* num_sms, int* max_pairs = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLMINT8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LLMINT8_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&]() {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.status = LLMINT8_ERR_CUDA;
      return;
    }
    if (major != 10 || minor != 0) {
      d.status = LLMINT8_ERR_UNSUPPORTED_ARCH;
      return;
    }
    if (set_attributes<false>() != cudaSuccess || set_attributes<true>() != cudaSuccess) {
      d.status = LLMINT8_ERR_CUDA;
      return;
    }
    d.num_sms = sms;
    // How many pairs the persistent GEMM can keep resident (GPCs with an odd
    // number of usable SMs leave one idle).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(gemm::P_THREADS);
    cfg.dynamicSmemBytes = gemm::P_SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm::gemm_pair_kernel<false>, &cfg) != cudaSuccess ||
        clusters < 1) {
      cudaGetLastError();
      clusters = sms / 2;
    }
    d.max_pairs = clusters;
  });
  if (num_sms) *num_sms = d.num_sms;
  if (max_pairs) *max_pairs = d.max_pairs;
  return d.status;
}

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer][inner], rows `row_bytes` apart, read in boxes
// of box_outer rows x box_inner elements.  With the 128-byte swizzle a box row
// is exactly 128 bytes; without swizzle it lands in shared memory row-major.
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Int8 matrix [rows][K] (K % 128 == 0) seen as 3-D: 128 bytes of a k-block,
// row, k-block; a box of `box_rows` rows x `kpb` k-blocks lands as kpb
// consecutive 128-byte-swizzled tiles of box_rows x 128 bytes, and reads
// kpb * 128 contiguous bytes of every row.
bool encode_kblocks_3d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows,
                       uint32_t kpb) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || K % 128 != 0) return false;
  const cuuint64_t dims[3] = {128, rows, K / 128};
  const cuuint64_t strides[2] = {K, 128};
  const cuuint32_t box[3] = {128, box_rows, kpb};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ workspace layout
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  int path = 0;
  int Kw = 0, rows_per_cta = 0, ldo = 0, nstrips = 0;
  size_t rowmax = 0, flags = 0, idx = 0, n_out = 0, sx = 0, xq = 0, xo = 0, wo = 0, total = 0;
};

bool make_layout(int64_t T, int64_t N, int64_t K, int path, Layout* L) {
  if (T < 0 || N < 0 || K < 16 || K % 16 != 0 || K > kMaxK) return false;
  if (path == LLMINT8_PATH_AUTO) path = T <= LLMINT8_GEMV_MAX_T ? LLMINT8_PATH_GEMV : LLMINT8_PATH_GEMM;
  if (path == LLMINT8_PATH_GEMV && T > LLMINT8_GEMV_MAX_T) return false;
  if (path != LLMINT8_PATH_GEMV && path != LLMINT8_PATH_GEMM) return false;
  L->path = path;
  L->Kw = static_cast<int>((K + 31) / 32);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + (bytes ? bytes : 1), 256);
    return at;
  };
  if (path == LLMINT8_PATH_GEMV) {
    L->idx = take(sizeof(int32_t) * K);
    L->n_out = take(sizeof(int32_t));
    L->sx = take(sizeof(float) * LLMINT8_GEMV_MAX_T);
    L->xq = take(static_cast<size_t>(LLMINT8_GEMV_MAX_T) * K);
    // decode_workspace_bytes() states the same sum as a constant expression
  } else {
    L->rows_per_cta = static_cast<int>(T > 0 ? (T + kDetectCluster - 1) / kDetectCluster : 1);
    L->nstrips = static_cast<int>((K + kDetectCols - 1) / kDetectCols);
    L->ldo = static_cast<int>((K + 63) / 64 * 64);
    L->flags = take(sizeof(uint32_t) * L->Kw);
    L->rowmax = take(sizeof(float) * static_cast<size_t>(T) * L->nstrips);
    L->idx = take(sizeof(int32_t) * K);
    L->n_out = take(sizeof(int32_t));
    L->sx = take(sizeof(float) * static_cast<size_t>(T));
    L->xq = take(static_cast<size_t>(T) * K);
    L->xo = take(sizeof(uint16_t) * static_cast<size_t>(T) * L->ldo);
    L->wo = take(sizeof(uint16_t) * static_cast<size_t>(N) * L->ldo);
  }
  L->total = off;
  return true;
}

// Bytes of the decode path's workspace for K columns (any T <= 16, any N):
// the outlier list, its length, 16 row scales and 16 rows of codes, each
// region 256-byte aligned, as make_layout lays them out.
constexpr size_t decode_workspace_bytes(int64_t K) {
  return ((sizeof(int32_t) * static_cast<size_t>(K) + 255) / 256 * 256) + 256 +
         ((sizeof(float) * LLMINT8_GEMV_MAX_T + 255) / 256 * 256) +
         ((static_cast<size_t>(LLMINT8_GEMV_MAX_T) * static_cast<size_t>(K) + 255) / 256 * 256);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------ launches
// Launch with programmatic stream serialization (when `pdl`) and, when
// `cluster` > 1, thread-block clusters of that many CTAs along x.
template <typename... Exp, typename... Act>
cudaError_t launch_ex(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      int cluster, Act&&... args) {
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

template <typename... Exp, typename... Act>
cudaError_t launch(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                   Act&&... args) {
  return launch_ex(kern, grid, block, smem, st, pdl, 1, std::forward<Act>(args)...);
}

struct Prep {
  // outputs of the activation stages (workspace or caller buffers)
  int8_t* xq;
  float* sx;
  int32_t* idx;
  int32_t* n_out;
};

// Activation stages.  Decode: one latency-oriented kernel.  Prefill: detection (one
// cluster of CTAs per column strip), then quantisation with the compaction and the
// gathers (the W gather only when W != nullptr, the store gather with a column store).
template <bool FP8>
int launch_prep(const Layout& L, const uint16_t* X, int T, int K, const uint16_t* W, int N, float tau,
                uint8_t* ws, const Prep& out, cudaStream_t st, const ColumnStore& cs = ColumnStore{}) {
  uint32_t* flags = reinterpret_cast<uint32_t*>(ws + L.flags);
  cudaError_t e;
  if (L.path == LLMINT8_PATH_GEMV) {
    auto k = T <= 1 ? decode_prep_kernel<1, FP8> : T <= 2 ? decode_prep_kernel<2, FP8>
           : T <= 4 ? decode_prep_kernel<4, FP8> : T <= 8 ? decode_prep_kernel<8, FP8> : decode_prep_kernel<16, FP8>;
    e = launch_ex(k, dim3(kDecodeCtas), dim3(kDecodeThreads), 0, st, true, kDecodeCtas, X, T, K, tau, out.xq,
                  out.sx, out.idx, out.n_out);
    return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
  }
  float* rowmax = reinterpret_cast<float*>(ws + L.rowmax);
  // up to 16 rows per thread (T <= 2048): the rows stay in registers between the two passes
  const int rpt = (L.rows_per_cta + 15) / 16;
  auto detect = rpt <= 4 ? detect_kernel<4> : rpt <= 16 ? detect_kernel<16> : detect_kernel<0>;
  e = launch_ex(detect, dim3(L.nstrips * kDetectCluster), dim3(kPrepThreads), 0, st, true, kDetectCluster, X, T, K,
                tau, L.rows_per_cta, flags, L.Kw, rowmax, L.nstrips);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  const int gather_ctas = W ? (N + kWoRowsPerCta - 1) / kWoRowsPerCta
                          : cs.slot ? (N + kStoreRowsPerCta - 1) / kStoreRowsPerCta : 0;
  e = launch(quant_gather_kernel<FP8>, dim3(gather_ctas + T), dim3(kQuantThreads), 8 * static_cast<size_t>(L.Kw),
             st, true, X, T, K, W, N, static_cast<const uint32_t*>(flags), L.Kw, static_cast<const float*>(rowmax),
             L.nstrips, out.idx, out.n_out, out.xq, out.sx, reinterpret_cast<uint16_t*>(ws + L.xo),
             reinterpret_cast<uint16_t*>(ws + L.wo), L.ldo, gather_ctas, cs);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

int check_common(const void* X, int64_t T, int64_t K, float threshold, const void* ws, size_t ws_bytes,
                 int path, Layout* L, int64_t N) {
  if (T < 0 || N < 0 || K < 16 || K > kMaxK || K > kMaxInt32Sum) return LLMINT8_ERR_INVALID_ARG;
  if (T > INT32_MAX || N > INT32_MAX) return LLMINT8_ERR_INVALID_ARG;
  if (std::isnan(threshold)) return LLMINT8_ERR_INVALID_ARG;
  if (path < LLMINT8_PATH_AUTO || path > LLMINT8_PATH_GEMM) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (!make_layout(T, N, K, path, L)) return LLMINT8_ERR_INVALID_ARG;
  if (T > 0 && (!X || !ws)) return LLMINT8_ERR_INVALID_ARG;
  if (T > 0 && (!aligned16(X) || !aligned16(ws))) return LLMINT8_ERR_ALIGNMENT;
  if (T > 0 && ws_bytes < L->total) return LLMINT8_ERR_WORKSPACE;
  return LLMINT8_OK;
}

struct Inspect {  // optional inspection outputs of llmint8_matmul_debug
  int32_t* acc = nullptr;
  int8_t* xq = nullptr;
  float* sx = nullptr;
  int32_t* idx = nullptr;
  int32_t* n = nullptr;
};

// Operands of one main-kernel launch (the GEMV or a GEMM).  For the plain
// int8 product of llmint8_int8_gemm_i32, n_out, Y and the fp operands are null:
// the kernels then take |O| = 0 and write only the int32 accumulator.
struct MainOps {
  const int8_t* xq = nullptr;     // activation codes [T][K]
  const float* sx = nullptr;      // row scales [T]
  const int32_t* idx = nullptr;   // outlier columns (decode path)
  const int32_t* n_out = nullptr; // |O| on the device
  const uint16_t* X = nullptr;    // fp16 activations (decode outlier products)
  const uint16_t* W = nullptr;    // fp16 weight (decode outlier products)
  const float* sw = nullptr;      // weight scales [N]
  uint16_t* Y = nullptr;          // fp16 output [T][N]
  int32_t* acc = nullptr;         // optional int32 output [T][N]
  const uint16_t* xo = nullptr;   // prefill: gathered outlier columns of X [T][ldo]
  const uint16_t* wo = nullptr;   // prefill: gathered outlier columns of W [N][ldo]
  int ldo = 0;
  const int32_t* slot = nullptr;  // decode with a column store (W null)
  const uint16_t* Wst = nullptr;
  const int8_t* Wqr = nullptr;
  int32_t* n_miss = nullptr;
};

// Encodes the main kernel's tensor maps (so that a failure launches nothing),
// runs `before()` (the call's activation-stage launches; it returns a status),
// then launches the main kernel `repeat` times, between `ev_begin` / `ev_end`
// when given.  `path` is LLMINT8_PATH_GEMV (T <= 16) or LLMINT8_PATH_GEMM.
template <bool FP8, typename Before>
int run_main(int path, int t, int n, int k, const int8_t* Wq, const MainOps& m, cudaStream_t st,
             Before before, cudaEvent_t ev_begin = nullptr, cudaEvent_t ev_end = nullptr, int repeat = 1) {
  int num_sms = 0, max_pairs = 0;
  int rc = device_info(&num_sms, &max_pairs);
  if (rc != LLMINT8_OK) return rc;
  const uint64_t wait_ns = g_wait_ns.load();

  if (path == LLMINT8_PATH_GEMV) {
    gemv::Params p;
    p.T = t;
    p.N = n;
    p.K = k;
    p.KB = (k + gemv::BK - 1) / gemv::BK;
    // Row slabs: every CTA takes CH chunks of H rows (a multiple of 8) over
    // all of K, about N / SMs rows in all, so the grid fills the SMs with
    // equal shares.  With K % 128 == 0 one copy brings KPB k-blocks of each
    // row (3-D tensor maps); otherwise one k-block (2-D maps, which zero the
    // ragged tail of K).
    const int per = (n + num_sms - 1) / num_sms;
    p.CH = (per + gemv::BM - 1) / gemv::BM;
    p.H = ((per + p.CH - 1) / p.CH + 7) / 8 * 8;
    const int grid = (n + p.CH * p.H - 1) / (p.CH * p.H);
    p.kpb3d = (k % gemv::BK) == 0 ? 1 : 0;
    p.KPB = p.kpb3d ? gemv::kpb_for_rows(p.H) : 1;
    p.NU = (p.KB + p.KPB - 1) / p.KPB;
    p.sx = m.sx;
    p.sw = m.sw;
    p.X = m.X;
    p.W = m.W;
    p.idx = m.idx;
    p.n_out = m.n_out;
    p.slot = m.slot;
    p.Wst = m.Wst;
    p.Wqr = m.Wqr;
    p.n_miss = m.n_miss;
    p.Y = m.Y;
    p.acc_out = m.acc;
    p.wait_ns = wait_ns;
    CUtensorMap tw, tx;
    const bool maps_ok =
        p.kpb3d ? encode_kblocks_3d(&tw, Wq, n, k, static_cast<uint32_t>(p.H), static_cast<uint32_t>(p.KPB)) &&
                      encode_kblocks_3d(&tx, m.xq, t, k, gemv::NT, static_cast<uint32_t>(p.KPB))
                : encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, k, n, k, gemv::BK, static_cast<uint32_t>(p.H)) &&
                      encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, m.xq, k, t, k, gemv::BK, gemv::NT);
    if (!maps_ok) return LLMINT8_ERR_CUDA;
    rc = before();
    if (rc != LLMINT8_OK) return rc;
    if (ev_begin && cudaEventRecord(ev_begin, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
    void (*kern)(const CUtensorMap, const CUtensorMap, const gemv::Params) =
        t <= 1 ? gemv::gemv_kernel<1, FP8> : t <= 2 ? gemv::gemv_kernel<2, FP8> : t <= 4 ? gemv::gemv_kernel<4, FP8>
        : t <= 8 ? gemv::gemv_kernel<8, FP8> : gemv::gemv_kernel<16, FP8>;
    for (int r = 0; r < repeat; ++r) {
      cudaError_t e = launch(kern, dim3(grid), dim3(gemv::THREADS), gemv::SMEM_BYTES, st, true, tw, tx, p);
      if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    }
    if (ev_end && cudaEventRecord(ev_end, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
    return LLMINT8_OK;
  }

  gemm::Params p;
  p.T = t;
  p.N = n;
  p.K = k;
  p.KB = (k + gemm::BK - 1) / gemm::BK;
  // More than one 128-row tile of tokens: CTA pairs, 256 rows per tile.
  const bool pair = t > gemm::BM;
  p.num_m = pair ? (t + 2 * gemm::BM - 1) / (2 * gemm::BM) : (t + gemm::BM - 1) / gemm::BM;
  p.sx = m.sx;
  p.sw = m.sw;
  p.n_out = m.n_out;
  p.Y = m.Y;
  p.acc_out = m.acc;
  p.wait_ns = wait_ns;
  // CTA pairs: the tile width with the least estimated time.  A pair runs
  // ceil(tiles / pairs) tiles one after the other; a tile costs one k-block
  // step per 128 bytes of K plus the accumulator drain that the next tile's
  // products wait for.  The step times are those measured on B200 for
  // gemm_pair_kernel at bn = 256, 192, 128 (operands staged per step: 32, 28,
  // 24 KiB per SM); a tie keeps the wider tile.
  p.bn = gemm::BN;
  if (pair) {
    struct Choice { int bn; double step_us, drain_us; };
    const Choice choices[] = {{256, 0.427, 1.4}, {192, 0.387, 1.05}, {128, 0.353, 0.7}};
    double best = -1.0;
    for (const Choice& c : choices) {
      const int64_t tiles = static_cast<int64_t>(p.num_m) * ((n + c.bn - 1) / c.bn);
      const int64_t rounds = (tiles + max_pairs - 1) / max_pairs;
      const double cost = static_cast<double>(rounds) * (p.KB * c.step_us + c.drain_us);
      if (best < 0.0 || cost < best * 0.999) {
        best = cost;
        p.bn = c.bn;
      }
    }
  }
  const int num_n = (n + p.bn - 1) / p.bn;
  p.num_tiles = p.num_m * num_n;
  p.num_pairs = pair ? (p.num_tiles < max_pairs ? p.num_tiles : max_pairs) : 0;
  p.y_tma = (pair && m.Y && n % 8 == 0) ? 1 : 0;
  CUtensorMap txq, twq, txo, two, ty;
  std::memset(&ty, 0, sizeof(ty));
  if (p.y_tma && !encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, m.Y, n, t, 2ull * n, gemm::P_YCOLS, gemm::BM))
    return LLMINT8_ERR_CUDA;
  // rows of B per copy: this CTA's half of the pair's N = bn
  const uint32_t b_rows = pair ? p.bn / 2 : gemm::BN;
  if (!encode_2d(&txq, CU_TENSOR_MAP_DATA_TYPE_UINT8, m.xq, k, t, k, gemm::BK, gemm::BM) ||
      !encode_2d(&twq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, k, n, k, gemm::BK, b_rows))
    return LLMINT8_ERR_CUDA;
  if (m.xo) {
    if (!encode_2d(&txo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, m.xo, m.ldo, t, 2ull * m.ldo, 64, gemm::BM) ||
        !encode_2d(&two, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, m.wo, m.ldo, n, 2ull * m.ldo, 64, b_rows))
      return LLMINT8_ERR_CUDA;
  } else {
    // No outlier operands: |O| = 0, so the kernels never load through these.
    txo = txq;
    two = twq;
  }
  rc = before();
  if (rc != LLMINT8_OK) return rc;
  if (ev_begin && cudaEventRecord(ev_begin, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
  for (int r = 0; r < repeat; ++r) {
    const cudaError_t e =
        pair ? launch_ex(gemm::gemm_pair_kernel<FP8>, dim3(2 * p.num_pairs), dim3(gemm::P_THREADS),
                         gemm::P_SMEM_BYTES, st, true, 2, txq, twq, txo, two, ty, p)
             : launch(gemm::gemm_kernel<FP8>, dim3(p.num_m * num_n), dim3(gemm::THREADS), gemm::SMEM_BYTES, st,
                      true, txq, twq, txo, two, p);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  }
  if (ev_end && cudaEventRecord(ev_end, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
  return LLMINT8_OK;
}

template <bool FP8>
int matmul_impl(const void* Xv, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                const void* Wv, int64_t N, float threshold, void* Yv, void* workspace,
                size_t ws_bytes, int path, const Inspect& ins, void* stream,
                cudaEvent_t ev_begin = nullptr, cudaEvent_t ev_end = nullptr, int repeat = 1,
                const ColumnStore* store = nullptr) {
  Layout L;
  int rc = check_common(Xv, T, K, threshold, workspace, ws_bytes, path, &L, N);
  if (rc != LLMINT8_OK) return rc;
  if (T == 0 || N == 0) return LLMINT8_OK;
  if (!Wq || !Wscale || !Yv || (!Wv && !store)) return LLMINT8_ERR_INVALID_ARG;
  if (store && (!store->slot || !store->Wst)) return LLMINT8_ERR_INVALID_ARG;
  if (store && (!aligned16(store->Wst) || (reinterpret_cast<uintptr_t>(store->slot) & 3u) ||
                (reinterpret_cast<uintptr_t>(store->n_miss) & 3u)))
    return LLMINT8_ERR_ALIGNMENT;
  if (!aligned16(Wq) || !aligned16(Wv) || !aligned16(Yv) || !aligned16(ins.xq) ||
      (reinterpret_cast<uintptr_t>(Wscale) & 3u) || (reinterpret_cast<uintptr_t>(ins.acc) & 3u) ||
      (reinterpret_cast<uintptr_t>(ins.sx) & 3u) || (reinterpret_cast<uintptr_t>(ins.idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(ins.n) & 3u))
    return LLMINT8_ERR_ALIGNMENT;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* X = static_cast<const uint16_t*>(Xv);
  const uint16_t* W = static_cast<const uint16_t*>(Wv);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int t = static_cast<int>(T), n = static_cast<int>(N), k = static_cast<int>(K);
  Prep out{ins.xq ? ins.xq : reinterpret_cast<int8_t*>(ws + L.xq),
           ins.sx ? ins.sx : reinterpret_cast<float*>(ws + L.sx),
           ins.idx ? ins.idx : reinterpret_cast<int32_t*>(ws + L.idx),
           ins.n ? ins.n : reinterpret_cast<int32_t*>(ws + L.n_out)};
  MainOps m;
  m.xq = out.xq;
  m.sx = out.sx;
  m.idx = out.idx;
  m.n_out = out.n_out;
  m.X = X;
  m.W = W;
  m.sw = Wscale;
  m.Y = static_cast<uint16_t*>(Yv);
  m.acc = ins.acc;
  if (L.path == LLMINT8_PATH_GEMM) {
    m.xo = reinterpret_cast<const uint16_t*>(ws + L.xo);
    m.wo = reinterpret_cast<const uint16_t*>(ws + L.wo);
    m.ldo = L.ldo;
  }
  ColumnStore cs;
  if (store) {
    cs = *store;
    cs.Wq = Wq;
    cs.sw = Wscale;
    m.slot = cs.slot;
    m.Wst = cs.Wst;
    m.Wqr = Wq;
    m.n_miss = cs.n_miss;
  }
  return run_main<FP8>(L.path, t, n, k, Wq, m, st,
                       [&]() { return launch_prep<FP8>(L, X, t, k, W, n, threshold, ws, out, st, cs); },
                       ev_begin, ev_end, repeat);
}

// ------------------------------------------------------------ SmoothQuant W8A8
// Workspace: row scales [T], then the codes [T][K] (256-byte aligned regions).
struct SmoothLayout {
  size_t sx = 0, xq = 0, total = 0;
};

bool smooth_layout(int64_t T, int64_t K, SmoothLayout* L) {
  if (T < 0 || K < 16 || K % 16 != 0 || K > kMaxK) return false;
  L->sx = 0;
  L->xq = align_up(sizeof(float) * static_cast<size_t>(T > 0 ? T : 1), 256);
  L->total = L->xq + align_up(static_cast<size_t>(T) * static_cast<size_t>(K) + 1, 256);
  return true;
}

int smoothquant_impl(const void* X, int64_t T, int64_t K, const float* s, const int8_t* Wq, const float* Wscale,
                     int64_t N, void* Y, void* workspace, size_t ws_bytes, int path, int32_t* acc_out,
                     int8_t* xq_out, float* sx_out, void* stream) {
  SmoothLayout L;
  if (T < 0 || N < 0 || T > INT32_MAX || N > INT32_MAX || K < 16 || K > kMaxK) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (path < LLMINT8_PATH_AUTO || path > LLMINT8_PATH_GEMM) return LLMINT8_ERR_INVALID_ARG;
  if (path == LLMINT8_PATH_AUTO) path = T <= LLMINT8_GEMV_MAX_T ? LLMINT8_PATH_GEMV : LLMINT8_PATH_GEMM;
  if (path == LLMINT8_PATH_GEMV && T > LLMINT8_GEMV_MAX_T) return LLMINT8_ERR_INVALID_ARG;
  if (!smooth_layout(T, K, &L)) return LLMINT8_ERR_INVALID_ARG;
  if (T == 0 || N == 0) return LLMINT8_OK;
  if (!X || !s || !Wq || !Wscale || !Y || !workspace) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(s) || !aligned16(Wq) || !aligned16(Y) || !aligned16(workspace) ||
      !aligned16(xq_out) || (reinterpret_cast<uintptr_t>(Wscale) & 3u) ||
      (reinterpret_cast<uintptr_t>(acc_out) & 3u) || (reinterpret_cast<uintptr_t>(sx_out) & 3u))
    return LLMINT8_ERR_ALIGNMENT;
  if (ws_bytes < L.total) return LLMINT8_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MainOps m;
  m.xq = xq_out ? xq_out : reinterpret_cast<int8_t*>(ws + L.xq);
  m.sx = sx_out ? sx_out : reinterpret_cast<float*>(ws + L.sx);
  m.sw = Wscale;
  m.Y = static_cast<uint16_t*>(Y);
  m.acc = acc_out;
  const int t = static_cast<int>(T), k = static_cast<int>(K);
  return run_main<false>(path, t, static_cast<int>(N), k, Wq, m, st, [&]() {
    const cudaError_t e = launch(smooth_quantize_activations_kernel, dim3(t), dim3(kSmoothThreads), 0, st, true,
                                 static_cast<const uint16_t*>(X), k, s, const_cast<int8_t*>(m.xq),
                                 const_cast<float*>(m.sx));
    return e == cudaSuccess ? static_cast<int>(LLMINT8_OK) : static_cast<int>(LLMINT8_ERR_CUDA);
  });
}

// ------------------------------------------------------------ allocation-free decode
// Scratch for llmint8_matmul_decode_noalloc: one array per device that loads
// the library, held until the process exits.  Sized for the decode path's
// workspace at T <= 16 and K <= kNoAllocMaxK (about 0.33 MB used of 1 MiB:
// the activation codes, their scales and the outlier list); the decode
// workspace does not grow with N.
constexpr int64_t kNoAllocMaxK = 16384;
constexpr size_t kNoAllocScratchBytes = 1u << 20;
static_assert(decode_workspace_bytes(kNoAllocMaxK) <= kNoAllocScratchBytes,
              "the decode workspace at the largest K fits the scratch array");
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocScratch {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
NoAllocScratch g_noalloc[kMaxDevices];

// Device address of this device's scratch array.  In host code the array's
// name stands for a host-side shadow, not device memory, so the address is
// queried once per device, with that device current.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LLMINT8_ERR_CUDA;
  NoAllocScratch& d = g_noalloc[dev];
  std::call_once(d.once, [&]() { d.err = cudaGetSymbolAddress(&d.ptr, g_noalloc_scratch); });
  if (d.err != cudaSuccess || d.ptr == nullptr) return LLMINT8_ERR_CUDA;
  *out = d.ptr;
  return LLMINT8_OK;
}

template <bool FP8>
int quantize_weight_impl(const void* W, int64_t N, int64_t K, int8_t* Wq, float* Wscale, void* stream) {
  if (N < 0 || N > INT32_MAX || K < 16 || K > kMaxInt32Sum) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (N == 0) return LLMINT8_OK;
  if (!W || !Wq || !Wscale) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(Wscale) & 3u)) return LLMINT8_ERR_ALIGNMENT;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  cudaError_t e = launch(quantize_weight_kernel<FP8>, dim3(static_cast<unsigned>(N)), dim3(kPrepThreads), 0,
                         static_cast<cudaStream_t>(stream), false, static_cast<const uint16_t*>(W),
                         static_cast<int>(K), Wq, Wscale);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

__global__ void selftest_timeout_kernel(uint64_t wait_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Phase 0 of `bar` never completes: nothing arrives on it.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, wait_ns, kErrTimeoutSelftest);
  __syncthreads();
}

}  // namespace
}  // namespace llmint8

using namespace llmint8;

extern "C" {

const char* llmint8_status_string(int status) {
  switch (status) {
    case LLMINT8_OK: return "ok";
    case LLMINT8_ERR_INVALID_ARG: return "invalid argument";
    case LLMINT8_ERR_ALIGNMENT: return "misaligned pointer or K not a multiple of 16";
    case LLMINT8_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
    case LLMINT8_ERR_WORKSPACE: return "workspace too small";
    case LLMINT8_ERR_CUDA: return "CUDA runtime error";
    case LLMINT8_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case LLMINT8_ERR_UNIMPLEMENTED: return "not implemented";
    default: return "unknown status";
  }
}

int llmint8_version(void) { return kVersion; }

int llmint8_set_wait_limit_ns(uint64_t ns) {
  if (ns < 1000ull || ns > 60000000000ull) return LLMINT8_ERR_INVALID_ARG;
  g_wait_ns.store(ns);
  return LLMINT8_OK;
}

size_t llmint8_workspace_bytes_path(int64_t T, int64_t N, int64_t K, int path) {
  Layout L;
  if (N < 0 || K > kMaxInt32Sum || !make_layout(T, N, K, path, &L)) return 0;
  return L.total;
}

int llmint8_kernel_launches(int64_t T, int64_t N, int64_t K, int path) {
  Layout L;
  if (T <= 0 || N <= 0 || !make_layout(T, N, K, path, &L)) return 0;
  return L.path == LLMINT8_PATH_GEMV ? 2 : 3;
}

size_t llmint8_workspace_bytes(int64_t T, int64_t N, int64_t K) {
  return llmint8_workspace_bytes_path(T, N, K, LLMINT8_PATH_AUTO);
}

int llmint8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* Wq, float* Wscale, void* stream) {
  return quantize_weight_impl<false>(W, N, K, Wq, Wscale, stream);
}

int llmint8_outlier_store_build(const void* W, int64_t N, int64_t K, const int32_t* cols, int64_t n_cols,
                                int32_t* slot, void* Wst, void* stream) {
  if (N < 0 || N > INT32_MAX || K < 16 || K > kMaxK || n_cols < 0 || n_cols > K) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (!slot) return LLMINT8_ERR_INVALID_ARG;
  if (n_cols > 0 && N > 0 && (!W || !cols || !Wst)) return LLMINT8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(slot) & 3u) || (reinterpret_cast<uintptr_t>(cols) & 3u) ||
      (n_cols > 0 && N > 0 && (!aligned16(W) || !aligned16(Wst))))
    return LLMINT8_ERR_ALIGNMENT;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(slot, 0xFF, sizeof(int32_t) * static_cast<size_t>(K), st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;  // every slot -1
  if (n_cols == 0 || N == 0) return LLMINT8_OK;
  int num_sms = 0;
  rc = device_info(&num_sms);
  if (rc != LLMINT8_OK) return rc;
  const int64_t total = n_cols * N;
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, 32LL * num_sms);
  const cudaError_t e = launch(store_build_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, false,
                               static_cast<const uint16_t*>(W), static_cast<int>(N), static_cast<int>(K), cols,
                               static_cast<int>(n_cols), slot, static_cast<uint16_t*>(Wst));
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

int llmint8_matmul_stored(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                          const int32_t* slot, const void* Wst, int64_t N, float threshold, void* Y, int32_t* n_miss,
                          void* workspace, size_t workspace_bytes, void* stream) {
  ColumnStore cs;
  cs.slot = slot;
  cs.Wst = static_cast<const uint16_t*>(Wst);
  cs.n_miss = n_miss;
  return matmul_impl<false>(X, T, K, Wq, Wscale, nullptr, N, threshold, Y, workspace, workspace_bytes,
                            LLMINT8_PATH_AUTO, Inspect{}, stream, nullptr, nullptr, 1, &cs);
}

int llmint8_matmul_stored_debug(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                                const int32_t* slot, const void* Wst, int64_t N, float threshold, void* Y,
                                int32_t* n_miss, void* workspace, size_t workspace_bytes, int path,
                                int32_t* acc_out, void* stream) {
  ColumnStore cs;
  cs.slot = slot;
  cs.Wst = static_cast<const uint16_t*>(Wst);
  cs.n_miss = n_miss;
  Inspect ins;
  ins.acc = acc_out;
  return matmul_impl<false>(X, T, K, Wq, Wscale, nullptr, N, threshold, Y, workspace, workspace_bytes, path, ins,
                            stream, nullptr, nullptr, 1, &cs);
}

int llmint8_fp8_quantize_weight(const void* W, int64_t N, int64_t K, uint8_t* Wq, float* Wscale, void* stream) {
  return quantize_weight_impl<true>(W, N, K, reinterpret_cast<int8_t*>(Wq), Wscale, stream);
}

int llmint8_fp8_matmul(const void* X, int64_t T, int64_t K, const uint8_t* Wq, const float* Wscale, const void* W,
                       int64_t N, float threshold, void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  return matmul_impl<true>(X, T, K, reinterpret_cast<const int8_t*>(Wq), Wscale, W, N, threshold, Y, workspace,
                           workspace_bytes, LLMINT8_PATH_AUTO, Inspect{}, stream);
}

int llmint8_fp8_matmul_debug(const void* X, int64_t T, int64_t K, const uint8_t* Wq, const float* Wscale,
                             const void* W, int64_t N, float threshold, void* Y, void* workspace,
                             size_t workspace_bytes, int path, float* acc_out, uint8_t* xq_out, float* xscale_out,
                             int32_t* outlier_idx_out, int32_t* n_outliers_out, void* stream) {
  Inspect ins;
  ins.acc = reinterpret_cast<int32_t*>(acc_out);
  ins.xq = reinterpret_cast<int8_t*>(xq_out);
  ins.sx = xscale_out;
  ins.idx = outlier_idx_out;
  ins.n = n_outliers_out;
  return matmul_impl<true>(X, T, K, reinterpret_cast<const int8_t*>(Wq), Wscale, W, N, threshold, Y, workspace,
                           workspace_bytes, path, ins, stream);
}

int llmint8_matmul(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                   const void* W, int64_t N, float threshold, void* Y, void* workspace,
                   size_t workspace_bytes, void* stream) {
  return matmul_impl<false>(X, T, K, Wq, Wscale, W, N, threshold, Y, workspace, workspace_bytes,
                            LLMINT8_PATH_AUTO, Inspect{}, stream);
}

int llmint8_matmul_debug(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                         const void* W, int64_t N, float threshold, void* Y, void* workspace,
                         size_t workspace_bytes, int path, int32_t* acc_out, int8_t* xq_out,
                         float* xscale_out, int32_t* outlier_idx_out, int32_t* n_outliers_out,
                         void* stream) {
  Inspect ins;
  ins.acc = acc_out;
  ins.xq = xq_out;
  ins.sx = xscale_out;
  ins.idx = outlier_idx_out;
  ins.n = n_outliers_out;
  return matmul_impl<false>(X, T, K, Wq, Wscale, W, N, threshold, Y, workspace, workspace_bytes, path, ins,
                            stream);
}

int llmint8_matmul_profile(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                           const void* W, int64_t N, float threshold, void* Y, void* workspace,
                           size_t workspace_bytes, int path, int repeat, void* ev_main_begin,
                           void* ev_main_end, void* stream) {
  if (repeat < 1 || repeat > 1000 || !ev_main_begin || !ev_main_end) return LLMINT8_ERR_INVALID_ARG;
  return matmul_impl<false>(X, T, K, Wq, Wscale, W, N, threshold, Y, workspace, workspace_bytes, path, Inspect{},
                     stream, static_cast<cudaEvent_t>(ev_main_begin), static_cast<cudaEvent_t>(ev_main_end),
                     repeat);
}

int llmint8_detect_quantize(const void* X, int64_t T, int64_t K, float threshold, int8_t* Xq,
                            float* xscale, int32_t* outlier_idx, int32_t* n_outliers, void* workspace,
                            size_t workspace_bytes, int path, void* stream) {
  Layout L;
  int rc = check_common(X, T, K, threshold, workspace, workspace_bytes, path, &L, 0);
  if (rc != LLMINT8_OK) return rc;
  if (!outlier_idx || !n_outliers) return LLMINT8_ERR_INVALID_ARG;
  if (T > 0 && (!Xq || !xscale)) return LLMINT8_ERR_INVALID_ARG;
  if ((T > 0 && !aligned16(Xq)) || (reinterpret_cast<uintptr_t>(xscale) & 3u) ||
      (reinterpret_cast<uintptr_t>(outlier_idx) & 3u) || (reinterpret_cast<uintptr_t>(n_outliers) & 3u))
    return LLMINT8_ERR_ALIGNMENT;
  rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  if (T == 0) return LLMINT8_OK;
  Prep out{Xq, xscale, outlier_idx, n_outliers};
  return launch_prep<false>(L, static_cast<const uint16_t*>(X), static_cast<int>(T), static_cast<int>(K), nullptr,
                     0, threshold, static_cast<uint8_t*>(workspace), out, static_cast<cudaStream_t>(stream));
}

int llmint8_int8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int64_t T, int64_t N, int64_t K, int32_t* acc,
                          void* stream) {
  if (T < 0 || N < 0 || T > INT32_MAX || N > INT32_MAX || K < 16 || K > kMaxK) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (T == 0 || N == 0) return LLMINT8_OK;
  if (!Xq || !Wq || !acc) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(acc) & 3u)) return LLMINT8_ERR_ALIGNMENT;
  MainOps m;
  m.xq = Xq;
  m.acc = acc;
  const int path = T <= LLMINT8_GEMV_MAX_T ? LLMINT8_PATH_GEMV : LLMINT8_PATH_GEMM;
  return run_main<false>(path, static_cast<int>(T), static_cast<int>(N), static_cast<int>(K), Wq, m,
                  static_cast<cudaStream_t>(stream), []() { return static_cast<int>(LLMINT8_OK); });
}

int llmint8_column_absmax(const void* A, int64_t rows, int64_t K, float* amax, int accumulate, void* stream) {
  if (rows < 0 || rows > INT32_MAX || K < 16 || K > kMaxK) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (!amax || (rows > 0 && !A)) return LLMINT8_ERR_INVALID_ARG;
  if ((rows > 0 && !aligned16(A)) || (reinterpret_cast<uintptr_t>(amax) & 3u)) return LLMINT8_ERR_ALIGNMENT;
  int num_sms = 0;
  int rc = device_info(&num_sms);
  if (rc != LLMINT8_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!accumulate && cudaMemsetAsync(amax, 0, sizeof(float) * static_cast<size_t>(K), st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (rows == 0) return LLMINT8_OK;
  const int strips = static_cast<int>((K + kColCols - 1) / kColCols);
  // Row chunks so that the grid holds about four CTAs per SM.
  int64_t R = (4 * num_sms + strips - 1) / strips;
  if (R > (rows + 3) / 4) R = (rows + 3) / 4;
  if (R < 1) R = 1;
  const int64_t rpc = (rows + R - 1) / R;
  R = (rows + rpc - 1) / rpc;
  const cudaError_t e = launch(column_absmax_kernel, dim3(strips, static_cast<unsigned>(R)), dim3(kColThreads), 0,
                               st, accumulate != 0, static_cast<const uint16_t*>(A), static_cast<int>(rows),
                               static_cast<int>(K), static_cast<int>(rpc), amax);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

int llmint8_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s, void* stream) {
  if (K < 0 || K > kMaxK || !(alpha >= 0.0f && alpha <= 1.0f)) return LLMINT8_ERR_INVALID_ARG;
  if (K == 0) return LLMINT8_OK;
  if (!ax || !aw || !s) return LLMINT8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ax) | reinterpret_cast<uintptr_t>(aw) | reinterpret_cast<uintptr_t>(s)) & 3u)
    return LLMINT8_ERR_ALIGNMENT;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  const cudaError_t e = launch(smooth_factors_kernel, dim3(static_cast<unsigned>((K + 255) / 256)), dim3(256), 0,
                               static_cast<cudaStream_t>(stream), true, ax, aw, static_cast<int>(K), alpha, s);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

int llmint8_smoothquant_quantize_weight(const void* W, int64_t N, int64_t K, const float* s, int8_t* Wq,
                                        float* Wscale, void* stream) {
  if (N < 0 || N > INT32_MAX || K < 16 || K > kMaxK) return LLMINT8_ERR_INVALID_ARG;
  if (K % 16 != 0) return LLMINT8_ERR_ALIGNMENT;
  if (N == 0) return LLMINT8_OK;
  if (!W || !s || !Wq || !Wscale) return LLMINT8_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(s) || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(Wscale) & 3u))
    return LLMINT8_ERR_ALIGNMENT;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  const cudaError_t e = launch(smooth_quantize_weight_kernel, dim3(static_cast<unsigned>(N)), dim3(kPrepThreads), 0,
                               static_cast<cudaStream_t>(stream), false, static_cast<const uint16_t*>(W),
                               static_cast<int>(K), s, Wq, Wscale);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

size_t llmint8_smoothquant_workspace_bytes(int64_t T, int64_t K) {
  SmoothLayout L;
  return smooth_layout(T, K, &L) ? L.total : 0;
}

int llmint8_smoothquant_matmul(const void* X, int64_t T, int64_t K, const float* s, const int8_t* Wq,
                               const float* Wscale, int64_t N, void* Y, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return smoothquant_impl(X, T, K, s, Wq, Wscale, N, Y, workspace, workspace_bytes, LLMINT8_PATH_AUTO, nullptr,
                          nullptr, nullptr, stream);
}

int llmint8_smoothquant_matmul_debug(const void* X, int64_t T, int64_t K, const float* s, const int8_t* Wq,
                                     const float* Wscale, int64_t N, void* Y, void* workspace,
                                     size_t workspace_bytes, int path, int32_t* acc_out, int8_t* xq_out,
                                     float* xscale_out, void* stream) {
  return smoothquant_impl(X, T, K, s, Wq, Wscale, N, Y, workspace, workspace_bytes, path, acc_out, xq_out,
                          xscale_out, stream);
}

int llmint8_matmul_decode_noalloc(const void* X, int64_t T, int64_t K, const int8_t* Wq,
                                  const float* Wscale, const void* W, int64_t N, float threshold,
                                  void* Y, void* stream) {
  if (T < 0 || T > LLMINT8_GEMV_MAX_T || K > kNoAllocMaxK || N < 0 || N > INT32_MAX)
    return LLMINT8_ERR_INVALID_ARG;
  Layout L;
  if (!make_layout(T, N, K, LLMINT8_PATH_GEMV, &L)) return LLMINT8_ERR_INVALID_ARG;
  if (L.total != decode_workspace_bytes(K)) return LLMINT8_ERR_INVALID_ARG;  // layouts agree
  if (T == 0 || N == 0) return LLMINT8_OK;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != LLMINT8_OK) return rc;
  // Every scratch word is written before it is read.
  return matmul_impl<false>(X, T, K, Wq, Wscale, W, N, threshold, Y, scratch, kNoAllocScratchBytes,
                     LLMINT8_PATH_GEMV, Inspect{}, stream);
}

int llmint8_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LLMINT8_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, g_error_word, sizeof(word), 0, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return LLMINT8_ERR_CUDA;
    return word == kErrBadColumn ? LLMINT8_ERR_INVALID_ARG : LLMINT8_ERR_TIMEOUT;
  }
  return LLMINT8_OK;
}

int llmint8_selftest_timeout(uint64_t wait_ns, void* stream) {
  if (wait_ns < 1000ull || wait_ns > 2000000000ull) return LLMINT8_ERR_INVALID_ARG;
  int rc = device_info(nullptr);
  if (rc != LLMINT8_OK) return rc;
  cudaError_t e = launch(selftest_timeout_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream),
                         false, wait_ns);
  return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

}  // extern "C"
