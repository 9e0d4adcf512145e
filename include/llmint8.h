/*
 * llmint8.h -- C ABI of the B200 (sm_100a) LLM.int8() mixed-precision
 * decomposition matmul  Y = X * W^T.
 *
 * The method (pages on LLM quantization; titles as printed, sections theirs):
 *   'LLM quantization, part 2' (hncyxsy.com/news/230290) §2.1: vector-wise
 *     quantization (one int8 scale per output feature of W) and mixed-precision
 *     decomposition: feature dims whose activation magnitude reaches a
 *     threshold (usually 6.0) are outliers; those columns of X and W are
 *     multiplied in fp16, all other columns as an int8 matrix product, and the
 *     two partial results are added.
 *   '三、模型量化' (lowentro.cn) Q2: symmetric int8, q = round(r/s),
 *     s = max|r| / 127, dequantised r' = s*q.  Q4: the same decomposition.
 *   '量化压缩实战：INT8 / INT4 / AWQ / GPTQ 全面对比' (tqpw.cn) §2.1: absmax
 *     recipe (scale = max_val/127, round, clip) and its worked example.
 *
 * Conventions for every entry point
 *   - Layouts: X fp16 [T][K] row-major, W fp16 [N][K] row-major (out-features
 *     x in-features), Wq int8 [N][K], Y fp16 [T][N]; all contiguous.
 *   - fp16 buffers are passed as `void*` holding IEEE binary16 values.
 *   - Every pointer is a DEVICE pointer on the current CUDA device unless the
 *     comment says host.  The caller owns all memory; the library allocates
 *     nothing on these calls and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it; outputs are ready when the stream reaches them.
 *   - Alignment: X, W, Wq, Y, workspace 16-byte aligned; K % 16 == 0.
 *   - Return value: an llmint8_status.  Argument and launch errors return at
 *     once and launch nothing.  A device-side fault detected by a kernel (a
 *     bounded wait that ran out) is recorded in a per-device error word and
 *     reported by llmint8_sync_status().
 *   - Requires an sm_100 device (B200); otherwise LLMINT8_ERR_UNSUPPORTED_ARCH.
 */
#ifndef LLMINT8_H
#define LLMINT8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLMINT8_API __attribute__((visibility("default")))
#else
#define LLMINT8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LLMINT8_OK = 0,
  LLMINT8_ERR_INVALID_ARG = -1,      /* null pointer, bad size, NaN threshold, bad path   */
  LLMINT8_ERR_ALIGNMENT = -2,        /* pointer not 16-byte aligned or K % 16 != 0         */
  LLMINT8_ERR_UNSUPPORTED_ARCH = -3, /* current device is not compute capability 10.x      */
  LLMINT8_ERR_WORKSPACE = -4,        /* workspace smaller than llmint8_workspace_bytes()   */
  LLMINT8_ERR_CUDA = -5,             /* a CUDA runtime call failed (launch, attribute ...) */
  LLMINT8_ERR_TIMEOUT = -6,          /* a kernel's bounded wait ran out (device error word) */
  LLMINT8_ERR_UNIMPLEMENTED = -7
} llmint8_status;

/* Kernel path of llmint8_matmul.  AUTO takes GEMV for T <= 16, else GEMM. */
enum {
  LLMINT8_PATH_AUTO = 0,
  LLMINT8_PATH_GEMV = 1, /* decode: one prep kernel + a weight-streaming tcgen05 GEMV,
                            each CTA a slab of output rows over all of K (T <= 16 only) */
  LLMINT8_PATH_GEMM = 2  /* prefill: activation kernels + a TMA-fed tcgen05 int8 GEMM
                            with the fp16 outlier GEMM in a second TMEM accumulator      */
};

/* Largest T the decode path takes. */
#define LLMINT8_GEMV_MAX_T 16

/* Static text for a status code (host only, never NULL). */
LLMINT8_API const char* llmint8_status_string(int status);

/* Library version, major*10000 + minor*100 + patch (host only). */
LLMINT8_API int llmint8_version(void);

/*
 * Offline weight quantisation, once per weight matrix
 * ('LLM quantization, part 2' §2.1 vector-wise quantization):
 *   Wscale[n] = max_k |W[n,k]| / 127                       (binary32, IEEE division)
 *   Wq[n,k]   = clamp(round_half_even(W[n,k] / Wscale[n]), -127, 127), 0 if Wscale[n] == 0
 * over all K columns.  W: fp16 [N][K] in; Wq: int8 [N][K] out; Wscale: float [N] out.
 * N >= 1, K >= 16, K % 16 == 0.
 */
LLMINT8_API int llmint8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* Wq, float* Wscale,
                            void* stream);

/* Bytes of device workspace llmint8_matmul needs for this shape on the AUTO path
 * (host only; 0 for invalid sizes).  The size covers the worst case |O| = K. */
LLMINT8_API size_t llmint8_workspace_bytes(int64_t T, int64_t N, int64_t K);

/* Same for an explicit path (LLMINT8_PATH_*); 0 if the path cannot take T. */
LLMINT8_API size_t llmint8_workspace_bytes_path(int64_t T, int64_t N, int64_t K, int path);

/* How many kernels one llmint8_matmul call of this shape launches on `path`
 * (no counterpart in the pages; for launch accounting): 2 for the decode path
 * (prep + GEMV), 3 for the prefill path (detection, quantisation with the
 * compaction and gathers, GEMM).  0 for shapes the path rejects or T == 0 / N == 0.  Host-only:
 * touches no device. */
LLMINT8_API int llmint8_kernel_launches(int64_t T, int64_t N, int64_t K, int path);

/*
 * Y = X * W^T by the LLM.int8() decomposition ('LLM quantization, part 2' §2.1;
 * '三、模型量化' Q4):
 *   O      = { k : |X[t,k]| >= threshold for some row t of this X }   (ascending)
 *   sx[t]  = max_{k not in O} |X[t,k]| / 127                           (binary32)
 *   Xq     = clamp(round_half_even(X / sx), -127, 127) on k not in O, 0 on O
 *   acc    = Xq * Wq^T                                                 (exact int32)
 *   yo     = X[:,O] * W[:,O]^T                                         (fp16 in, fp32 sum)
 *   Y      = fp16( acc * sx[t] * Wscale[n] + yo )
 * X: fp16 [T][K]; Wq/Wscale from llmint8_quantize_weight(W); W: the fp16 weight
 * [N][K], read only at the outlier columns; Y: fp16 [T][N] out.
 * threshold: +inf disables the outlier part; NaN is rejected.
 * workspace: device scratch of at least llmint8_workspace_bytes(T, N, K) bytes,
 * owned by the caller, contents on entry ignored; calls that share a workspace
 * must be ordered on one stream.  The outlier set never returns to the host.
 * The kernels launch with programmatic dependent launch and start reading Wq
 * before the kernel queued ahead of them on `stream` is done (X, W, Wscale
 * and the workspace only after it): Wq must not be written by a kernel that
 * lets its dependents launch before its own writes are complete.
 * T >= 1, N >= 1, K >= 16, K % 16 == 0, K * 127 * 127 < 2^31.
 */
LLMINT8_API int llmint8_matmul(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                   const void* W, int64_t N, float threshold, void* Y, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * Inspection variant of llmint8_matmul used by the parity tests: `path` picks
 * the kernel path (LLMINT8_PATH_*), and each non-NULL output receives an
 * intermediate of that very call (all device buffers, written in full):
 *   acc_out         int32 [T][N]  the exact int8 products acc
 *   xq_out          int8  [T][K]  the activation codes Xq (16-byte aligned)
 *   xscale_out      float [T]     the per-row scales sx
 *   outlier_idx_out int32 [K]     the outlier columns, ascending (first *n valid)
 *   n_outliers_out  int32 [1]     |O|
 * The workspace must hold llmint8_workspace_bytes_path(T, N, K, path) bytes.
 */
LLMINT8_API int llmint8_matmul_debug(const void* X, int64_t T, int64_t K, const int8_t* Wq,
                         const float* Wscale, const void* W, int64_t N, float threshold, void* Y,
                         void* workspace, size_t workspace_bytes, int path, int32_t* acc_out,
                         int8_t* xq_out, float* xscale_out, int32_t* outlier_idx_out,
                         int32_t* n_outliers_out, void* stream);

/*
 * Profiling variant of llmint8_matmul_debug: runs the activation stages once,
 * records `ev_main_begin` (cudaEvent_t, created by the caller), launches the
 * main kernel (the GEMV or the GEMM) `repeat` times back to back (1..1000;
 * each launch recomputes the same Y from the same workspace), then records
 * `ev_main_end`.  (elapsed time) / repeat is the main kernel's duration per
 * launch as consecutive layers would run it, with the events' own overhead
 * spread over the repeats.
 */
LLMINT8_API int llmint8_matmul_profile(const void* X, int64_t T, int64_t K, const int8_t* Wq,
                                       const float* Wscale, const void* W, int64_t N,
                                       float threshold, void* Y, void* workspace,
                                       size_t workspace_bytes, int path, int repeat,
                                       void* ev_main_begin, void* ev_main_end, void* stream);

/*
 * The activation stages alone (outlier detection, compaction, per-row scale,
 * int8 codes), run by the kernels and launch configuration that `path` uses
 * inside llmint8_matmul (AUTO: the decode kernel for T <= 16, else the
 * prefill kernels; GEMM: the prefill kernels for any T >= 1):
 *   Xq int8 [T][K], xscale float [T], outlier_idx int32 [K] (first *n_outliers
 *   entries valid, ascending), n_outliers int32 [1]; all device, all outputs.
 * workspace: llmint8_workspace_bytes_path(T, 0, K, path) bytes.
 */
LLMINT8_API int llmint8_detect_quantize(const void* X, int64_t T, int64_t K, float threshold, int8_t* Xq,
                            float* xscale, int32_t* outlier_idx, int32_t* n_outliers,
                            void* workspace, size_t workspace_bytes, int path, void* stream);

/*
 * The int8 product of the regular columns on its own ('LLM quantization,
 * part 2' §2.1: the non-outlier columns are multiplied as an int8 matrix
 * product; '三、模型量化' Q4: INT8 matrix multiplication of the normal part):
 *   acc[t,n] = sum_k Xq[t,k] * Wq[n,k]        (exact, int32)
 * Xq: int8 [T][K] (any codes, -128 included), Wq: int8 [N][K], acc: int32
 * [T][N] out; all device, row-major.  Runs the kernels llmint8_matmul uses
 * for its int8 part on the tensor cores: the GEMV for T <= 16, the one-CTA
 * GEMM for 17 <= T <= 128, the CTA-pair GEMM for larger T, with no outlier
 * part and no dequantisation.  Xq and Wq 16-byte aligned, acc 4-byte
 * aligned; 16 <= K <= 65536, K % 16 == 0 (K * 128 * 128 < 2^31, so no sum can
 * overflow).  T == 0 or N == 0: OK, nothing launched.  Launched with
 * programmatic dependent launch: Wq must not be written by a kernel that lets
 * its dependents launch before its writes are complete (as for llmint8_matmul).
 */
LLMINT8_API int llmint8_int8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int64_t T, int64_t N, int64_t K,
                                      int32_t* acc, void* stream);

/*
 * ---------------------------------------------------------------- stored outlier columns
 * 'LLM quantization, part 2' §2.2: 8-bit weights exist to halve the weight
 * memory (26 GB -> about 13 GB at 13B), while §2.1 multiplies the outlier
 * columns with their fp16 weights.  Instead of the whole fp16 W, a store
 * keeps fp16 copies of a chosen set of columns (those calibration found to be
 * outliers), laid out column by column:
 *   Wst fp16 [n_store][N], Wst[i][n] = W[n, cols[i]];  slot int32 [K],
 *   slot[cols[i]] = i, -1 for columns not stored.
 * A call reads an outlier column k from Wst[slot[k]][:] (contiguous over the
 * output channels).  An outlier column with no stored copy (a miss) uses the
 * fp16 value of its int8 weight, fp16(fl(Wscale[n] * Wq[n,k])), and is
 * counted in *n_miss so that the caller can add it to the store.  Resident
 * weight bytes: N*K (Wq) + 4N + 2*N*n_store + 4K instead of 3*N*K.
 */

/* Fills slot (all -1, then slot[cols[i]] = i) and Wst[i][:] = W[:, cols[i]].
 * cols: device int32 [n_cols], distinct, in [0, K) (a column outside is
 * skipped and reported by llmint8_sync_status as LLMINT8_ERR_INVALID_ARG);
 * 0 <= n_cols <= K.  W 16-byte aligned, Wst fp16 [n_cols][N] 16-byte
 * aligned.  The fp16 W may be freed once the stream is past this call. */
LLMINT8_API int llmint8_outlier_store_build(const void* W, int64_t N, int64_t K, const int32_t* cols, int64_t n_cols,
                                            int32_t* slot, void* Wst, void* stream);

/* llmint8_matmul with the outlier weights from the store instead of the fp16
 * W (which the call does not take).  n_miss: optional device int32 [1], set
 * to the number of this call's outlier columns missing from the store.
 * Workspace: llmint8_workspace_bytes(T, N, K).  Other conventions as
 * llmint8_matmul. */
LLMINT8_API int llmint8_matmul_stored(const void* X, int64_t T, int64_t K, const int8_t* Wq, const float* Wscale,
                                      const int32_t* slot, const void* Wst, int64_t N, float threshold, void* Y,
                                      int32_t* n_miss, void* workspace, size_t workspace_bytes, void* stream);

/* Inspection variant: `path` (LLMINT8_PATH_*) and an optional int32 [T][N]
 * accumulator output, as llmint8_matmul_debug. */
LLMINT8_API int llmint8_matmul_stored_debug(const void* X, int64_t T, int64_t K, const int8_t* Wq,
                                            const float* Wscale, const int32_t* slot, const void* Wst, int64_t N,
                                            float threshold, void* Y, int32_t* n_miss, void* workspace,
                                            size_t workspace_bytes, int path, int32_t* acc_out, void* stream);

/*
 * ---------------------------------------------------------------- FP8 E4M3 variant
 * '量化压缩实战' §3.6: FP8 is an 8-bit float format; E4M3 (1 sign, 4 exponent,
 * 3 mantissa bits, largest finite 448) is the inference variant, native on
 * B200.  The same decomposition as llmint8_matmul with E4M3 codes for the
 * regular columns:
 *   Wscale[n] = max_k |W[n,k]| / 448,  Wq[n,k] = e4m3(W[n,k] / Wscale[n])
 *   sx[t]     = max_{k not in O} |X[t,k]| / 448,  Xq = e4m3(X / sx), 0 on O
 *   acc       = Xq * Wq^T on the tensor cores (tcgen05 kind::f8f6f4), f32
 *   Y         = fp16( acc * sx[t] * Wscale[n] + X[:,O] W[:,O]^T )
 * e4m3(v): binary32 quotient, then round to nearest even, saturating at
 * +-448, sign kept; a zero scale gives code 0.  Codes are uint8 bit patterns.
 * The f32 sum of the products is not exact (the int8 path's int32 sum is),
 * so only the codes, scales and outlier list are bit-exact results.
 */

/* Per-output-channel E4M3 weight codes: Wq uint8 [N][K], Wscale float [N]. */
LLMINT8_API int llmint8_fp8_quantize_weight(const void* W, int64_t N, int64_t K, uint8_t* Wq, float* Wscale,
                                            void* stream);

/* Y = X W^T by the decomposition with E4M3 codes.  Arguments, workspace
 * (llmint8_workspace_bytes) and conventions as llmint8_matmul. */
LLMINT8_API int llmint8_fp8_matmul(const void* X, int64_t T, int64_t K, const uint8_t* Wq, const float* Wscale,
                                   const void* W, int64_t N, float threshold, void* Y, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Inspection variant, as llmint8_matmul_debug: acc_out float [T][N] (the f32
 * accumulator), xq_out uint8 [T][K] (16-byte aligned), xscale_out float [T],
 * outlier_idx_out int32 [K], n_outliers_out int32 [1]. */
LLMINT8_API int llmint8_fp8_matmul_debug(const void* X, int64_t T, int64_t K, const uint8_t* Wq,
                                         const float* Wscale, const void* W, int64_t N, float threshold, void* Y,
                                         void* workspace, size_t workspace_bytes, int path, float* acc_out,
                                         uint8_t* xq_out, float* xscale_out, int32_t* outlier_idx_out,
                                         int32_t* n_outliers_out, void* stream);

/*
 * ---------------------------------------------------------------- SmoothQuant W8A8
 * 'LLM quantization, part 2' §5 and '三、模型量化' Q9-Q10: Y = X W^T =
 * (X diag(s)^-1)(W diag(s))^T exactly; per-channel factors s move the
 * activations' outlier range into the weights, then both sides are int8
 * (X per row, W per output channel) on the int8 tensor cores, no fp16 part:
 *   s[k]  = max|X[:,k]|^alpha / max|W[:,k]|^(1 - alpha)   (1 if either max is 0)
 *   W~    = W[n,k] * s[k]  -> Wscale[n] = max|W~[n,:]| / 127, Wq = codes
 *   X~    = X[t,k] / s[k]  -> sx[t] = max|X~[t,:]| / 127, Xq = codes
 *   Y     = fp16( (Xq Wq^T) * sx[t] * Wscale[n] )
 * Products and quotients binary32 (round to nearest even); codes as for
 * llmint8_quantize_weight.  The factor reading: the pages print the Q10
 * formula as a product; the quotient is the form whose alpha = 0.5 balances
 * the two sides' channel ranges, as Q10 says the factor should.
 */

/* amax[k] = max over the rows of |A[r,k]| for an fp16 matrix A [rows][K]
 * (the channel maxima of a calibration batch X, or of a weight W).  With
 * accumulate != 0 the result is max(amax[k], ...), so several calibration
 * batches can be folded in; otherwise amax is cleared first.  A 16-byte
 * aligned, K % 16 == 0, amax float [K] (4-byte aligned). */
LLMINT8_API int llmint8_column_absmax(const void* A, int64_t rows, int64_t K, float* amax, int accumulate,
                                      void* stream);

/* s[k] = ax[k]^alpha / aw[k]^(1 - alpha), 0 <= alpha <= 1; 1 where ax[k] or
 * aw[k] is 0.  alpha 0, 1/2 and 1 are exact or correctly rounded (sqrt);
 * other alphas use powf.  All float [K], device. */
LLMINT8_API int llmint8_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s,
                                       void* stream);

/* Offline: W~ = W diag(s), quantised per output channel: Wq int8 [N][K],
 * Wscale float [N].  s float [K], 16-byte aligned. */
LLMINT8_API int llmint8_smoothquant_quantize_weight(const void* W, int64_t N, int64_t K, const float* s,
                                                    int8_t* Wq, float* Wscale, void* stream);

/* Device workspace of llmint8_smoothquant_matmul (row scales and codes). */
LLMINT8_API size_t llmint8_smoothquant_workspace_bytes(int64_t T, int64_t K);

/* Y fp16 [T][N] = the W8A8 product of X fp16 [T][K] under factors s with the
 * smoothed weight (Wq, Wscale).  One activation kernel (X / s, row scale,
 * codes) then the GEMV (T <= 16) or GEMM of llmint8_matmul with no outlier
 * part.  Same conventions as llmint8_matmul; K <= 65536. */
LLMINT8_API int llmint8_smoothquant_matmul(const void* X, int64_t T, int64_t K, const float* s,
                                           const int8_t* Wq, const float* Wscale, int64_t N, void* Y,
                                           void* workspace, size_t workspace_bytes, void* stream);

/* Inspection variant: `path` (LLMINT8_PATH_*) picks the kernel path; non-NULL
 * acc_out int32 [T][N], xq_out int8 [T][K] (16-byte aligned), xscale_out
 * float [T] receive the call's intermediates. */
LLMINT8_API int llmint8_smoothquant_matmul_debug(const void* X, int64_t T, int64_t K, const float* s,
                                                 const int8_t* Wq, const float* Wscale, int64_t N, void* Y,
                                                 void* workspace, size_t workspace_bytes, int path,
                                                 int32_t* acc_out, int8_t* xq_out, float* xscale_out,
                                                 void* stream);

/*
 * llmint8_matmul for decode shapes (T <= 16) without a caller workspace and
 * without allocating anything.  The pages have no counterpart: this entry
 * serves callers that cannot call cudaMalloc, such as a host program that owns
 * all device memory through its own pool (a library may not take memory behind
 * its back) or a latency-critical loop where an allocation could stall the
 * device or fail mid-run.  Scratch comes from one fixed array in device memory
 * per GPU that loads the library (1 MiB, kept until the process exits).
 *   Limits: 0 <= T <= 16, 16 <= K <= 16384, K % 16 == 0, 0 <= N < 2^31.
 *   T == 0 or N == 0 is an empty problem: OK, nothing launched.  Sizes past
 *   these limits return LLMINT8_ERR_INVALID_ARG and launch nothing.  The
 *   scratch holds the outlier list, the row scales and the codes of at most
 *   16 x 16384 activations (about 0.33 MB); it does not depend on N.
 *   The first call on a device looks up that device's array address (a
 *   runtime symbol query); later calls only launch kernels.
 *   Every call on a device shares the array and leaves its contents behind, so
 *   calls must not overlap on the GPU: order them on one stream, or two
 *   overlapping calls race on the scratch and both results are undefined.
 * Arguments, layouts and results are those of llmint8_matmul.
 */
LLMINT8_API int llmint8_matmul_decode_noalloc(const void* X, int64_t T, int64_t K, const int8_t* Wq,
                                              const float* Wscale, const void* W, int64_t N,
                                              float threshold, void* Y, void* stream);

/*
 * Waits for `stream`, then reads and clears this device's error word.
 * Returns LLMINT8_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last call, LLMINT8_ERR_INVALID_ARG if llmint8_outlier_store_build met a
 * column outside [0, K), LLMINT8_ERR_CUDA if the stream reported an error,
 * else OK.
 */
LLMINT8_API int llmint8_sync_status(void* stream);

/*
 * Self-test of the failure path: launches one kernel that waits on an
 * mbarrier no thread ever arrives at, gives up after `wait_ns` nanoseconds
 * (1 000 .. 2e9), records LLMINT8_ERR_TIMEOUT in the error word and returns
 * normally.  A following llmint8_sync_status() must report the timeout.
 */
LLMINT8_API int llmint8_selftest_timeout(uint64_t wait_ns, void* stream);

/* Per-wait limit used by every kernel's bounded waits (default 2 s). */
LLMINT8_API int llmint8_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* LLMINT8_H */
