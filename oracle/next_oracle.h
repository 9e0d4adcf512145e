/*
 * next_oracle.h -- plain CPU statement of three variants built on the
 * LLM.int8() path: SmoothQuant W8A8, the same decomposition with FP8 (E4M3)
 * codes instead of int8, and the decomposition reading its fp16 outlier
 * weights from a store of columns instead of the full fp16 weight.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load or call this code.  The CUDA library
 * shares no code, header, table or constant with it.  It is compiled together
 * with llmint8_oracle.c and uses that file's fp16 conversions, int8 codes,
 * outlier detection, compaction and int8 product.
 *
 * Sources (pages on LLM quantization; titles as printed, sections theirs):
 *   [P1] "LLM quantization, part 2" (hncyxsy.com/news/230290) §5 SmoothQuant
 *        (move quantization difficulty from activations to weights by an exact
 *        per-channel rescaling; strength alpha, usually about 0.5); §2.2 the
 *        memory case for keeping only 8-bit weights.
 *   [P2] "三、模型量化" (lowentro.cn) Q9 Y = (X diag(s)^-1)(diag(s) W); Q10 the
 *        smoothing factor from the channel maxima of X and W and alpha.
 *   [P5] "量化压缩实战：INT8 / INT4 / AWQ / GPTQ 全面对比" (tqpw.cn) §3.6 FP8:
 *        an 8-bit float format, E4M3 (1 sign, 4 exponent, 3 mantissa bits) for
 *        inference, native on B200.
 *
 * Layouts as in llmint8_oracle.h: X fp16 [T][K], W fp16 [N][K] (out x in),
 * fp16 values as binary16 bit patterns.  Integer- and code-producing steps are
 * binary32; sums of products are binary64 and exact where stated.
 */
#ifndef NEXT_ORACLE_H
#define NEXT_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ SmoothQuant */

/* amax[k] = max_r |A[r,k]| over the rows of an fp16 matrix [rows][K]: the
 * per-input-channel maxima of an activation batch or of a weight matrix. */
void onext_column_absmax(const uint16_t* A, int64_t rows, int64_t K, float* amax);

/* p^a in binary32: 1 for a == 0, p for a == 1, sqrtf(p) for a == 0.5 (these
 * three exact or correctly rounded), powf(p, a) otherwise. */
float onext_pow(float p, float a);

/* Smoothing factors s[k] = ax[k]^alpha / aw[k]^(1 - alpha) (binary32; the
 * exponent 1 - alpha is formed in binary32).  A channel with ax[k] == 0 or
 * aw[k] == 0 carries nothing to balance and keeps s[k] = 1. */
void onext_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s);

/* diag(s) W folded into the weight, then per-output-channel int8:
 *   W~[n,k] = fl(W[n,k] * s[k]);  sw[n] = max_k |W~[n,k]| / 127;
 *   Wq[n,k] = clamp(rint(fl(W~[n,k] / sw[n])), +-127), 0 if sw[n] == 0. */
void onext_smooth_quantize_weight(const uint16_t* W, const float* s, int64_t N, int64_t K, int8_t* Wq,
                                  float* sw);

/* X diag(s)^-1, then per-row int8 over every column (no outlier part):
 *   X~[t,k] = fl(X[t,k] / s[k]);  sx[t] = max_k |X~[t,k]| / 127;  Xq = codes. */
void onext_smooth_quantize_activations(const uint16_t* X, const float* s, int64_t T, int64_t K,
                                       int8_t* Xq, float* sx);

/* The W8A8 matmul: codes of X diag(s)^-1, acc = Xq Wq^T (exact), Y[t,n] =
 * fp16(acc * sx[t] * sw[n]) in binary64 with one rounding.  Xq, sx, acc may be
 * NULL.  Returns 0, -1 on int32 overflow, -2 on allocation failure. */
int onext_smoothquant_matmul(const uint16_t* X, const float* s, int64_t T, int64_t K, const int8_t* Wq,
                             const float* sw, int64_t N, uint16_t* Y, int8_t* Xq, float* sx, int32_t* acc);

/* ------------------------------------------------------------ FP8 E4M3 */

/* Value of an E4M3 code: bias 7; exponent field 0 is subnormal (m * 2^-9);
 * exponent 15 with mantissa 7 is NaN (no infinities); largest finite 448. */
float onext_e4m3_to_float(uint8_t c);

/* binary32 -> E4M3, round to nearest with ties to even, magnitudes past 448
 * saturate to 448 (finite); the sign is kept (-0 and negatives that round to
 * zero give 0x80); NaN gives 0x7f. */
uint8_t onext_float_to_e4m3(float x);

/* E4M3 code of x under scale s: e4m3(fl(x / s)); 0 when s == 0. */
uint8_t onext_quantize_e4m3(float x, float s);

/* Per-output-channel E4M3 weight codes: sw[n] = max_k |W[n,k]| / 448. */
void onext_fp8_quantize_weight(const uint16_t* W, int64_t N, int64_t K, uint8_t* Wq, float* sw);

/* Per-row E4M3 activation codes over the regular columns (flag[k] == 0):
 * sx[t] = max_{k not in O} |X[t,k]| / 448; outlier columns get code 0. */
void onext_fp8_quantize_activations(const uint16_t* X, int64_t T, int64_t K, const uint8_t* flag,
                                    uint8_t* Xq, float* sx);

/* acc[t,n] = sum_k e4m3(Xq[t,k]) * e4m3(Wq[n,k]) in binary64.  Every product
 * has at most 8 significant bits and lies on the grid 2^-18, every partial sum
 * stays below 2^35: the binary64 sum is exact for K <= 65536. */
void onext_fp8_gemm(const uint8_t* Xq, const uint8_t* Wq, int64_t T, int64_t N, int64_t K, double* acc);

/* The decomposition with E4M3 codes: outlier detection and list as for int8,
 * E4M3 activation codes, acc (binary64, exact), the fp16 outlier part, then
 * Y[t,n] = fp16(acc * sx[t] * sw[n] + yo[t,n]) with one rounding.  Every
 * intermediate may be NULL.  Returns 0, -2 on allocation failure. */
int onext_fp8_matmul(const uint16_t* X, int64_t T, int64_t K, const uint8_t* Wq, const float* sw,
                     const uint16_t* W, int64_t N, float tau, uint16_t* Y, uint8_t* flag, int32_t* idx,
                     int64_t* nO, uint8_t* Xq, float* sx, double* acc, double* yo);

/* ------------------------------------------------------------ stored outlier columns */

/* The fp16 weight of one int8 code when no stored column holds it:
 * fp16(fl(s * q)) -- the binary32 product, then one rounding to binary16. */
uint16_t onext_reconstruct_weight(int8_t q, float s);

/* yo[t,n] = sum_j X[t,O_j] * w(n, O_j) in binary64, ascending j, where
 * w(n,k) = Wst[slot[k]][n] when slot[k] >= 0 (a stored fp16 column; Wst is
 * [n_store][N], one column of W per row), else onext_reconstruct_weight(
 * Wq[n,k], sw[n]).  Returns the misses: outlier columns with slot[k] < 0. */
int64_t onext_outlier_gemm_stored(const uint16_t* X, const int8_t* Wq, const float* sw, const int32_t* slot,
                                  const uint16_t* Wst, int64_t T, int64_t N, int64_t K, const int32_t* idx,
                                  int64_t nO, double* yo);

/* The LLM.int8() matmul with its outlier weights from the store (a1..a7 as
 * oracle_matmul, a6 by onext_outlier_gemm_stored).  *n_miss receives the
 * misses.  Returns 0, -1 on int32 overflow, -2 on allocation failure. */
int onext_matmul_stored(const uint16_t* X, int64_t T, int64_t K, const int8_t* Wq, const float* sw,
                        const int32_t* slot, const uint16_t* Wst, int64_t N, float tau, uint16_t* Y,
                        int64_t* n_miss);

#ifdef __cplusplus
}
#endif
#endif
