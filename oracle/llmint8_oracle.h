/*
 * llmint8_oracle.h -- plain CPU statement of the LLM.int8() mixed-precision
 * decomposition matmul Y = X * W^T.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load or call this code.  The CUDA library
 * shares no code, header, table or constant with it, and the product path
 * never calls it.
 *
 * Sources (pages on LLM quantization; titles as printed, sections theirs):
 *   [P1] "LLM quantization, part 2" (hncyxsy.com/news/230290), §1 and §2.1
 *        vector-wise quantization + mixed-precision decomposition, threshold 6.0.
 *   [P2] "三、模型量化" (lowentro.cn interview notes), Q2 symmetric quantization
 *        formulas, Q4 LLM.int8(), Q11 outliers.
 *   [P5] "量化压缩实战：INT8 / INT4 / AWQ / GPTQ 全面对比" (tqpw.cn/news/5683),
 *        §2.1 the absmax recipe and its worked example, §3.1 LLM.int8().
 *
 * Layouts: X fp16 [T][K] row-major (token-major), W fp16 [N][K] row-major
 * (out-features x in-features), so Y = X * W^T is [T][N].  fp16 values travel
 * as their IEEE binary16 bit patterns (uint16_t).  Sizes are int64_t.
 *
 * Precision: decisions that produce an integer (the outlier test, the scales,
 * the int8 codes) are taken in IEEE binary32, the precision the CUDA kernels
 * use, so both sides must agree bit for bit.  Everything after the integer
 * product (the fp16 outlier product, dequantisation and the sum) is carried in
 * binary64 and rounded once to binary16: the oracle states the exact value of
 * the method; the kernels' fp32 accumulation is judged against it with a
 * tolerance.
 */
#ifndef LLMINT8_ORACLE_H
#define LLMINT8_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* binary16 bits -> value (exact). */
float oracle_h2f(uint16_t h);
/* value -> binary16 bits, round to nearest, ties to even, overflow to inf. */
uint16_t oracle_d2h(double v);

void oracle_h2f_array(const uint16_t* h, int64_t n, float* out);
void oracle_d2h_array(const double* v, int64_t n, uint16_t* out);

/* Symmetric absmax int8 code of x under scale s (binary32):
 * clamp(round_half_even(x / s), -127, 127); 0 when s == 0. */
int8_t oracle_quantize_value(float x, float s);

/* a0: per-output-channel (per row of W) scale sw[n] = max_k |W[n,k]| / 127 and
 * codes Wq[n,k] over all K. */
void oracle_quantize_weight(const uint16_t* W, int64_t N, int64_t K, int8_t* Wq, float* sw);

/* a1: flag[k] = 1 iff some row t has |X[t,k]| >= tau. */
void oracle_detect_outliers(const uint16_t* X, int64_t T, int64_t K, float tau, uint8_t* flag);

/* a4 (index part): ascending list of flagged k; returns |O|. */
int64_t oracle_compact(const uint8_t* flag, int64_t K, int32_t* idx);

/* a2+a3: per-row scale over the non-outlier columns and int8 codes; outlier
 * columns get code 0. */
void oracle_quantize_activations(const uint16_t* X, int64_t T, int64_t K, const uint8_t* flag,
                                 int8_t* Xq, float* sx);

/* a5: acc[t,n] = sum_k Xq[t,k] * Wq[n,k], summed in int64.  Returns 0, or -1
 * if some sum does not fit int32 (acc then holds the low 32 bits). */
int oracle_int8_gemm(const int8_t* Xq, const int8_t* Wq, int64_t T, int64_t N, int64_t K,
                     int32_t* acc);

/* a6: yo[t,n] = sum_{j<nO} X[t,idx[j]] * W[n,idx[j]] in binary64, ascending j. */
void oracle_outlier_gemm(const uint16_t* X, const uint16_t* W, int64_t T, int64_t N, int64_t K,
                         const int32_t* idx, int64_t nO, double* yo);

/* a7: Y[t,n] = fp16( acc[t,n] * sx[t] * sw[n] + yo[t,n] ), binary64 then one
 * rounding.  yo may be NULL (no outliers). */
void oracle_dequant_combine(const int32_t* acc, const float* sx, const float* sw, const double* yo,
                            int64_t T, int64_t N, uint16_t* Y);

/* a1..a7 in order.  Every intermediate pointer may be NULL; when NULL the
 * oracle allocates its own.  Returns 0, -1 on int32 overflow, -2 on allocation
 * failure. */
int oracle_matmul(const uint16_t* X, int64_t T, int64_t K, const int8_t* Wq, const float* sw,
                  const uint16_t* W, int64_t N, float tau, uint16_t* Y,
                  uint8_t* flag, int32_t* idx, int64_t* nO, int8_t* Xq, float* sx,
                  int32_t* acc, double* yo);

/* Threads the OpenMP loops use (1 without OpenMP). */
int oracle_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
