/*
 * next_oracle.c -- plain CPU statement of SmoothQuant W8A8, the FP8 (E4M3)
 * decomposition and the decomposition with stored outlier-weight columns.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline of the bench).
 * Shares no code with the CUDA library.  See next_oracle.h for the sources,
 * layouts and precision rules.  Scalar loops in the order the method states;
 * OpenMP splits independent output rows only.
 *
 * Build with llmint8_oracle.c: gcc -O2 -std=c11 -fno-fast-math
 * -ffp-contract=off -fopenmp -fPIC -shared.
 */
#include "next_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "llmint8_oracle.h"

/* ================================================================ SmoothQuant
 * [P2] Q9: Y = X W = (X diag(s)^-1)(diag(s) W) holds exactly, so activation
 * channels with large values can be scaled down and the same weight channels
 * scaled up.  [P2] Q10 / [P1] §5: s_j from the channel maxima of X and W with
 * migration strength alpha; the balance it aims at (equal ranges of both
 * sides at alpha = 0.5) is the quotient form max|X_j|^a / max|W_j|^(1-a). */

void onext_column_absmax(const uint16_t* A, int64_t rows, int64_t K, float* amax) {
  for (int64_t k = 0; k < K; ++k) amax[k] = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(oracle_h2f(A[r * K + k]));
      if (a > amax[k]) amax[k] = a;
    }
}

float onext_pow(float p, float a) {
  if (a == 0.0f) return 1.0f;
  if (a == 1.0f) return p;
  if (a == 0.5f) return sqrtf(p);
  return powf(p, a);
}

void onext_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s) {
  const float beta = 1.0f - alpha;
  for (int64_t k = 0; k < K; ++k) {
    if (ax[k] == 0.0f || aw[k] == 0.0f) {
      s[k] = 1.0f;
      continue;
    }
    s[k] = onext_pow(ax[k], alpha) / onext_pow(aw[k], beta);
  }
}

void onext_smooth_quantize_weight(const uint16_t* W, const float* s, int64_t N, int64_t K, int8_t* Wq,
                                  float* sw) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(oracle_h2f(W[n * K + k]) * s[k]);
      if (a > amax) amax = a;
    }
    float sc = amax / 127.0f;
    sw[n] = sc;
    for (int64_t k = 0; k < K; ++k) Wq[n * K + k] = oracle_quantize_value(oracle_h2f(W[n * K + k]) * s[k], sc);
  }
}

void onext_smooth_quantize_activations(const uint16_t* X, const float* s, int64_t T, int64_t K,
                                       int8_t* Xq, float* sx) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(oracle_h2f(X[t * K + k]) / s[k]);
      if (a > amax) amax = a;
    }
    float sc = amax / 127.0f;
    sx[t] = sc;
    for (int64_t k = 0; k < K; ++k) Xq[t * K + k] = oracle_quantize_value(oracle_h2f(X[t * K + k]) / s[k], sc);
  }
}

int onext_smoothquant_matmul(const uint16_t* X, const float* s, int64_t T, int64_t K, const int8_t* Wq,
                             const float* sw, int64_t N, uint16_t* Y, int8_t* Xq, float* sx, int32_t* acc) {
  int8_t* own_xq = NULL; float* own_sx = NULL; int32_t* own_acc = NULL;
  int rc = 0;
  if (!Xq) Xq = own_xq = (int8_t*)malloc((size_t)(T * K > 0 ? T * K : 1));
  if (!sx) sx = own_sx = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1));
  if (!acc) acc = own_acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * N > 0 ? T * N : 1));
  if (!Xq || !sx || !acc) {
    rc = -2;
    goto done;
  }
  onext_smooth_quantize_activations(X, s, T, K, Xq, sx);
  rc = oracle_int8_gemm(Xq, Wq, T, N, K, acc);
  oracle_dequant_combine(acc, sx, sw, NULL, T, N, Y);
done:
  free(own_xq); free(own_sx); free(own_acc);
  return rc;
}

/* ================================================================ FP8 E4M3
 * [P5] §3.6: E4M3 = 1 sign, 4 exponent, 3 mantissa bits, the inference
 * format.  The variant keeps the LLM.int8() decomposition ([P1] §2.1) and
 * replaces the 8-bit integer codes by E4M3 codes with absmax scales mapping
 * the largest regular magnitude to the largest finite code, 448. */

float onext_e4m3_to_float(uint8_t c) {
  const int sign = (c >> 7) & 1;
  const int e = (c >> 3) & 0xf;
  const int m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);                  /* subnormal: m * 2^-9 */
  else
    v = ldexp((double)(8 + m), e - 10);        /* (1 + m/8) * 2^(e-7) */
  return (float)(sign ? -v : v);
}

uint8_t onext_float_to_e4m3(float x) {
  if (isnan(x)) return 0x7f;
  const uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7e;          /* saturate to the largest finite, 1.75 * 2^8 */
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: units of 2^-9; q == 8 is the smallest normal (code 8) */
    double q = nearbyint(ldexp(a, 9));
    return sign | (uint8_t)q;
  }
  int ex;
  frexp(a, &ex);                               /* a in [2^(ex-1), 2^ex) */
  int E = ex - 1;
  double q = nearbyint(ldexp(a, 3 - E));       /* in [8, 16] */
  if (q == 16.0) {
    q = 8.0;
    E += 1;
  }
  if (E > 8) return sign | 0x7e;               /* unreachable below 448; kept for clarity */
  return sign | (uint8_t)(((E + 7) << 3) | ((int)q - 8));
}

uint8_t onext_quantize_e4m3(float x, float s) {
  if (s == 0.0f) return 0;
  float r = x / s;                             /* binary32, round to nearest even */
  return onext_float_to_e4m3(r);
}

void onext_fp8_quantize_weight(const uint16_t* W, int64_t N, int64_t K, uint8_t* Wq, float* sw) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(oracle_h2f(W[n * K + k]));
      if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    sw[n] = s;
    for (int64_t k = 0; k < K; ++k) Wq[n * K + k] = onext_quantize_e4m3(oracle_h2f(W[n * K + k]), s);
  }
}

void onext_fp8_quantize_activations(const uint16_t* X, int64_t T, int64_t K, const uint8_t* flag,
                                    uint8_t* Xq, float* sx) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      if (flag[k]) continue;
      float a = fabsf(oracle_h2f(X[t * K + k]));
      if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    sx[t] = s;
    for (int64_t k = 0; k < K; ++k)
      Xq[t * K + k] = flag[k] ? 0 : onext_quantize_e4m3(oracle_h2f(X[t * K + k]), s);
  }
}

void onext_fp8_gemm(const uint8_t* Xq, const uint8_t* Wq, int64_t T, int64_t N, int64_t K, double* acc) {
  /* Each code is decoded once into a binary64 copy; the products and sums
   * are the same (and exact, see next_oracle.h) in any order. */
  double* xd = (double*)malloc(sizeof(double) * (size_t)(T * K > 0 ? T * K : 1));
  double* wd = (double*)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
  if (!xd || !wd) {
    for (int64_t i = 0; i < T * N; ++i) acc[i] = NAN;
    free(xd); free(wd);
    return;
  }
  for (int64_t i = 0; i < T * K; ++i) xd[i] = (double)onext_e4m3_to_float(Xq[i]);
  for (int64_t i = 0; i < N * K; ++i) wd[i] = (double)onext_e4m3_to_float(Wq[i]);
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k) s += xd[t * K + k] * wd[n * K + k];
      acc[t * N + n] = s;
    }
  }
  free(xd); free(wd);
}

int onext_fp8_matmul(const uint16_t* X, int64_t T, int64_t K, const uint8_t* Wq, const float* sw,
                     const uint16_t* W, int64_t N, float tau, uint16_t* Y, uint8_t* flag, int32_t* idx,
                     int64_t* nO_out, uint8_t* Xq, float* sx, double* acc, double* yo) {
  uint8_t* own_flag = NULL; int32_t* own_idx = NULL; uint8_t* own_xq = NULL;
  float* own_sx = NULL; double* own_acc = NULL; double* own_yo = NULL;
  int rc = 0;
  if (!flag) flag = own_flag = (uint8_t*)malloc((size_t)(K > 0 ? K : 1));
  if (!idx) idx = own_idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
  if (!Xq) Xq = own_xq = (uint8_t*)malloc((size_t)(T * K > 0 ? T * K : 1));
  if (!sx) sx = own_sx = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1));
  if (!acc) acc = own_acc = (double*)malloc(sizeof(double) * (size_t)(T * N > 0 ? T * N : 1));
  if (!yo) yo = own_yo = (double*)malloc(sizeof(double) * (size_t)(T * N > 0 ? T * N : 1));
  if (!flag || !idx || !Xq || !sx || !acc || !yo) {
    rc = -2;
    goto done;
  }
  oracle_detect_outliers(X, T, K, tau, flag);
  int64_t nO = oracle_compact(flag, K, idx);
  if (nO_out) *nO_out = nO;
  onext_fp8_quantize_activations(X, T, K, flag, Xq, sx);
  onext_fp8_gemm(Xq, Wq, T, N, K, acc);
  oracle_outlier_gemm(X, W, T, N, K, idx, nO, yo);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t n = 0; n < N; ++n)
      Y[t * N + n] = oracle_d2h(acc[t * N + n] * (double)sx[t] * (double)sw[n] + yo[t * N + n]);
done:
  free(own_flag); free(own_idx); free(own_xq); free(own_sx); free(own_acc); free(own_yo);
  return rc;
}

/* ================================================================ stored outlier columns
 * [P1] §2.2: the point of 8-bit weights is memory (26 GB -> about 13 GB at
 * 13B), while [P1] §2.1 keeps the outlier columns' weights in fp16.  Here the
 * fp16 weights are kept only for a chosen set of columns; an outlier column
 * outside that set uses the fp16 value of its dequantised int8 weight (the
 * closest thing to its fp16 weight the call still holds) and counts as a miss. */

uint16_t onext_reconstruct_weight(int8_t q, float s) {
  float p = s * (float)q;                      /* binary32, round to nearest even */
  return oracle_d2h((double)p);
}

int64_t onext_outlier_gemm_stored(const uint16_t* X, const int8_t* Wq, const float* sw, const int32_t* slot,
                                  const uint16_t* Wst, int64_t T, int64_t N, int64_t K, const int32_t* idx,
                                  int64_t nO, double* yo) {
  int64_t miss = 0;
  for (int64_t j = 0; j < nO; ++j)
    if (slot[idx[j]] < 0) ++miss;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t j = 0; j < nO; ++j) {
        const int64_t k = idx[j];
        const int32_t sl = slot[k];
        const uint16_t w = sl >= 0 ? Wst[(int64_t)sl * N + n] : onext_reconstruct_weight(Wq[n * K + k], sw[n]);
        s += (double)oracle_h2f(X[t * K + k]) * (double)oracle_h2f(w);
      }
      yo[t * N + n] = s;
    }
  }
  return miss;
}

int onext_matmul_stored(const uint16_t* X, int64_t T, int64_t K, const int8_t* Wq, const float* sw,
                        const int32_t* slot, const uint16_t* Wst, int64_t N, float tau, uint16_t* Y,
                        int64_t* n_miss) {
  uint8_t* flag = (uint8_t*)malloc((size_t)(K > 0 ? K : 1));
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
  int8_t* Xq = (int8_t*)malloc((size_t)(T * K > 0 ? T * K : 1));
  float* sx = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1));
  int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * N > 0 ? T * N : 1));
  double* yo = (double*)malloc(sizeof(double) * (size_t)(T * N > 0 ? T * N : 1));
  int rc = 0;
  if (!flag || !idx || !Xq || !sx || !acc || !yo) {
    rc = -2;
    goto done;
  }
  oracle_detect_outliers(X, T, K, tau, flag);
  int64_t nO = oracle_compact(flag, K, idx);
  oracle_quantize_activations(X, T, K, flag, Xq, sx);
  rc = oracle_int8_gemm(Xq, Wq, T, N, K, acc);
  int64_t m = onext_outlier_gemm_stored(X, Wq, sw, slot, Wst, T, N, K, idx, nO, yo);
  if (n_miss) *n_miss = m;
  oracle_dequant_combine(acc, sx, sw, yo, T, N, Y);
done:
  free(flag); free(idx); free(Xq); free(sx); free(acc); free(yo);
  return rc;
}
