/*
 * llmint8_oracle.c -- plain CPU statement of the LLM.int8() matmul.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline of the bench).
 * Shares no code with the CUDA library.  See llmint8_oracle.h for the sources,
 * layouts and precision rules.  Scalar loops, no blocking or reordering beyond
 * what the method states; OpenMP splits independent output rows only, which
 * leaves every result unchanged.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fopenmp -fPIC -shared
 * (x86-64 SSE arithmetic, so binary32 operations round once, to nearest even).
 */
#include "llmint8_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- IEEE binary16 <-> value, written from the format's definition ---- */

float oracle_h2f(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1f;
  const int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
  }
  return (float)(sign ? -v : v);
}

uint16_t oracle_d2h(double v) {
  if (isnan(v)) return 0x7e00;
  const uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  /* 65504 is the largest finite half; 65520 lies half-way to 2^16 and rounds
   * (to even) away to infinity. */
  if (a >= 65520.0) return sign | 0x7c00;
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: units of 2^-24; a result of 1024 is the smallest normal */
    double q = nearbyint(ldexp(a, 24));
    return sign | (uint16_t)q;
  }
  int ex;
  frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1)  =>  a in [2^(ex-1), 2^ex) */
  int E = ex - 1;
  double q = nearbyint(ldexp(a, 10 - E));      /* in [1024, 2048] */
  if (q == 2048.0) {
    q = 1024.0;
    E += 1;
  }
  if (E + 15 >= 31) return sign | 0x7c00;
  return sign | (uint16_t)(((E + 15) << 10) | ((int)q - 1024));
}

void oracle_h2f_array(const uint16_t* h, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_h2f(h[i]);
}

void oracle_d2h_array(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_d2h(v[i]);
}

/* ---- symmetric absmax int8 ([P2] Q2: q = round(r/s), s = max|r| / (2^(b-1)-1);
 *      [P5] §2.1: scale = max_val / 127, round, clip) ---- */

int8_t oracle_quantize_value(float x, float s) {
  if (s == 0.0f) return 0;
  float r = x / s;                /* binary32, round to nearest even */
  float q = nearbyintf(r);        /* ties to even in the default rounding mode */
  if (q > 127.0f) q = 127.0f;
  if (q < -127.0f) q = -127.0f;
  return (int8_t)q;
}

/* a0 -- [P1] §2.1: one scale per output feature of the weight matrix. */
void oracle_quantize_weight(const uint16_t* W, int64_t N, int64_t K, int8_t* Wq, float* sw) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint16_t* row = W + n * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(oracle_h2f(row[k]));
      if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    sw[n] = s;
    for (int64_t k = 0; k < K; ++k) Wq[n * K + k] = oracle_quantize_value(oracle_h2f(row[k]), s);
  }
}

/* a1 -- [P1] §2.1: a feature dim whose activation magnitude reaches the
 * threshold (6.0) is an outlier; the whole column leaves the int8 product. */
void oracle_detect_outliers(const uint16_t* X, int64_t T, int64_t K, float tau, uint8_t* flag) {
  memset(flag, 0, (size_t)K);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t k = 0; k < K; ++k)
      if (fabsf(oracle_h2f(X[t * K + k])) >= tau) flag[k] = 1;
}

int64_t oracle_compact(const uint8_t* flag, int64_t K, int32_t* idx) {
  int64_t n = 0;
  for (int64_t k = 0; k < K; ++k)
    if (flag[k]) idx[n++] = (int32_t)k;
  return n;
}

/* a2 + a3 -- per-row absmax over the regular columns only, so that an outlier
 * no longer sets the scale ([P1] §1), then the int8 codes. */
void oracle_quantize_activations(const uint16_t* X, int64_t T, int64_t K, const uint8_t* flag,
                                 int8_t* Xq, float* sx) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const uint16_t* row = X + t * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      if (flag[k]) continue;
      float a = fabsf(oracle_h2f(row[k]));
      if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    sx[t] = s;
    for (int64_t k = 0; k < K; ++k)
      Xq[t * K + k] = flag[k] ? 0 : oracle_quantize_value(oracle_h2f(row[k]), s);
  }
}

/* a5 -- int8 x int8 products summed exactly. */
int oracle_int8_gemm(const int8_t* Xq, const int8_t* Wq, int64_t T, int64_t N, int64_t K,
                     int32_t* acc) {
  int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : overflow)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* a = Xq + t * K;
      const int8_t* b = Wq + n * K;
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
      acc[t * N + n] = (int32_t)(uint32_t)(uint64_t)s;
    }
  }
  return overflow ? -1 : 0;
}

/* a6 -- the outlier columns multiplied at full precision ([P1] §2.1 and
 * [P2] Q4 keep them in fp16; every fp16 product is exact in binary64). */
void oracle_outlier_gemm(const uint16_t* X, const uint16_t* W, int64_t T, int64_t N, int64_t K,
                         const int32_t* idx, int64_t nO, double* yo) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t j = 0; j < nO; ++j) {
        int64_t k = idx[j];
        s += (double)oracle_h2f(X[t * K + k]) * (double)oracle_h2f(W[n * K + k]);
      }
      yo[t * N + n] = s;
    }
  }
}

/* a7 -- dequantise by both scales ([P2] Q2: r' = s * q, on each operand) and
 * add the outlier part; one rounding to fp16 ([P1] §2.1: the two partial
 * results are summed to give the output in fp16). */
void oracle_dequant_combine(const int32_t* acc, const float* sx, const float* sw, const double* yo,
                            int64_t T, int64_t N, uint16_t* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      double v = (double)acc[t * N + n] * (double)sx[t] * (double)sw[n];
      if (yo) v += yo[t * N + n];
      Y[t * N + n] = oracle_d2h(v);
    }
  }
}

int oracle_matmul(const uint16_t* X, int64_t T, int64_t K, const int8_t* Wq, const float* sw,
                  const uint16_t* W, int64_t N, float tau, uint16_t* Y,
                  uint8_t* flag, int32_t* idx, int64_t* nO_out, int8_t* Xq, float* sx,
                  int32_t* acc, double* yo) {
  uint8_t* own_flag = NULL; int32_t* own_idx = NULL; int8_t* own_xq = NULL;
  float* own_sx = NULL; int32_t* own_acc = NULL; double* own_yo = NULL;
  int rc = 0;
  if (!flag) flag = own_flag = (uint8_t*)malloc((size_t)(K > 0 ? K : 1));
  if (!idx) idx = own_idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
  if (!Xq) Xq = own_xq = (int8_t*)malloc((size_t)(T * K > 0 ? T * K : 1));
  if (!sx) sx = own_sx = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1));
  if (!acc) acc = own_acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * N > 0 ? T * N : 1));
  if (!yo) yo = own_yo = (double*)malloc(sizeof(double) * (size_t)(T * N > 0 ? T * N : 1));
  if (!flag || !idx || !Xq || !sx || !acc || !yo) {
    rc = -2;
    goto done;
  }
  oracle_detect_outliers(X, T, K, tau, flag);                     /* a1 */
  int64_t nO = oracle_compact(flag, K, idx);                       /* a4 */
  if (nO_out) *nO_out = nO;
  oracle_quantize_activations(X, T, K, flag, Xq, sx);              /* a2, a3 */
  rc = oracle_int8_gemm(Xq, Wq, T, N, K, acc);                     /* a5 */
  oracle_outlier_gemm(X, W, T, N, K, idx, nO, yo);                 /* a6 */
  oracle_dequant_combine(acc, sx, sw, yo, T, N, Y);                /* a7 */
done:
  free(own_flag); free(own_idx); free(own_xq); free(own_sx); free(own_acc); free(own_yo);
  return rc;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
