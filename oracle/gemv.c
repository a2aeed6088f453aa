/*
 * Float64 matrix-vector products for the CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY: called by oracle/model.py, never by the product
 * path.  Each function is the definition y[n] = sum_k w[n][k] * x[k] written
 * out with a float64 accumulator, rows in parallel; nothing is blocked or
 * reordered beyond the row split.  The FP8 variant takes the 256-entry E4M3
 * value table from oracle/numerics.py (pinned there against the format
 * definition) and applies the per-128x128-block scale to each weight:
 * w[n][k] = E4M3(q[n][k]) * s[n/128][k/128].
 */
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_gemv_f32(const float* W, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) acc += (double)w[k] * x[k];
    y[n] = acc;
  }
}

void oracle_gemv_bf16(const uint16_t* W, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint16_t* w = W + n * K;
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      uint32_t u = (uint32_t)w[k] << 16; /* bf16 = upper half of binary32 */
      float f;
      memcpy(&f, &u, 4);
      acc += (double)f * x[k];
    }
    y[n] = acc;
  }
}

void oracle_gemv_fp8(const uint8_t* q, const float* s, int64_t N, int64_t K, const double* table, const double* x,
                     double* y) {
  const int64_t nbc = (K + 127) / 128;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* w = q + n * K;
    const float* srow = s + (n / 128) * nbc;
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) acc += table[w[k]] * (double)srow[k / 128] * x[k];
    y[n] = acc;
  }
}

/*
 * Float32-accumulation twins.  NOT the definition: the same products, summed
 * in a float32 accumulator per 128-column block and the blocks then added in
 * float32, as an implementation that accumulates in float32 would.  Tests use
 * them only to measure how far such an implementation can land from the
 * float64 definition on a chaotic random-init model (a calibration of the
 * end-to-end tolerance); no expected value is ever taken from them.
 */
void oracle_gemv_f32_acc32(const float* W, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    float acc = 0.f;
    for (int64_t k0 = 0; k0 < K; k0 += 128) {
      float part = 0.f;
      for (int64_t k = k0; k < K && k < k0 + 128; ++k) part += w[k] * (float)x[k];
      acc += part;
    }
    y[n] = acc;
  }
}

void oracle_gemv_bf16_acc32(const uint16_t* W, int64_t N, int64_t K, const double* x, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint16_t* w = W + n * K;
    float acc = 0.f;
    for (int64_t k0 = 0; k0 < K; k0 += 128) {
      float part = 0.f;
      for (int64_t k = k0; k < K && k < k0 + 128; ++k) {
        uint32_t u = (uint32_t)w[k] << 16;
        float f;
        memcpy(&f, &u, 4);
        part += f * (float)x[k];
      }
      acc += part;
    }
    y[n] = acc;
  }
}

void oracle_gemv_fp8_acc32(const uint8_t* q, const float* s, int64_t N, int64_t K, const double* table,
                           const double* x, double* y) {
  const int64_t nbc = (K + 127) / 128;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* w = q + n * K;
    const float* srow = s + (n / 128) * nbc;
    float acc = 0.f;
    for (int64_t b = 0; b < nbc; ++b) {
      float part = 0.f;
      for (int64_t k = b * 128; k < K && k < b * 128 + 128; ++k) part += (float)table[w[k]] * (float)x[k];
      acc += part * srow[b];
    }
    y[n] = acc;
  }
}
