/*
 * gen.c -- seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.
 *
 * This module holds no quantization or GEMM arithmetic: it only draws numbers.
 *
 * Generator: counter-based SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014: the 64-bit finaliser "mix64" applied to a
 * Weyl sequence). Value i of stream s under seed q is mix64(key(q, s) + (i + 1) * gamma), so any
 * slice of a tensor can be generated independently and in parallel.
 * Normals: Box-Muller (one normal per pair of uniforms). Student-t(3): Z / sqrt(chi2_3 / 3).
 * Values go double -> fp32 (round to nearest) -> bf16 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t gen_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed + GAMMA) ^ (stream * 0xD1B54A32D192ED03ULL));
}

uint64_t gen_draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

/* uniform on the open interval (0, 1) */
double gen_u01(uint64_t key, uint64_t i) { return ((double)(gen_draw(key, i) >> 11) + 0.5) * 0x1.0p-53; }

double gen_normal(uint64_t key, uint64_t i) {
  double u1 = gen_u01(key, 2 * i), u2 = gen_u01(key, 2 * i + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

double gen_student_t3(uint64_t key, uint64_t i) {
  double z = gen_normal(key, 4 * i);
  double c = 0.0;
  for (int j = 1; j <= 3; ++j) {
    double n = gen_normal(key, 4 * i + j);
    c += n * n;
  }
  return z / sqrt(c / 3.0);
}

static uint16_t to_bf16(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * Rows [r0, r1) of a [rows, cols] bf16 matrix, element (m, k) drawn at counter m*cols + k.
 * dist 0: normal(0, std); dist 1: std * Student-t(3). col_mult (nullable, length cols) scales
 * whole columns (outlier channels) before rounding. out points at row r0, row stride ld.
 */
void gen_matrix_bf16(uint64_t seed, uint64_t stream, int dist, int64_t cols, double stdv, const double* col_mult,
                     int64_t r0, int64_t r1, uint16_t* out, int64_t ld) {
  uint64_t key = gen_key(seed, stream);
  for (int64_t m = r0; m < r1; ++m)
    for (int64_t k = 0; k < cols; ++k) {
      uint64_t i = (uint64_t)(m * cols + k);
      double v = (dist == 1) ? gen_student_t3(key, i) : gen_normal(key, i);
      v *= stdv;
      if (col_mult) v *= col_mult[k];
      out[(m - r0) * ld + k] = to_bf16(v);
    }
}

/* n distinct channels out of [0, K): the first n slots of a partial Fisher-Yates shuffle. */
void gen_channel_set(uint64_t seed, uint64_t stream, int64_t K, int64_t n, int32_t* perm_scratch, int32_t* out) {
  uint64_t key = gen_key(seed, stream);
  for (int64_t k = 0; k < K; ++k) perm_scratch[k] = (int32_t)k;
  for (int64_t i = 0; i < n; ++i) {
    int64_t j = i + (int64_t)(gen_draw(key, (uint64_t)i) % (uint64_t)(K - i));
    int32_t t = perm_scratch[i];
    perm_scratch[i] = perm_scratch[j];
    perm_scratch[j] = t;
    out[i] = perm_scratch[i];
  }
}

/* n log-uniform magnitudes in [lo, hi]: lo * (hi/lo)^U. */
void gen_log_uniform(uint64_t seed, uint64_t stream, int64_t n, double lo, double hi, double* out) {
  uint64_t key = gen_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = lo * pow(hi / lo, gen_u01(key, (uint64_t)i));
}
