/*
 * arc_oracle.c -- CPU oracle for NVFP4 quantization with augmented residual channels (ARC),
 * the block-scaled GEMM over the augmented operands, the BF16 switch and the pieces of the
 * recurrent SwiGLU block.
 *
 * TEST INFRASTRUCTURE. This library exists to check the CUDA path. Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark load it. It shares no code, header,
 * table or constant generator with the CUDA library, and the CUDA library never calls it.
 *
 * Precision contract (where the pages fix nothing the reading is stated at each function):
 *   every float operation is IEEE binary32 round-to-nearest-even, no FMA contraction
 *   (build with -ffp-contract=off, no fast-math), no flush-to-zero; GEMM sums are FP64 or
 *   exact int64.
 *
 * Sources (page title, then section):
 *   [ARC]  "ARCQuant: Boosting NVFP4 Quantization with Augmented Residual Channels for LLMs"
 *          (gist.science explainer), Technische Samenvatting -> Methodologie:
 *          "Adaptieve Uitschieter-identificatie", "Dual-Stage Quantisatie",
 *          "Augmented Matrixvermenigvuldiging", "Unified GEMM Executie", "Kernel Implementatie";
 *          and the problem statement on NVFP4 block size 16.
 *   [DAY0] "Day 0 LLM Inference Support: Hierarchical Quantization and Memory Access
 *          Optimization Practices", section V (Engineering Implementation Details): item 4
 *          (numerical safety: all-zero groups, clipping to the format range) and the per-group
 *          dynamic quantization pseudo-code (scale = amax / FMT_MAX, zero guard, clip).
 *   [RAMP] "RAMP: Recurrent Adaptive Mixed Precision for Efficient Prefill in Recurrent-Depth
 *          Language Models", section 2.1 (shared block applied repeatedly), 4.1 (switch from low
 *          to reference precision at step K), 4.2 (hidden state and surrounding ops stay BF16).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                                               */
/* ------------------------------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round-to-nearest-even fp32 -> bf16 (finite inputs; NaN maps to a quiet NaN). */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

float oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }
uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16(f); }

/* ------------------------------------------------------------------------------------------ */
/* E2M1 (the 4-bit NVFP4 element): [ARC] "E2M1 mantissa"                                       */
/* ------------------------------------------------------------------------------------------ */

/* The eight magnitudes of E2M1 (1 sign, 2 exponent, 1 mantissa bit, bias 1): codes 0..7. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float oracle_e2m1_decode(uint8_t code) {
  double m = E2M1_MAG[code & 7];
  return (float)((code & 8) ? -m : m);
}

/*
 * Encode v as the nearest E2M1 value, ties to the even code, magnitudes beyond 6 saturate to
 * 6 (the "clip to the representable range" rule of [DAY0] item 4). The sign bit follows the
 * sign of v also when the magnitude rounds to zero (-0.1 -> 0x8): this is IEEE rounding of a
 * signed value and is the reading this build takes where the pages say nothing.
 * Implementation: exhaustive nearest search over the eight magnitudes (distances in double,
 * exact for the neighbours that matter).
 */
uint8_t oracle_e2m1_encode(float v) {
  int neg = signbit(v) ? 1 : 0;
  double a = fabs((double)v);
  int best = 0;
  if (a >= 6.0) {
    best = 7;
  } else {
    double bestd = a;  /* distance to magnitude 0 */
    for (int i = 1; i < 8; ++i) {
      double d = fabs(a - E2M1_MAG[i]);
      if (d < bestd || (d == bestd && (i & 1) == 0 && (best & 1) == 1)) {
        best = i;
        bestd = d;
      }
    }
  }
  return (uint8_t)((neg << 3) | best);
}

/* ------------------------------------------------------------------------------------------ */
/* E4M3 block scale (unsigned use): bias 7, 3 mantissa bits, subnormal step 2^-9, max 448,     */
/* code 0x7F is NaN and never produced. [DAY0] pseudo-code: FP8_MAX = 448.                      */
/* ------------------------------------------------------------------------------------------ */

float oracle_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 7;
  double v;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  if (e == 15 && m == 7) v = NAN;
  return (float)(s ? -v : v);
}

/*
 * Nearest E4M3 value to v >= 0, ties to the even code, values at or above 448 saturate to
 * 448 (0x7E). Linear search over the 127 non-negative finite codes in value order; it stops
 * once the distance grows.
 */
uint8_t oracle_e4m3_encode_nonneg(float v) {
  double a = (double)v;
  if (!(a > 0.0)) return 0; /* +0, -0 and (never expected) negatives encode as 0 */
  if (a >= 448.0) return 0x7E;
  int best = 0;
  double bestd = a;
  for (int c = 1; c <= 0x7E; ++c) {
    double d = fabs(a - (double)oracle_e4m3_decode((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    } else if (d > bestd) {
      break; /* values grow with the code, so distances only grow from here */
    }
  }
  return (uint8_t)best;
}

/* ------------------------------------------------------------------------------------------ */
/* Per-tensor scale: scale = amax / FMT_MAX with the all-zero guard ([DAY0] pseudo-code), where */
/* FMT_MAX of the two-level NVFP4 code is 6 (largest E2M1) * 448 (largest E4M3) = 2688.         */
/* ------------------------------------------------------------------------------------------ */

float oracle_tensor_scale(float amax) { return amax > 0.0f ? amax / 2688.0f : 1.0f; }

/* max |x| over a bf16 matrix [rows, cols] with row stride ld (elements). */
float oracle_amax_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
  float m = 0.0f;
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t k = 0; k < cols; ++k) {
      float a = fabsf(bf16_to_f32(x[i * ld + k]));
      if (a > m) m = a;
    }
  return m;
}

/* ------------------------------------------------------------------------------------------ */
/* One 16-element NVFP4 block ([ARC] block size 16; [DAY0] scale = amax / FMT_MAX, zero guard).  */
/*   sf = E4M3( (amax_b / 6) / s_t )     two fp32 divides                                       */
/*   d  = E4M3value(sf) * s_t            fp32 multiply (the block's decode scale)               */
/*   q_i = E2M1( x_i / d ), or 0 for all i when d == 0 (all-zero / underflowed group)           */
/* ------------------------------------------------------------------------------------------ */

static void encode_block(const float* x, float s_t, uint8_t* codes16, uint8_t* sf_out, float* d_out) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  float t = amax / 6.0f;
  t = t / s_t;
  uint8_t sf = oracle_e4m3_encode_nonneg(t);
  float d = oracle_e4m3_decode(sf) * s_t;
  for (int i = 0; i < 16; ++i) codes16[i] = (d == 0.0f) ? 0 : oracle_e2m1_encode(x[i] / d);
  *sf_out = sf;
  if (d_out) *d_out = d;
}

void oracle_encode_block(const float* x16, float s_t, uint8_t* codes16, uint8_t* sf, float* d) {
  encode_block(x16, s_t, codes16, sf, d);
}

static int64_t kpad_of(int64_t k_aug) { return (k_aug + 63) / 64 * 64; }
int64_t oracle_kpad(int64_t k_aug) { return kpad_of(k_aug); }

static void put_code(uint8_t* row_codes, int64_t k, uint8_t c) {
  /* element k lives in byte k/2; even k in the low nibble */
  uint8_t* b = &row_codes[k >> 1];
  if (k & 1)
    *b = (uint8_t)((*b & 0x0F) | (c << 4));
  else
    *b = (uint8_t)((*b & 0xF0) | (c & 0x0F));
}

uint8_t oracle_get_code(const uint8_t* row_codes, int64_t k) {
  uint8_t b = row_codes[k >> 1];
  return (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0x0F);
}

/* ------------------------------------------------------------------------------------------ */
/* RMSNorm prologue ([ARC] Kernel Implementatie: RMSNorm fused before quantization).             */
/* Reading: n_i = bf16( fp32( (h_i * inv) * g_i ) ) with inv = 1 / sqrt(ss/d + eps) in double   */
/* and ss = sum of h_i^2 computed exactly (then rounded once to double), so the statistic does  */
/* not depend on summation order. Exact sum: every bf16 square is m^2 * 2^(2e-268) with m < 256;*/
/* the squares are accumulated as a 128-bit integer in units of 2^(2*emax-268-94), emax the     */
/* largest biased exponent in the row; squares more than 2^94 below the largest are truncated   */
/* (never the case for rows spanning fewer than 47 binades).                                     */
/* ------------------------------------------------------------------------------------------ */

/* Round-to-nearest-even conversion of an unsigned 128-bit integer times 2^e2 to double. */
static double u128_to_double_scaled(unsigned __int128 v, int e2) {
  if (v == 0) return 0.0;
  int p = 127;
  while (!((v >> p) & 1)) --p;
  if (p <= 52) return ldexp((double)(uint64_t)v, e2);
  int sh = p - 52;
  unsigned __int128 mant = v >> sh;
  unsigned __int128 rem = v & ((((unsigned __int128)1) << sh) - 1);
  unsigned __int128 half = ((unsigned __int128)1) << (sh - 1);
  if (rem > half || (rem == half && (mant & 1))) mant += 1;
  return ldexp((double)(uint64_t)mant, e2 + sh);
}

double oracle_row_sumsq(const uint16_t* h, int64_t d) {
  int emax = 0;
  for (int64_t i = 0; i < d; ++i) {
    int e = (h[i] >> 7) & 0xFF;
    if ((h[i] & 0x7FFF) == 0) continue;
    if (e == 0) e = 1;
    if (e > emax) emax = e;
  }
  if (emax == 0) return 0.0;
  unsigned __int128 acc = 0;
  for (int64_t i = 0; i < d; ++i) {
    uint16_t b = h[i] & 0x7FFF;
    if (b == 0) continue;
    int e = (b >> 7) & 0xFF;
    uint32_t m = b & 0x7F;
    if (e == 0)
      e = 1;
    else
      m |= 0x80;
    uint64_t sq = (uint64_t)m * m;
    int sh = 2 * (e - emax) + 94;
    if (sh >= 0)
      acc += ((unsigned __int128)sq) << sh;
    else if (sh > -64)
      acc += (unsigned __int128)(sq >> (-sh));
  }
  return u128_to_double_scaled(acc, 2 * emax - 268 - 94);
}

double oracle_rms_inv(const uint16_t* h, int64_t d, double eps) {
  double ss = oracle_row_sumsq(h, d);
  double ms = ss / (double)d;
  return 1.0 / sqrt(ms + eps);
}

/* n = RMSNorm(h) * g, one row, written as bf16 bits. g may be NULL (all ones). */
void oracle_rmsnorm_row(const uint16_t* h, const uint16_t* g, int64_t d, double eps, uint16_t* out) {
  double inv = oracle_rms_inv(h, d, eps);
  for (int64_t i = 0; i < d; ++i) {
    double v = (double)bf16_to_f32(h[i]) * inv;
    if (g) v = v * (double)bf16_to_f32(g[i]);
    out[i] = f32_to_bf16((float)v);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Activation quantization with augmented residual channels ([ARC] Dual-Stage Quantisatie,     */
/* Augmented Matrixvermenigvuldiging).                                                          */
/*   primary stage: blocks of 16 consecutive channels k = 16b..16b+15, b < K/16                  */
/*   residual stage: for j < r, c = idx[j]: res_j = x_c - E2M1value(q_c) * d_block(c)           */
/*                   (fp32 multiply then fp32 subtract); res values in idx order form r/16       */
/*                   blocks quantized with the same tensor scale s_t, written at K + j           */
/*   padding: columns K+r .. K_pad-1 carry code 0 and scale 0 (K_pad = K+r rounded up to 64)     */
/* Outputs (canonical, unswizzled): codes [rows, K_pad/2] bytes, sf [rows, K_pad/16] bytes.      */
/* rms_g: NULL = no RMSNorm prologue; otherwise the row is RMS-normalised first (rms_g may      */
/* point to the gain vector, or to a one-element sentinel when use_ones != 0).                  */
/* res_out (optional): [rows, r] fp32 residual values, for tests.                               */
/* Rows [m0, m1) only, so callers can split rows across threads.                                 */
/* ------------------------------------------------------------------------------------------ */

static void quantize_rows_impl(const uint16_t* x, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                               int dup_mode, int rms, const uint16_t* rms_g, double eps, float s_t,
                               uint8_t* codes, uint8_t* sf, float* res_out, int64_t m0, int64_t m1) {
  int64_t kaug = K + r, kpad = kpad_of(kaug);
  float* row = (float*)malloc(sizeof(float) * (size_t)K);
  float* d_blk = (float*)malloc(sizeof(float) * (size_t)(K / 16 + 1));
  uint16_t* nrm = rms ? (uint16_t*)malloc(sizeof(uint16_t) * (size_t)K) : NULL;
  float ext[16];
  uint8_t c16[16];
  for (int64_t m = m0; m < m1; ++m) {
    const uint16_t* xr = x + m * ldx;
    if (rms) {
      oracle_rmsnorm_row(xr, rms_g, K, eps, nrm);
      xr = nrm;
    }
    for (int64_t k = 0; k < K; ++k) row[k] = bf16_to_f32(xr[k]);
    uint8_t* crow = codes + m * (kpad / 2);
    uint8_t* srow = sf + m * (kpad / 16);
    memset(crow, 0, (size_t)(kpad / 2));
    memset(srow, 0, (size_t)(kpad / 16));
    /* primary stage */
    for (int64_t b = 0; b < K / 16; ++b) {
      uint8_t s;
      encode_block(row + 16 * b, s_t, c16, &s, &d_blk[b]);
      srow[b] = s;
      for (int i = 0; i < 16; ++i) put_code(crow, 16 * b + i, c16[i]);
    }
    /* residual (activations) or duplicated columns (weights), in idx order */
    for (int32_t jb = 0; jb < r / 16; ++jb) {
      for (int i = 0; i < 16; ++i) {
        int32_t c = idx[16 * jb + i];
        if (dup_mode) {
          ext[i] = row[c];
        } else {
          float deq = oracle_e2m1_decode(oracle_get_code(crow, c)) * d_blk[c / 16];
          ext[i] = row[c] - deq;
        }
        if (res_out) res_out[m * r + 16 * jb + i] = ext[i];
      }
      uint8_t s;
      encode_block(ext, s_t, c16, &s, NULL);
      srow[K / 16 + jb] = s;
      for (int i = 0; i < 16; ++i) put_code(crow, K + 16 * jb + i, c16[i]);
    }
  }
  free(row);
  free(d_blk);
  free(nrm);
}

void oracle_quantize_act_rows(const uint16_t* x, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                              const uint16_t* rms_g, int32_t use_rms, double eps, float s_t, uint8_t* codes,
                              uint8_t* sf, float* res_out, int64_t m0, int64_t m1) {
  quantize_rows_impl(x, K, ldx, idx, r, 0, use_rms, rms_g, eps, s_t, codes, sf, res_out, m0, m1);
}

/* Weights ([ARC] "de bijbehorende gewichten gedupliceerd"): W_aug = [W | W[:, idx]], then the
 * same block code on each augmented row with the weight tensor scale s_W. */
void oracle_pack_weight_rows(const uint16_t* w, int64_t K, int64_t ldw, const int32_t* idx, int32_t r,
                             float s_w, uint8_t* codes, uint8_t* sf, int64_t n0, int64_t n1) {
  quantize_rows_impl(w, K, ldw, idx, r, 1, 0, NULL, 0.0, s_w, codes, sf, NULL, n0, n1);
}

/* Dequantize canonical rows without the tensor scale: out[m, k] = E2M1value * E4M3value. */
void oracle_dequant_rows(const uint8_t* codes, const uint8_t* sf, int64_t kpad, float* out, int64_t m0,
                         int64_t m1) {
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t k = 0; k < kpad; ++k)
      out[m * kpad + k] = oracle_e2m1_decode(oracle_get_code(codes + m * (kpad / 2), k)) *
                          oracle_e4m3_decode(sf[m * (kpad / 16) + k / 16]);
}

/* ------------------------------------------------------------------------------------------ */
/* Scale-factor layout consumed by the tensor cores (the "interleaved layout ready for the     */
/* GEMM" of [ARC] Kernel Implementatie; [DAY0] item 2 asks for scales laid out for vectorised   */
/* loads in the main loop). The pages fix no layout; this build's layout:                       */
/*   atoms of 128 rows x 4 scale bytes (64 K-elements) = 512 bytes;                             */
/*   atom (i, j) for rows 128i.., scale columns 4j.. sits at byte (i * ceil(nsf/4) + j) * 512;  */
/*   inside the atom, row m and scale column kb go to (m%32)*16 + ((m/32)%4)*4 + kb%4.           */
/*   Rows are padded to a multiple of 128 with zero bytes.                                       */
/* ------------------------------------------------------------------------------------------ */

static int64_t swz_off(int64_t m, int64_t kb, int64_t nsf) {
  int64_t katoms = (nsf + 3) / 4;
  return ((m / 128) * katoms + kb / 4) * 512 + (m % 32) * 16 + ((m / 32) % 4) * 4 + (kb % 4);
}

int64_t oracle_sf_swizzled_bytes(int64_t rows, int64_t nsf) { return (rows + 127) / 128 * ((nsf + 3) / 4) * 512; }

void oracle_sf_swizzle(const uint8_t* canon, int64_t rows, int64_t nsf, uint8_t* swz) {
  memset(swz, 0, (size_t)oracle_sf_swizzled_bytes(rows, nsf));
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t kb = 0; kb < nsf; ++kb) swz[swz_off(m, kb, nsf)] = canon[m * nsf + kb];
}

void oracle_sf_unswizzle(const uint8_t* swz, int64_t rows, int64_t nsf, uint8_t* canon) {
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t kb = 0; kb < nsf; ++kb) canon[m * nsf + kb] = swz[swz_off(m, kb, nsf)];
}

/* ------------------------------------------------------------------------------------------ */
/* GEMM of depth K_aug over the augmented operands ([ARC] Unified GEMM Executie: one GEMM of     */
/* shape (N, K_in + S, M); linearity of accumulation adds main and correction terms).            */
/*   Y[m, n] = s_A * s_W * sum_k (E2M1(a_mk) sfA_m,k/16) (E2M1(b_nk) sfB_n,k/16), FP64 sum.       */
/* Rows rows[0..nrows) of A (a list, so tests can sample), all N columns.                        */
/* ------------------------------------------------------------------------------------------ */

void oracle_gemm_nvfp4_f64(const uint8_t* a_codes, const uint8_t* a_sf, float s_a, const uint8_t* b_codes,
                           const uint8_t* b_sf, float s_b, int64_t N, int64_t kpad, const int64_t* rows,
                           int64_t nrows, int64_t k_lo, int64_t k_hi, double* y) {
  double* av = (double*)malloc(sizeof(double) * (size_t)kpad);
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t m = rows[t];
    for (int64_t k = k_lo; k < k_hi; ++k)
      av[k] = (double)oracle_e2m1_decode(oracle_get_code(a_codes + m * (kpad / 2), k)) *
              (double)oracle_e4m3_decode(a_sf[m * (kpad / 16) + k / 16]);
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* bc = b_codes + n * (kpad / 2);
      const uint8_t* bs = b_sf + n * (kpad / 16);
      double acc = 0.0;
      for (int64_t k = k_lo; k < k_hi; ++k)
        acc += av[k] * (double)oracle_e2m1_decode(oracle_get_code(bc, k)) * (double)oracle_e4m3_decode(bs[k / 16]);
      y[t * N + n] = (double)s_a * (double)s_b * acc;
    }
  }
  free(av);
}

/* Exact integer form: a' = 2*E2M1 * 512*E4M3 is an integer (|a'| < 2^22); the sum of a'b' over
 * k in [k_lo, k_hi) fits int64 for K_aug < 2^15. Y = sum * 2^-20 * s_A * s_W. */
void oracle_gemm_nvfp4_i64(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes,
                           const uint8_t* b_sf, int64_t N, int64_t kpad, const int64_t* rows, int64_t nrows,
                           int64_t k_lo, int64_t k_hi, int64_t* y) {
  int64_t* av = (int64_t*)malloc(sizeof(int64_t) * (size_t)kpad);
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t m = rows[t];
    for (int64_t k = k_lo; k < k_hi; ++k)
      av[k] = (int64_t)llround(2.0 * oracle_e2m1_decode(oracle_get_code(a_codes + m * (kpad / 2), k))) *
              (int64_t)llround(512.0 * oracle_e4m3_decode(a_sf[m * (kpad / 16) + k / 16]));
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* bc = b_codes + n * (kpad / 2);
      const uint8_t* bs = b_sf + n * (kpad / 16);
      int64_t acc = 0;
      for (int64_t k = k_lo; k < k_hi; ++k)
        acc += av[k] * (int64_t)llround(2.0 * oracle_e2m1_decode(oracle_get_code(bc, k))) *
               (int64_t)llround(512.0 * oracle_e4m3_decode(bs[k / 16]));
      y[t * N + n] = acc;
    }
  }
  free(av);
}

/* BF16 switch ([RAMP] 4.1/4.2 reference precision): Y = X W^T over bf16 inputs, FP64 sum. */
void oracle_gemm_bf16_f64(const uint16_t* x, int64_t ldx, const uint16_t* w, int64_t ldw, int64_t N, int64_t K,
                          const int64_t* rows, int64_t nrows, double* y) {
  double* xv = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t m = rows[t];
    for (int64_t k = 0; k < K; ++k) xv[k] = (double)bf16_to_f32(x[m * ldx + k]);
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += xv[k] * (double)bf16_to_f32(w[n * ldw + k]);
      y[t * N + n] = acc;
    }
  }
  free(xv);
}

/* ------------------------------------------------------------------------------------------ */
/* Offline outlier identification ([ARC] Adaptieve Uitschieter-identificatie: rank channels by  */
/* absolute maximum over calibration data, keep the top S). Ties by ascending channel index.    */
/* ------------------------------------------------------------------------------------------ */

void oracle_channel_absmax(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, float* out) {
  for (int64_t k = 0; k < K; ++k) out[k] = 0.0f;
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(x[m * ld + k]));
      if (a > out[k]) out[k] = a;
    }
}

static const float* g_sort_key;
static int cmp_channels(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  if (g_sort_key[a] > g_sort_key[b]) return -1;
  if (g_sort_key[a] < g_sort_key[b]) return 1;
  return (a < b) ? -1 : (a > b);
}

void oracle_top_channels(const float* absmax, int64_t K, int32_t r, int32_t* idx) {
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
  for (int64_t k = 0; k < K; ++k) order[k] = (int32_t)k;
  g_sort_key = absmax;
  qsort(order, (size_t)K, sizeof(int32_t), cmp_channels);
  for (int32_t j = 0; j < r; ++j) idx[j] = order[j];
  free(order);
}

/* ------------------------------------------------------------------------------------------ */
/* SwiGLU gating of the recurrent block: a = bf16( silu(g) * u ), silu(g) = g / (1 + exp(-g)),  */
/* in double; g = columns [0, F) and u = columns [F, 2F) of the gate|up GEMM output.            */
/* ------------------------------------------------------------------------------------------ */

void oracle_silu_mul_rows(const uint16_t* gu, int64_t F, int64_t ld, uint16_t* out, int64_t ldo, int64_t m0,
                          int64_t m1) {
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t j = 0; j < F; ++j) {
      double g = (double)bf16_to_f32(gu[m * ld + j]);
      double u = (double)bf16_to_f32(gu[m * ld + F + j]);
      double s = g / (1.0 + exp(-g));
      out[m * ldo + j] = f32_to_bf16((float)(s * u));
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Array forms of the element codecs, for exhaustive tests.                                    */
/* ------------------------------------------------------------------------------------------ */

void oracle_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(v[i]);
}

void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode_nonneg(v[i]);
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 W8A8 with per-tensor scales (the low-precision format of RAMP's own instantiation,        */
/* "RAMP" §4.1: FP8 weights and activations): s = amax / 448 (the largest E4M3 magnitude), the  */
/* all-zero guard s = 1, code = signed E4M3 of the fp32 quotient x / s (ties to even, saturating */
/* at 448, the sign kept on values that round to zero, as for the E2M1 codes).                   */
/* ------------------------------------------------------------------------------------------ */

float oracle_fp8_scale(float amax) { return amax > 0.0f ? amax / 448.0f : 1.0f; }

uint8_t oracle_e4m3_encode_signed(float v) {
  const uint8_t mag = oracle_e4m3_encode_nonneg(fabsf(v));
  return (uint8_t)((signbit(v) ? 0x80 : 0x00) | mag);
}

void oracle_quantize_fp8_rows(const uint16_t* x, int64_t K, int64_t ldx, float s, uint8_t* codes, int64_t ldc,
                              int64_t m0, int64_t m1) {
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t k = 0; k < K; ++k) codes[m * ldc + k] = oracle_e4m3_encode_signed(bf16_to_f32(x[m * ldx + k]) / s);
}

/* ------------------------------------------------------------------------------------------ */
/* MXFP4 ("ARCQuant", Methodologie: the approach extends to the MXFP4 format), read as the OCP  */
/* microscaling format: blocks of 32 consecutive values share one power-of-two scale X =        */
/* 2^(floor(log2(amax_block)) - 2) (2 = the largest E2M1 exponent), stored as E8M0 = exponent + */
/* 127 clamped to [0, 254]; elements are E2M1_rn_sat(x / X) with the sign kept on zero, as for  */
/* NVFP4. An all-zero block has scale byte 0 and zero codes. No tensor scale.                  */
/* ------------------------------------------------------------------------------------------ */

uint8_t oracle_mxfp4_scale_byte(float amax) {
  if (!(amax > 0.0f)) return 0;
  int e2 = 0;
  (void)frexpf(amax, &e2); /* amax = f * 2^e2, f in [0.5, 1): floor(log2(amax)) = e2 - 1 */
  int e = (e2 - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return (uint8_t)(e + 127);
}

void oracle_quantize_mxfp4_rows(const uint16_t* x, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                                int64_t m0, int64_t m1) {
  const int64_t nb = K / 32;
  for (int64_t m = m0; m < m1; ++m) {
    const uint16_t* row = x + m * ldx;
    for (int64_t b = 0; b < nb; ++b) {
      float v[32];
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) {
        v[i] = bf16_to_f32(row[32 * b + i]);
        if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
      }
      const uint8_t sb = oracle_mxfp4_scale_byte(amax);
      scales[m * nb + b] = sb;
      for (int i = 0; i < 32; i += 2) {
        uint8_t lo = 0, hi = 0;
        if (amax > 0.0f) {
          /* x / 2^(sb - 127): exact in fp32 for every bf16 x (a power-of-two scaling) */
          lo = oracle_e2m1_encode(ldexpf(v[i], 127 - (int)sb));
          hi = oracle_e2m1_encode(ldexpf(v[i + 1], 127 - (int)sb));
        }
        codes[m * (K / 2) + (32 * b + i) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* MXFP4 with augmented residual channels ("ARCQuant", Resultaten / Generaliseerbaarheid: the   */
/* approach extends to MXFP4): the dual-stage code with MXFP4 blocks in place of NVFP4 blocks.  */
/*   primary   MXFP4 of the row in blocks of 32 consecutive channels (the code above);          */
/*   residual  for outlier channel c = idx[j]: x_c - E2M1(code_c) * X_b(c), fp32 multiply (exact: */
/*             X is a power of two) then fp32 subtract; the residuals in idx order form r/32    */
/*             blocks coded the same way and written at columns K + j;                          */
/*   weights   append the duplicated channels W[:, idx] instead (re-blocked among themselves).  */
/* K % 32 == 0, r % 32 == 0; K_pad = K + r rounded up to 64 (one tensor-core K step); padding   */
/* codes and scale bytes are 0. Scale bytes canonical: [rows, K_pad / 32].                      */
/* ------------------------------------------------------------------------------------------ */

/* One 32-value block: its scale byte, its codes and its scale X = 2^(byte - 127). */
static void mxfp4_block(const float* v, uint8_t* c32, uint8_t* sb_out, float* X_out) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i)
    if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
  const uint8_t sb = oracle_mxfp4_scale_byte(amax);
  for (int i = 0; i < 32; ++i) c32[i] = amax > 0.0f ? oracle_e2m1_encode(ldexpf(v[i], 127 - (int)sb)) : 0;
  *sb_out = sb;
  if (X_out) *X_out = ldexpf(1.0f, (int)sb - 127);
}

void oracle_quantize_mxfp4_arc_rows(const uint16_t* x, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                                    int32_t dup_mode, uint8_t* codes, uint8_t* sc, float* res_out, int64_t m0,
                                    int64_t m1) {
  const int64_t kpad = kpad_of(K + r);
  float* row = (float*)malloc(sizeof(float) * (size_t)K);
  float* X_blk = (float*)malloc(sizeof(float) * (size_t)(K / 32 + 1));
  float ext[32];
  uint8_t c32[32];
  for (int64_t m = m0; m < m1; ++m) {
    for (int64_t k = 0; k < K; ++k) row[k] = bf16_to_f32(x[m * ldx + k]);
    uint8_t* crow = codes + m * (kpad / 2);
    uint8_t* srow = sc + m * (kpad / 32);
    memset(crow, 0, (size_t)(kpad / 2));
    memset(srow, 0, (size_t)(kpad / 32));
    for (int64_t b = 0; b < K / 32; ++b) {
      mxfp4_block(row + 32 * b, c32, &srow[b], &X_blk[b]);
      for (int i = 0; i < 32; ++i) put_code(crow, 32 * b + i, c32[i]);
    }
    for (int32_t jb = 0; jb < r / 32; ++jb) {
      for (int i = 0; i < 32; ++i) {
        const int32_t c = idx[32 * jb + i];
        ext[i] = dup_mode ? row[c] : row[c] - oracle_e2m1_decode(oracle_get_code(crow, c)) * X_blk[c / 32];
        if (res_out) res_out[m * r + 32 * jb + i] = ext[i];
      }
      mxfp4_block(ext, c32, &srow[K / 32 + jb], NULL);
      for (int i = 0; i < 32; ++i) put_code(crow, K + 32 * jb + i, c32[i]);
    }
  }
  free(row);
  free(X_blk);
}

/* Y[rows[t], n] = sum_k E2M1(a) 2^(sa - 127) E2M1(b) 2^(sb - 127) in FP64 (exact per product). */
void oracle_gemm_mxfp4_f64(const uint8_t* a_codes, const uint8_t* a_sc, const uint8_t* b_codes, const uint8_t* b_sc,
                           int64_t N, int64_t K, const int64_t* rows, int64_t nrows, double* y) {
  const int64_t nb = K / 32;
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t m = rows[t];
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t b = 0; b < nb; ++b) {
        const double sa = ldexp(1.0, (int)a_sc[m * nb + b] - 127), sw = ldexp(1.0, (int)b_sc[n * nb + b] - 127);
        double part = 0.0;
        for (int i = 0; i < 32; ++i) {
          const int64_t k = 32 * b + i;
          const uint8_t ca = (uint8_t)((a_codes[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 15);
          const uint8_t cb = (uint8_t)((b_codes[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 15);
          part += (double)oracle_e2m1_decode(ca) * (double)oracle_e2m1_decode(cb);
        }
        acc += part * sa * sw;
      }
      y[t * N + n] = acc;
    }
  }
}

void oracle_e4m3_decode_array(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

void oracle_e2m1_decode_array(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_decode(c[i]);
}

/* E2M1 code of x / d for each x, as the block code does it (fp32 divide, then encode). */
void oracle_e2m1_of_quotient_array(const float* x, int64_t n, float d, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (d == 0.0f) ? 0 : oracle_e2m1_encode(x[i] / d);
}

void oracle_rmsnorm_rows(const uint16_t* h, int64_t d, int64_t ld, const uint16_t* g, double eps, uint16_t* out,
                         int64_t ldo, int64_t m0, int64_t m1) {
  for (int64_t m = m0; m < m1; ++m) oracle_rmsnorm_row(h + m * ld, g, d, eps, out + m * ldo);
}
