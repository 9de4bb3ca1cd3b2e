// quant.cuh -- the memory-bound half of the hot path: RMSNorm statistics and the single-launch
// NVFP4 quantizer with its augmented residual channels.
//
// Method ("ARCQuant: Boosting NVFP4 Quantization with Augmented Residual Channels for LLMs",
// Methodologie, Dual-Stage Quantisatie / Kernel Implementatie; "Day 0 LLM Inference Support",
// section V items 1, 2 and 4): per 16-element block sf = E4M3((amax/6)/s), d = E4M3(sf)*s,
// code = E2M1(x/d) with the sign of x, all-zero blocks give sf 0 and codes 0; the residual of
// each outlier channel, x - E2M1(code)*d, is quantized again with the same tensor scale and
// appended after the K primary channels (weights append the channel itself).
//
// Work split:
//   k_row_stats    one warp per row: exact sum of squares -> 1/rms (double); with a dynamic
//                  scale also max |RMSNorm(x)|, one partial per CTA
//   k_quant_fused  one cooperative launch, one CTA per SM, tiles of 128 rows x 128 channels
//                  TMA-loaded into a ring of shared-memory buffers by a producer warp, which
//                  also lists each tile's outlier channels; sixteen coding warps take the tiles
//                  (full/empty mbarriers between the two roles):
//     phase 1  (dynamic scale without RMSNorm) max |x| over the CTA's tiles, the last ones
//              staying resident in the ring; grid barrier; every CTA reduces the partials
//     phase 2  code the tiles (resident ones first): each coding warp takes eight rows of a
//              tile, one lane per 16-element block; codes and scale bytes go straight to
//              global memory; then the warp stashes the residuals of the outlier channels
//              of its rows in the column-major stash [r, M] (one (row, outlier) pair per
//              lane, operands fetched by warp shuffles); the warps never wait for one
//              another, only for tiles
//     phase 3  after a second grid barrier: the appended residual blocks and the zero
//              padding up to K_pad, one lane per (row, block) with rows fastest, so the
//              stash reads are coalesced
// Divisions are correctly rounded: x/d is formed as the negated quotient from -RN(1/d) with one
// exact-remainder correction (Markstein), which keeps the sign of zero quotients, and the codes
// of the negated quotients have their sign bits flipped back; a plain IEEE divide is used when
// an operand is outside [2^-90, 2^90].
#pragma once

#include "arc_device.cuh"

namespace arc {

constexpr int kMaxPartials = 2048;  // per-CTA abs-max partials at the start of the workspace

struct QuantArgs {
  const __nv_bfloat16* x;
  int64_t ldx;
  int M, K, r, kpad, katoms;
  const int32_t* idx;
  const __nv_bfloat16* gain;  // RMSNorm prologue gain, or nullptr
  const double* inv_rms;      // [M] from k_row_stats when gain != nullptr
  const float* static_scale;  // or nullptr (dynamic)
  const uint32_t* partials;   // fp32 bits of per-CTA max |x| (dynamic)
  int npartials;
  float* scale_out;
  uint8_t* codes;
  uint8_t* sf;
  float* stash;  // [r, M]: column j holds channel idx[j] of every row
  int dup;       // 1: weights (stash the value itself), 0: activations (stash the residual)
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ bool in_safe_range(float v) {
  return v >= 8.077935669463161e-28f && v <= 1.2379400392853803e27f;  // [2^-90, 2^90]
}

// Tensor scale of this call, by one CTA (all threads return the same value).
__device__ float cta_tensor_scale(const QuantArgs& a) {
  if (a.static_scale) return *a.static_scale;
  __shared__ uint32_t red[32];
  uint32_t mx = 0;
  for (int i = threadIdx.x; i < a.npartials; i += blockDim.x) mx = max(mx, a.partials[i]);
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  uint32_t b = 0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) b = max(b, red[i]);
  __syncthreads();
  const float am = __uint_as_float(b);
  return am > 0.0f ? __fdiv_rn(am, 2688.0f) : 1.0f;
}

// Byte offset of scale (row m, scale column kb) in the swizzled layout.
__device__ __forceinline__ int64_t sf_offset(int64_t m, int64_t kb, int katoms) {
  return ((m >> 7) * katoms + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

// Scale byte and decode scale d of a block with abs-max `amax` under tensor scale s:
// t = (amax / 6) / s (two correctly rounded divides), sf = E4M3(t), d = E4M3value(sf) * s.
__device__ __forceinline__ uint32_t block_scale(float amax, float s, float rcp_s, float rcp6, float* d) {
  float t;
  if (in_safe_range(amax) && in_safe_range(s)) {
    const float t1 = div_rn_from_rcp(amax, 6.0f, rcp6);
    const float q0 = __fmul_rn(t1, rcp_s);
    // outside [2^-20, 2^20] the E4M3 result is 0 or 448 whatever the last bit of t
    t = (q0 >= 9.5367431640625e-07f && q0 <= 1048576.0f) ? div_rn_from_rcp(t1, s, rcp_s) : q0;
  } else {
    t = __fdiv_rn(__fdiv_rn(amax, 6.0f), s);
  }
  const uint32_t sfb = e4m3_rn_sat(t);
  *d = __fmul_rn(e4m3_value(sfb), s);
  return sfb;
}

// Codes of 16 values (8 packed pairs) against decode scale d > 0: E2M1 of the correctly rounded
// quotient with the sign of x (a quotient that rounds to zero keeps it: -0.1 -> 0x8). The
// quotients are formed negated, which keeps signed zeros exact, and since E2M1 is sign-magnitude
// with symmetric rounding and saturation, code(q) = code(-q) ^ 8 nibble by nibble. Element i of
// pair j in bits 8j + 4i.
__device__ __forceinline__ uint2 encode16(const uint64_t (&p)[8], float d) {
  float nq[16];
  if (in_safe_range(d)) {
    const float nrcp = -__frcp_rn(d);
    const uint64_t nrcp2 = f2_pack(nrcp, nrcp), d2 = f2_pack(d, d);
#pragma unroll
    for (int j = 0; j < 8; ++j) f2_unpack(neg_div2_rn(p[j], d2, nrcp2), nq[2 * j], nq[2 * j + 1]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float x0, x1;
      f2_unpack(p[j], x0, x1);
      nq[2 * j] = -__fdiv_rn(x0, d);
      nq[2 * j + 1] = -__fdiv_rn(x1, d);
    }
  }
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = nq[i];
    hi[i] = nq[8 + i];
  }
  return make_uint2(e2m1x8_rn_sat(lo) ^ 0x88888888u, e2m1x8_rn_sat(hi) ^ 0x88888888u);
}

// RMSNorm of one bf16 value: bf16( fp32( (h * inv) * g ) ), products in double.
__device__ __forceinline__ float rms_apply(float h, double inv, float g) {
  const double t = __dmul_rn(__dmul_rn(static_cast<double>(h), inv), static_cast<double>(g));
  return __bfloat162float(__float2bfloat16_rn(__double2float_rn(t)));
}

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t m, uint4 w) {
  m = __vmaxu2(m, w.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, w.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
  return __vmaxu2(m, w.w & 0x7FFF7FFFu);
}

// Block-wide max of a per-thread value, written by thread 0 to *dst.
__device__ __forceinline__ void cta_max_to(uint32_t v, uint32_t* dst) {
  __shared__ uint32_t red[32];
  v = __reduce_max_sync(0xFFFFFFFFu, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) b = max(b, red[i]);
    *dst = b;
  }
}

// ---------------------------------------------------------------------------------------------

// Round-to-nearest-even value of v * 2^e2 as a double (v < 2^128).
__device__ __forceinline__ double u128_scaled_to_double(unsigned __int128 v, int e2) {
  if (v == 0) return 0.0;
  const uint64_t hi = static_cast<uint64_t>(v >> 64), lo = static_cast<uint64_t>(v);
  const int p = hi ? 127 - __clzll(static_cast<long long>(hi)) : 63 - __clzll(static_cast<long long>(lo));
  if (p <= 52) return ldexp(static_cast<double>(lo), e2);
  const int sh = p - 52;
  unsigned __int128 mant = v >> sh;
  const unsigned __int128 one = 1;
  const unsigned __int128 rem = v & ((one << sh) - 1);
  const unsigned __int128 half = one << (sh - 1);
  if (rem > half || (rem == half && (mant & 1))) mant += 1;
  return ldexp(static_cast<double>(static_cast<uint64_t>(mant)), e2 + sh);
}

// One warp: 1/rms of row h[0..K) with the exact sum of squares (every bf16 square is
// m^2 2^(2e-268), m < 256; summed as a 128-bit integer in units of 2^(2 emax - 362), squares
// more than 2^94 below the largest truncated), widened eps. Lane-strided 16-byte loads.
__device__ double warp_row_inv_rms(const __nv_bfloat16* __restrict__ h, int K, double eps, int lane) {
  int emax = 0;
  for (int k = 8 * lane; k < K; k += 256) {
    const uint4 w = ld_nc_v4(h + k);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t b = (ws[i >> 1] >> (16 * (i & 1))) & 0x7FFFu;
      if (b) emax = max(emax, max(static_cast<int>(b >> 7), 1));
    }
  }
  emax = static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, static_cast<unsigned>(emax)));
  unsigned __int128 acc = 0;
  for (int k = 8 * lane; k < K; k += 256) {
    const uint4 w = ld_nc_v4(h + k);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t b = (ws[i >> 1] >> (16 * (i & 1))) & 0x7FFFu;
      if (!b) continue;
      int e = static_cast<int>(b >> 7);
      uint32_t m = b & 0x7Fu;
      if (e == 0)
        e = 1;
      else
        m |= 0x80u;
      const uint64_t sq = static_cast<uint64_t>(m) * m;
      const int sh = 2 * (e - emax) + 94;
      if (sh >= 0)
        acc += static_cast<unsigned __int128>(sq) << sh;
      else if (sh > -64)
        acc += static_cast<unsigned __int128>(sq >> (-sh));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const uint64_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint64_t>(acc), o);
    const uint64_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint64_t>(acc >> 64), o);
    acc += (static_cast<unsigned __int128>(hi) << 64) | lo;
  }
  const double ss = u128_scaled_to_double(acc, 2 * emax - 268 - 94);
  return __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(K)), eps)));
}

// Warps over rows (grid-stride): inv_rms[m]; with partials != nullptr also max |RMSNorm(h)*g|,
// one partial per CTA.
__global__ void __launch_bounds__(256) k_row_stats(const __nv_bfloat16* __restrict__ h, int64_t ldh, int M, int K,
                                                   const __nv_bfloat16* __restrict__ gain, double eps,
                                                   double* inv_rms, uint32_t* partials) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t mx = 0;
  for (int m = blockIdx.x * 8 + warp; m < M; m += gridDim.x * 8) {
    const __nv_bfloat16* row = h + static_cast<int64_t>(m) * ldh;
    const double inv = warp_row_inv_rms(row, K, eps, lane);
    if (lane == 0) inv_rms[m] = inv;
    if (partials) {
      for (int k = 8 * lane; k < K; k += 256) {
        const uint4 w = ld_nc_v4(row + k);
        const uint4 g = ld_nc_v4(gain + k);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, gs[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float hv = (i & 1) ? bf16_hi(ws[i >> 1]) : bf16_lo(ws[i >> 1]);
          const float gv = (i & 1) ? bf16_hi(gs[i >> 1]) : bf16_lo(gs[i >> 1]);
          mx = max(mx, __float_as_uint(fabsf(rms_apply(hv, inv, gv))));
        }
      }
    }
  }
  if (partials) cta_max_to(mx, &partials[blockIdx.x]);
}

// ---------------------------------------------------------------------------------------------
// Single-launch quantizer (cooperative launch, one CTA per SM, all CTAs resident).
// The grid barriers need no initialised memory: each CTA stores the call's epoch (a number the
// host never reuses) in its own flag and waits until every flag shows it, with the usual time
// limit; a wait that runs out sets the status word and stops the CTA.
// ---------------------------------------------------------------------------------------------
constexpr int kQTileBytes = 128 * 128 * 2;  // one X tile: two TMA boxes of 128 rows x 64 channels
constexpr int kCodeWarps = 16;                      // warps that code tiles
constexpr int kFusedThreads = (kCodeWarps + 1) * 32;  // plus one producer warp (loads, outlier lists)
constexpr int kFusedBufs = 6;
constexpr int kIdxSmem = 1024;  // outlier indices kept in shared memory (the rest read from L2)
// dynamic shared memory: the ring of X tiles, 1024-aligned for the 128-byte swizzle
constexpr int kFusedSmem = 1024 + kFusedBufs * kQTileBytes;

// Grid barrier over co-resident CTAs: each CTA publishes the call's epoch in its own arrival
// word; CTA 0 gathers them (one polling thread per word) and then publishes the epoch in the
// go word, which one thread of every CTA polls. Polling from every CTA on every arrival word
// crowds a few L2 lines with requests and costs about twice as much. Release stores and acquire
// loads at GPU scope carry each CTA's earlier writes (made visible to thread 0 by the CTA
// barrier) to every CTA after the barrier. Every wait is bounded; one that runs out sets the
// status word and makes the barrier return false in every CTA that sees it.
__device__ __forceinline__ bool grid_barrier(unsigned long long* arrive, unsigned long long* go, int G,
                                             unsigned long long epoch, uint64_t wait_ns, int* abort_sh) {
  __syncthreads();
  if (threadIdx.x == 0) st_release_gpu(&arrive[blockIdx.x], epoch);
  const uint64_t t0 = globaltimer_ns();
  bool ok = true;
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < G && ok; i += blockDim.x)
      while (ld_acquire_gpu(&arrive[i]) != epoch) {
        if (globaltimer_ns() - t0 > wait_ns) {
          ok = false;
          break;
        }
      }
    ok = __syncthreads_and(ok);
    if (threadIdx.x == 0 && ok) st_release_gpu(go, epoch);
  }
  if (threadIdx.x == 0 && ok) {
    while (ld_acquire_gpu(go) != epoch) {
      if (globaltimer_ns() - t0 > wait_ns) {
        ok = false;
        break;
      }
    }
  }
  if (!ok) {
    set_status(kStatusTimeout);
    *reinterpret_cast<volatile int*>(abort_sh) = 1;
  }
  __syncthreads();
  return *reinterpret_cast<volatile int*>(abort_sh) == 0;
}

struct FusedArgs {
  int tiles_k, ntiles;
  int do_amax;                  // phase 1 runs (dynamic scale without RMSNorm)
  uint32_t* partials;           // [gridDim.x] written by phase 1
  unsigned long long* flags;    // barrier words: go words at [0] and [16], arrivals at [32 ..)
  unsigned long long epoch;     // this call's barrier epochs: epoch and epoch + 1
  uint64_t wait_ns;
  int mpad;                     // rows rounded up to 128 (scale padding rows)
};

// Shared-memory address of 16-byte chunk j (0..7) of tile row `row` in half h (channels
// 64h .. 64h+63): each half is 128 rows x 128 bytes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t qtile_chunk(uint32_t base, int h, int row, int j) {
  return base + h * (128 * 128) + row * 128 + ((j ^ (row & 7)) << 4);
}

// Outlier list of one column tile: entries (j << 7) | (channel - k0) for the index-list
// positions j whose channel falls in the tile, in increasing j.
constexpr int kOCap = 256;  // entries per tile (128 distinct channels at most)
struct OutlierList {
  int n;
  uint32_t e[kOCap];
};

// Codes of one resident tile, by one coding warp: lane l takes row 8w + l%8 and blocks l/8 and
// 4 + l/8 of it (eight rows per 16-byte read hit eight distinct swizzled bank groups, and each
// code store is 32 contiguous bytes in each of eight rows). Both blocks are loaded first and
// coded side by side, and the lane writes its codes and scale bytes. Then the warp stashes the
// outlier channels of its eight rows: lane l takes row l%8 and outlier entry l/8 (four entries
// per pass), fetching the decode scale and code word of that element from the lane that coded
// it by warp shuffles, and writes x (weights) or x minus its dequantized value (activations) to
// column j of the stash. Nothing here waits for another warp.
//   sf_lane: this lane's constant part of the scale offset, (mm%32)*16 + (mm/32)*4 + l/8
template <bool RMS>
__device__ __forceinline__ void code_rows(const QuantArgs& a, uint32_t tbase, int tm, int tk, float s, float rcp_s,
                                          float rcp6, const OutlierList& ol, int sf_lane) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mm = warp * 8 + (lane & 7), bq = lane >> 3;
  const int m0 = tm * 128, k0 = tk * 128;
  const int m = m0 + mm;
  const bool rowok = m < a.M;
  double inv = 0.0;
  if (RMS) inv = rowok ? a.inv_rms[m] : 0.0;
  uint32_t ws[2][8];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 w0 = lds_v4(qtile_chunk(tbase, h, mm, 2 * bq));
    const uint4 w1 = lds_v4(qtile_chunk(tbase, h, mm, 2 * bq + 1));
    ws[h][0] = w0.x, ws[h][1] = w0.y, ws[h][2] = w0.z, ws[h][3] = w0.w;
    ws[h][4] = w1.x, ws[h][5] = w1.y, ws[h][6] = w1.z, ws[h][7] = w1.w;
  }
  float v[2][16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int kcol = k0 + 16 * (4 * h + bq);
    if (RMS) {
      uint4 g0 = make_uint4(0, 0, 0, 0), g1 = g0;
      if (kcol < a.K) {
        g0 = ld_nc_v4(a.gain + kcol);
        g1 = ld_nc_v4(a.gain + kcol + 8);
      }
      const uint32_t gs[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[h][2 * j] = rms_apply(bf16_lo(ws[h][j]), inv, bf16_lo(gs[j]));
        v[h][2 * j + 1] = rms_apply(bf16_hi(ws[h][j]), inv, bf16_hi(gs[j]));
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[h][2 * j] = bf16_lo(ws[h][j]);
        v[h][2 * j + 1] = bf16_hi(ws[h][j]);
      }
    }
  }
  float d[2];
  uint32_t sfv[2];
  uint2 codes[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float a0 = fmax3_abs(v[h][0], v[h][1], v[h][2]), a1 = fmax3_abs(v[h][3], v[h][4], v[h][5]),
                a2 = fmax3_abs(v[h][6], v[h][7], v[h][8]), a3 = fmax3_abs(v[h][9], v[h][10], v[h][11]),
                a4 = fmax3_abs(v[h][12], v[h][13], v[h][14]);
    sfv[h] = block_scale(fmaxf(fmax3(a0, a1, a2), fmax3(a3, a4, fabsf(v[h][15]))), s, rcp_s, rcp6, &d[h]);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint64_t p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = f2_pack(v[h][2 * j], v[h][2 * j + 1]);
    codes[h] = (d[h] == 0.0f) ? make_uint2(0u, 0u) : encode16(p, d[h]);
  }
  uint8_t* crow = a.codes + static_cast<int64_t>(rowok ? m : 0) * (a.kpad >> 1) + (k0 >> 1);
  uint8_t* sft = a.sf + (static_cast<int64_t>(tm) * a.katoms + (k0 >> 6)) * 512 + sf_lane;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (k0 + 16 * (4 * h + bq) >= a.K) continue;
    if (rowok) *reinterpret_cast<uint2*>(crow + 8 * (4 * h + bq)) = codes[h];
    // padding rows (up to the next multiple of 128) carry zero scales
    sft[h * 512] = rowok ? static_cast<uint8_t>(sfv[h]) : 0;
  }
  // outlier channels of the warp's eight rows, four entries per pass (the lane keeps its row)
  for (int base = 0; base < ol.n; base += 4) {
    const int o = base + (lane >> 3);
    const bool act = o < ol.n && rowok;
    const uint32_t ent = (o < ol.n) ? ol.e[o] : 0u;
    const int col = static_cast<int>(ent & 127u), j = static_cast<int>(ent >> 7);
    const int blk = col >> 4, e = col & 15;
    const int src = (lane & 7) + 8 * (blk & 3);  // the lane that coded (this row, block blk)
    const float dd0 = __shfl_sync(0xFFFFFFFFu, d[0], src), dd1 = __shfl_sync(0xFFFFFFFFu, d[1], src);
    const uint32_t c0x = __shfl_sync(0xFFFFFFFFu, codes[0].x, src), c0y = __shfl_sync(0xFFFFFFFFu, codes[0].y, src);
    const uint32_t c1x = __shfl_sync(0xFFFFFFFFu, codes[1].x, src), c1y = __shfl_sync(0xFFFFFFFFu, codes[1].y, src);
    if (!act) continue;
    uint16_t hv;
    asm volatile("ld.shared.u16 %0, [%1];"
                 : "=h"(hv)
                 : "r"(qtile_chunk(tbase, blk >> 2, mm, (col & 63) >> 3) + 2 * (col & 7)));
    float x = __uint_as_float(static_cast<uint32_t>(hv) << 16);
    if (RMS) x = rms_apply(x, inv, __bfloat162float(a.gain[k0 + col]));
    float res = x;
    if (!a.dup) {
      const uint32_t cw = (blk >> 2) ? ((e < 8) ? c1x : c1y) : ((e < 8) ? c0x : c0y);
      const uint32_t c = (cw >> (4 * (e & 7))) & 15u;
      res = __fsub_rn(x, __fmul_rn(e2m1_value(c), (blk >> 2) ? dd1 : dd0));
    }
    a.stash[static_cast<int64_t>(j) * a.M + m] = res;
  }
}

// The outlier list of column tile k0 .. k0+127, by one warp (ballot compaction).
__device__ __forceinline__ void build_olist(const QuantArgs& a, const int32_t* idx_sh, int k0, OutlierList& ol,
                                            int lane) {
  int n = 0;
  for (int base = 0; base < a.r; base += 32) {
    const int j = base + lane;
    const int c = (j < a.r) ? (j < kIdxSmem ? idx_sh[j] : __ldg(a.idx + j)) : -1;
    const bool hit = j < a.r && c < a.K && static_cast<unsigned>(c - k0) < 128u;
    const uint32_t mask = __ballot_sync(0xFFFFFFFFu, hit);
    const int pos = n + __popc(mask & ((1u << lane) - 1u));
    if (hit && pos < kOCap) ol.e[pos] = (static_cast<uint32_t>(j) << 7) | static_cast<uint32_t>(c - k0);
    n += __popc(mask);
  }
  if (n > kOCap) {
    if (lane == 0) set_status(kStatusInvalidArg);  // more entries than distinct channels
    n = kOCap;
  }
  if (lane == 0) ol.n = n;
  __syncwarp();
}

// The appended residual blocks (from the stash) and zero padding up to K_pad: one (row, block)
// per thread, rows fastest.
__device__ __forceinline__ void tail_items(const QuantArgs& a, int mpad, float s, float rcp_s, float rcp6) {
  const int nres = a.r >> 4;
  const int ntail = (a.kpad - a.K) >> 4;
  const int64_t cpitch = a.kpad >> 1;
  const int64_t items = static_cast<int64_t>(mpad) * ntail;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items; it += stride) {
    const int b = static_cast<int>(it / mpad), m = static_cast<int>(it - static_cast<int64_t>(b) * mpad);
    uint32_t sfv = 0;
    uint2 codes = make_uint2(0u, 0u);
    if (m < a.M && b < nres) {
      const float* src = a.stash + static_cast<int64_t>(16 * b) * a.M + m;
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __ldcg(src + static_cast<int64_t>(i) * a.M);
      uint64_t p[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) p[j] = f2_pack(v[2 * j], v[2 * j + 1]);
      const float a0 = fmax3_abs(v[0], v[1], v[2]), a1 = fmax3_abs(v[3], v[4], v[5]),
                  a2 = fmax3_abs(v[6], v[7], v[8]), a3 = fmax3_abs(v[9], v[10], v[11]),
                  a4 = fmax3_abs(v[12], v[13], v[14]);
      const float am = fmaxf(fmax3(a0, a1, a2), fmax3(a3, a4, fabsf(v[15])));
      float d;
      sfv = block_scale(am, s, rcp_s, rcp6, &d);
      if (d != 0.0f) codes = encode16(p, d);
    }
    if (m < a.M) *reinterpret_cast<uint2*>(a.codes + static_cast<int64_t>(m) * cpitch + ((a.K + 16 * b) >> 1)) = codes;
    a.sf[sf_offset(m, (a.K >> 4) + b, a.katoms)] = static_cast<uint8_t>(sfv);
  }
}

template <bool RMS>
__global__ void __launch_bounds__(kFusedThreads, 1) k_quant_fused(const __grid_constant__ CUtensorMap tmX,
                                                                  QuantArgs a, FusedArgs f) {
  extern __shared__ uint8_t fsmem_raw[];
  uint8_t* qs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fsmem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kFusedBufs], empty[kFusedBufs];
  __shared__ int32_t idx_sh[kIdxSmem];
  __shared__ OutlierList olist[kFusedBufs];  // outlier list of the tile in each ring buffer
  __shared__ int abort_sh;
  __shared__ float s_sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == kCodeWarps;
  const int G = gridDim.x;
  const int n_c = (f.ntiles > static_cast<int>(blockIdx.x)) ? (f.ntiles - blockIdx.x + G - 1) / G : 0;
  const uint32_t xbase = smem_u32(qs);
  // CTA-local tile i is tile blockIdx.x + i * G. Phase 1 streams i = 0 .. n_c-1 through slots
  // 0 .. n_c-1 and leaves the last `resident` of them in the ring; phase 2 codes those first,
  // then the others, which come through the ring again. Slot sl uses buffer sl % kFusedBufs.
  const int resident = f.do_amax ? min(n_c, kFusedBufs) : 0;
  const int first_slot = f.do_amax ? n_c - resident : 0;  // slot of processing position q = 0
  auto tile_at = [&](int q) {
    const int i = f.do_amax ? (q < resident ? n_c - resident + q : q - resident) : q;
    return static_cast<int>(blockIdx.x) + i * G;
  };
  int issued = 0;  // producer lane 0: slots issued so far
  auto issue = [&](int slot, int t) {
    const int tm = t / f.tiles_k, tk = t - tm * f.tiles_k;
    const int buf = slot % kFusedBufs;
    mbar_arrive_expect_tx(&full[buf], kQTileBytes);
    uint8_t* dst = qs + buf * kQTileBytes;
    tma_load_2d(dst, &tmX, &full[buf], tk * 128, tm * 128);
    tma_load_2d(dst + 128 * 128, &tmX, &full[buf], tk * 128 + 64, tm * 128);
    issued = slot + 1;
  };
  // producer: before reusing a buffer, wait until the coding warps released its previous slot
  // (sleeping between polls, so the wait leaves the issue slots to the coding warps)
  auto wait_free = [&](int slot) -> bool {
    if (slot < kFusedBufs) return true;
    return mbar_wait(&empty[slot % kFusedBufs], static_cast<uint32_t>((slot / kFusedBufs - 1) & 1), f.wait_ns,
                     &abort_sh, 128);
  };
  // producer lane 0 after an abort: the last load issued into each buffer lands (bounded)
  auto drain = [&]() {
    const uint64_t t0 = globaltimer_ns();
    for (int b = 0; b < kFusedBufs; ++b) {
      int sl = issued - 1 - ((issued - 1 - b) % kFusedBufs + kFusedBufs) % kFusedBufs;
      if (sl < 0) continue;
      while (!mbar_test(&full[b], static_cast<uint32_t>((sl / kFusedBufs) & 1)) && globaltimer_ns() - t0 < f.wait_ns) {
      }
    }
  };
  auto release = [&](int slot) {  // coding warp done with the slot's buffer and outlier list
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot % kFusedBufs]);
  };
  // A full barrier completes on the tile's bytes plus two producer arrivals: one with the
  // byte count when the loads are issued, one when the tile's outlier list is written.
  if (producer && lane == 0) {
    for (int i = 0; i < kFusedBufs; ++i) {
      mbar_init(&full[i], 2);
      mbar_init(&empty[i], kCodeWarps);
    }
    abort_sh = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    // the first kFusedBufs slots hold tiles 0 .. kFusedBufs-1 in either phase order
    for (int sl = 0; sl < min(n_c, kFusedBufs); ++sl) issue(sl, static_cast<int>(blockIdx.x) + sl * G);
  }
  for (int j = tid; j < min(a.r, kIdxSmem); j += kFusedThreads) idx_sh[j] = a.idx[j];
  if (blockIdx.x == 0)
    for (int j = tid; j < a.r; j += kFusedThreads)
      if (static_cast<unsigned>(a.idx[j]) >= static_cast<unsigned>(a.K)) set_status(kStatusInvalidArg);
  __syncthreads();
  if (f.do_amax) {
    // ------------------------------------------------------------------ phase 1: max |x|
    uint32_t mx = 0;
    if (producer) {
      if (lane == 0) {
        for (int sl = 0; sl < n_c; ++sl) {
          if (sl >= kFusedBufs) {
            if (!wait_free(sl)) break;
            issue(sl, static_cast<int>(blockIdx.x) + sl * G);
          }
          mbar_arrive(&full[sl % kFusedBufs]);  // phase 1 reads no outlier list
        }
      }
      __syncwarp();
      // outlier lists of the tiles that stay resident (their buffers hold no list in phase 1;
      // the grid barrier below publishes them)
      for (int sl = first_slot; sl < n_c; ++sl)
        build_olist(a, idx_sh, (tile_at(sl - first_slot) % f.tiles_k) * 128, olist[sl % kFusedBufs], lane);
    } else {
      for (int sl = 0; sl < n_c; ++sl) {
        const int buf = sl % kFusedBufs;
        if (!mbar_wait(&full[buf], static_cast<uint32_t>((sl / kFusedBufs) & 1), f.wait_ns, &abort_sh)) break;
        const uint32_t tb = xbase + buf * kQTileBytes;
        // 512 threads x 4 chunks of 16 bytes = the 32 KB tile
#pragma unroll
        for (int j = 0; j < 4; ++j) mx = absmax_bf16x2(mx, lds_v4(tb + (tid + j * kCodeWarps * 32) * 16));
        if (sl < first_slot) release(sl);
      }
    }
    cta_max_to(max(mx & 0xFFFFu, mx >> 16) << 16, &f.partials[blockIdx.x]);
    if (!grid_barrier(f.flags + 32, f.flags, G, f.epoch, f.wait_ns, &abort_sh)) {
      if (producer && lane == 0) drain();
      return;
    }
  }
  // ---------------------------------------------------------------------- phase 2: code tiles
  {
    QuantArgs aa = a;
    if (f.do_amax) {
      aa.partials = f.partials;
      aa.npartials = G;
    }
    const float s = cta_tensor_scale(aa);
    if (tid == 0) s_sh = s;
  }
  __syncthreads();
  const float s = s_sh;
  if (blockIdx.x == 0 && tid == 0) *a.scale_out = s;
  const float rcp_s = __frcp_rn(s), rcp6 = __frcp_rn(6.0f);
  if (producer) {
    for (int q = resident; q < n_c; ++q) {
      const int sl = first_slot + q, buf = sl % kFusedBufs;
      const int t = tile_at(q);
      bool ok = true;
      if (lane == 0 && sl >= kFusedBufs) {  // the first kFusedBufs slots were issued at the start
        ok = wait_free(sl);
        if (ok) issue(sl, t);
      }
      if (!__shfl_sync(0xFFFFFFFFu, static_cast<int>(ok), 0)) break;
      build_olist(a, idx_sh, (t % f.tiles_k) * 128, olist[buf], lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[buf]);
    }
  } else {
    const int mm = warp * 8 + (lane & 7);
    const int sf_lane = (mm & 31) * 16 + (mm >> 5) * 4 + (lane >> 3);
    for (int q = 0; q < n_c; ++q) {
      const int sl = first_slot + q, buf = sl % kFusedBufs;
      const int t = tile_at(q);
      const int tm = t / f.tiles_k, tk = t - tm * f.tiles_k;
      // resident tiles were waited for in phase 1
      if (q >= resident &&
          !mbar_wait(&full[buf], static_cast<uint32_t>((sl / kFusedBufs) & 1), f.wait_ns, &abort_sh))
        break;
      code_rows<RMS>(a, xbase + buf * kQTileBytes, tm, tk, s, rcp_s, rcp6, olist[buf], sf_lane);
      release(sl);
    }
  }
  __syncthreads();  // both roles are done with the ring
  if (abort_sh) {
    if (producer && lane == 0) drain();
    return;
  }
  if (a.kpad == a.K) return;
  // ---------------------------------------------------------------------- phase 3: tail
  if (!grid_barrier(f.flags + 32 + G, f.flags + 16, G, f.epoch + 1, f.wait_ns, &abort_sh)) return;
  tail_items(a, f.mpad, s, rcp_s, rcp6);
}

}  // namespace arc
