// quant.cuh -- the memory-bound half of the hot path: tensor abs-max, RMSNorm statistics,
// fused primary NVFP4 quantization with the residual stash, and the residual-channel tail.
//
// Method ("ARCQuant: Boosting NVFP4 Quantization with Augmented Residual Channels for LLMs",
// Methodologie, Dual-Stage Quantisatie / Kernel Implementatie; "Day 0 LLM Inference Support",
// section V items 1, 2 and 4): per 16-element block sf = E4M3((amax/6)/s), d = E4M3(sf)*s,
// code = E2M1(x/d) with the sign of x, all-zero blocks give sf 0 and codes 0; the residual of
// each outlier channel, x - E2M1(code)*d, is quantized again with the same tensor scale and
// appended after the K primary channels.
//
// Work split:
//   k_amax        whole-tensor max |x|: 16-byte loads, 4 in flight per thread, integer max on
//                 |bf16| bit patterns; one partial per CTA in the workspace (no atomics, no
//                 initialisation of the workspace needed)
//   k_row_stats   one warp per row: exact sum of squares -> 1/rms (double); with a dynamic
//                 scale also max |RMSNorm(x)|, one partial per CTA
//   k_quant_stream persistent CTAs over tiles of 128 rows x 128 channels, the X tile TMA-loaded
//                 into shared memory (double-buffered); one lane per 16-element block (8 lanes
//                 per row, 4 rows per warp step), packed-pair division, 8 code bytes per lane (a
//                 row's 64 code bytes contiguous), scale bytes staged in shared memory and written
//                 as whole 512-byte atoms; outlier channels leave x (weights) or x - deq
//                 (activations) in a [rows, r] fp32 stash
//   k_quant_tail  one warp per row: the r/16 appended blocks from the stash plus zero padding up
//                 to K_pad, including the zero scale bytes of padding rows
// Divisions are correctly rounded: x/d uses RN(1/d) and one exact-remainder correction
// (Markstein), with a plain IEEE divide when an operand is outside [2^-90, 2^90].
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
  float* stash;  // [M, r]
  int dup;       // 1: weights (stash the value itself), 0: activations (stash the residual)
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
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
// quotient. The hardware conversion keeps the sign of a quotient that rounds to zero (-0.1 ->
// 0x8), so the sign bit follows x without extra work. Element i of pair j in bits 8j + 4i.
__device__ __forceinline__ uint2 encode16(const uint64_t (&p)[8], float d) {
  float q[16];
  if (in_safe_range(d)) {
    const float rcp = __frcp_rn(d);
    const uint64_t rcp2 = f2_pack(rcp, rcp), nd2 = f2_pack(-d, -d);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // the correction turns a -0 quotient into +0 ((+0) + (-0)); the quotient takes x's sign
      const uint64_t qq = div2_rn_from_rcp(p[j], nd2, rcp2);
      const uint64_t sg = 0x8000000080000000ull;
      f2_unpack((qq & ~sg) | (p[j] & sg), q[2 * j], q[2 * j + 1]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float x0, x1;
      f2_unpack(p[j], x0, x1);
      q[2 * j] = __fdiv_rn(x0, d);
      q[2 * j + 1] = __fdiv_rn(x1, d);
    }
  }
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = q[i];
    hi[i] = q[8 + i];
  }
  return make_uint2(e2m1x8_rn_sat(lo), e2m1x8_rn_sat(hi));
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

// Contiguous X (ldx == K): a flat stream of 16-byte vectors, 4 loads in flight per thread.
__global__ void __launch_bounds__(256) k_amax(const __nv_bfloat16* __restrict__ x, int64_t nvec, uint32_t* partials) {
  const uint4* p = reinterpret_cast<const uint4*>(x);
  const int64_t T = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t mx = 0;
  int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; v + 3 * T < nvec; v += 4 * T) {
    const uint4 w0 = ld_nc_v4(p + v), w1 = ld_nc_v4(p + v + T), w2 = ld_nc_v4(p + v + 2 * T),
                w3 = ld_nc_v4(p + v + 3 * T);
    mx = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(mx, w0), w1), w2), w3);
  }
  for (; v < nvec; v += T) mx = absmax_bf16x2(mx, ld_nc_v4(p + v));
  cta_max_to(max(mx & 0xFFFFu, mx >> 16) << 16, &partials[blockIdx.x]);
}

// Strided X (ldx > K): one row per warp-iteration.
__global__ void __launch_bounds__(256) k_amax_rows(const __nv_bfloat16* __restrict__ x, int64_t ldx, int M, int K,
                                                   uint32_t* partials) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t mx = 0;
  for (int m = blockIdx.x * 8 + warp; m < M; m += gridDim.x * 8)
    for (int k = 8 * lane; k < K; k += 256) mx = absmax_bf16x2(mx, ld_nc_v4(x + static_cast<int64_t>(m) * ldx + k));
  cta_max_to(max(mx & 0xFFFFu, mx >> 16) << 16, &partials[blockIdx.x]);
}

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

// Persistent, TMA-fed variant of the primary pass. Each CTA walks tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ... of 128 rows x 128 channels; the X tile arrives in shared memory
// as two TMA boxes of 64 channels with 128-byte swizzle (bank-conflict-free 16-byte reads),
// double-buffered so the next tile loads while this one is coded. The tensor scale is reduced
// from the abs-max partials while the first tiles are in flight.
constexpr int kQTileBytes = 128 * 128 * 2;
constexpr int kQuantSmem = 2 * kQTileBytes + 1024 + 1024;

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Shared-memory byte address of 16-byte chunk `c` (0..15) of tile row `row` (two 64-channel
// halves, each rows x 128 bytes with the 128-byte swizzle: chunk j of row r at (j ^ r%8) * 16).
__device__ __forceinline__ uint32_t qtile_chunk(uint32_t base, int row, int c) {
  const int h = c >> 3, j = c & 7;
  return base + h * (128 * 128) + row * 128 + ((j ^ (row & 7)) << 4);
}

template <bool RMS>
__global__ void __launch_bounds__(256) k_quant_stream(const __grid_constant__ CUtensorMap tmX, QuantArgs a,
                                                      int tiles_k, int ntiles, uint64_t wait_ns) {
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* qs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* sf_tile = reinterpret_cast<uint32_t*>(qs + 2 * kQTileBytes);
  __shared__ uint64_t bar[2];
  __shared__ uint32_t omask[4];
  __shared__ int16_t ocol[128];
  __shared__ int abort_sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t xbase = smem_u32(qs);

  auto issue = [&](int t, int buf) {
    const int tm = t / tiles_k, tk = t - (t / tiles_k) * tiles_k;
    mbar_arrive_expect_tx(&bar[buf], kQTileBytes);
    uint8_t* dst = qs + buf * kQTileBytes;
    tma_load_2d(dst, &tmX, &bar[buf], tk * 128, tm * 128);
    tma_load_2d(dst + 128 * 128, &tmX, &bar[buf], tk * 128 + 64, tm * 128);
  };
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_sh = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    if (blockIdx.x < ntiles) issue(blockIdx.x, 0);
    if (blockIdx.x + gridDim.x < ntiles) issue(blockIdx.x + gridDim.x, 1);
  }
  const float s = cta_tensor_scale(a);  // overlaps the first loads; contains __syncthreads
  if (blockIdx.x == 0 && tid == 0) *a.scale_out = s;
  const float rcp_s = __frcp_rn(s), rcp6 = __frcp_rn(6.0f);
  const int b = lane & 7;      // block inside the tile
  const int rsub = lane >> 3;  // row inside the warp's group of 4
  const int64_t cpitch = a.kpad >> 1;
  uint8_t* sfb = reinterpret_cast<uint8_t*>(sf_tile);

  int it = 0;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
    const int buf = it & 1;
    const uint32_t par = (it >> 1) & 1;
    const int tm = t / tiles_k, tk = t - tm * tiles_k;
    const int m0 = tm * 128, k0 = tk * 128;
    __syncthreads();  // the previous tile's scale atoms are written out
    for (int i = tid; i < 256; i += 256) sf_tile[i] = 0;
    if (tid < 4) omask[tid] = 0;
    __syncthreads();
    for (int j = tid; j < a.r; j += 256) {
      const int c = a.idx[j];
      if (c >= k0 && c < k0 + 128) {
        ocol[c - k0] = static_cast<int16_t>(j);
        atomicOr(&omask[(c - k0) >> 5], 1u << ((c - k0) & 31));
      }
    }
    // every thread waits for the tile; a wait that runs out stops the whole CTA
    if (!mbar_wait(&bar[buf], par, wait_ns, &abort_sh)) abort_sh = 1;
    __syncthreads();
    if (abort_sh) break;

    const int kcol = k0 + 16 * b;
    const bool colok = kcol < a.K;
    const uint32_t obits = (omask[b >> 1] >> ((b & 1) * 16)) & 0xFFFFu;
    float g[16];
    if (RMS) {
      uint4 g0 = make_uint4(0, 0, 0, 0), g1 = g0;
      if (colok) {
        g0 = ld_nc_v4(a.gain + kcol);
        g1 = ld_nc_v4(a.gain + kcol + 8);
      }
      const uint32_t gs[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) g[i] = (i & 1) ? bf16_hi(gs[i >> 1]) : bf16_lo(gs[i >> 1]);
    }
    const uint32_t tbase = xbase + buf * kQTileBytes;
#pragma unroll 1
    for (int rg = 0; rg < 4; ++rg) {
      const int mm = rg * 32 + warp * 4 + rsub;
      const int m = m0 + mm;
      const uint4 w0 = lds_v4(qtile_chunk(tbase, mm, 2 * b));
      const uint4 w1 = lds_v4(qtile_chunk(tbase, mm, 2 * b + 1));
      const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      uint64_t p[8];
      float amax;
      double inv = 0.0;
      if (RMS) {
        inv = (m < a.M) ? a.inv_rms[m] : 0.0;
        float mx = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v0 = rms_apply(bf16_lo(ws[j]), inv, g[2 * j]);
          const float v1 = rms_apply(bf16_hi(ws[j]), inv, g[2 * j + 1]);
          mx = fmaxf(mx, fmaxf(fabsf(v0), fabsf(v1)));
          p[j] = f2_pack(v0, v1);
        }
        amax = mx;
      } else {
        uint32_t am2 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          am2 = __vmaxu2(am2, ws[j] & 0x7FFF7FFFu);
          p[j] = f2_pack(bf16_lo(ws[j]), bf16_hi(ws[j]));
        }
        amax = __uint_as_float(max(am2 & 0xFFFFu, am2 >> 16) << 16);
      }
      float d;
      const uint32_t sfv = block_scale(amax, s, rcp_s, rcp6, &d);
      const uint2 codes = (d == 0.0f) ? make_uint2(0u, 0u) : encode16(p, d);
      if (m < a.M && colok) {
        *reinterpret_cast<uint2*>(a.codes + static_cast<int64_t>(m) * cpitch + (kcol >> 1)) = codes;
        sfb[(b >> 2) * 512 + (mm & 31) * 16 + (mm >> 5) * 4 + (b & 3)] = static_cast<uint8_t>(sfv);
        uint32_t ob = obits;
        while (ob) {
          const int e = __ffs(ob) - 1;
          ob &= ob - 1;
          const uint32_t hv = *reinterpret_cast<const uint16_t*>(qs + buf * kQTileBytes +
                                                                 (qtile_chunk(tbase, mm, 2 * b + (e >> 3)) - tbase) +
                                                                 2 * (e & 7));
          float v = __uint_as_float(hv << 16);
          if (RMS) v = rms_apply(v, inv, __bfloat162float(a.gain[kcol + e]));
          const uint32_t c = ((e < 8 ? codes.x : codes.y) >> (4 * (e & 7))) & 15u;
          const float deq = __fmul_rn(e2m1_value(c), d);
          a.stash[static_cast<int64_t>(m) * a.r + ocol[16 * b + e]] = a.dup ? v : __fsub_rn(v, deq);
        }
      }
    }
    __syncthreads();  // tile buffer and scale staging complete
    if (tid == 0 && t + 2 * static_cast<int>(gridDim.x) < ntiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(t + 2 * gridDim.x, buf);
    }
    const int natoms = min(2, (a.K - k0 + 63) >> 6);
    uint4* dst = reinterpret_cast<uint4*>(a.sf + (static_cast<int64_t>(tm) * a.katoms + (k0 >> 6)) * 512);
    const uint4* src = reinterpret_cast<const uint4*>(sf_tile);
    for (int i = tid; i < natoms * 32; i += 256) dst[i] = src[i];
  }
  // loads still in flight after an abort land before the CTA exits
  if (tid == 0 && abort_sh) {
    const uint64_t t0 = globaltimer_ns();
    for (int i = 0; i < 2; ++i)
      while (!mbar_test(&bar[(it + i) & 1], ((it + i) >> 1) & 1) && globaltimer_ns() - t0 < wait_ns) {
      }
  }
}

// One warp per row (rows up to the 128-padded count): appended residual blocks and padding.
__global__ void __launch_bounds__(256) k_quant_tail(QuantArgs a, int mpad) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  if (m >= mpad) return;
  const float s = (a.static_scale) ? *a.static_scale : *a.scale_out;
  const float rcp_s = __frcp_rn(s), rcp6 = __frcp_rn(6.0f);
  const int nres = a.r >> 4;
  const int ntail = (a.kpad - a.K) >> 4;
  const int64_t cpitch = a.kpad >> 1;
  for (int b = lane; b < ntail; b += 32) {
    uint32_t sfv = 0;
    uint2 codes = make_uint2(0u, 0u);
    if (m < a.M && b < nres) {
      const float4* src = reinterpret_cast<const float4*>(a.stash + static_cast<int64_t>(m) * a.r + 16 * b);
      uint64_t p[8];
      float am = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 q = src[i];
        p[2 * i] = f2_pack(q.x, q.y);
        p[2 * i + 1] = f2_pack(q.z, q.w);
        am = fmaxf(am, fmaxf(fmaxf(fabsf(q.x), fabsf(q.y)), fmaxf(fabsf(q.z), fabsf(q.w))));
      }
      float d;
      sfv = block_scale(am, s, rcp_s, rcp6, &d);
      if (d != 0.0f) codes = encode16(p, d);
    }
    if (m < a.M) *reinterpret_cast<uint2*>(a.codes + static_cast<int64_t>(m) * cpitch + ((a.K + 16 * b) >> 1)) = codes;
    a.sf[sf_offset(m, (a.K >> 4) + b, a.katoms)] = static_cast<uint8_t>(sfv);
  }
}

}  // namespace arc
