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

// ---------------------------------------------------------------------------------------------
// Single-launch quantizer (cooperative launch, one CTA per SM, all CTAs resident).
//   phase 1  (dynamic scale, no RMSNorm): stream the CTA's tiles through a ring of kFusedBufs
//            shared-memory buffers, reduce max |x|, publish one partial per CTA;
//   barrier  every CTA waits for every partial;
//   phase 2  code the tiles: first those still resident in the ring, then the others, which
//            stream through the ring again (mostly L2 hits);
//   barrier  every residual value is in the stash;
//   phase 3  the appended residual blocks and the padding, rows spread over all CTAs.
// The grid barrier needs no initialised memory: each CTA stores the call's epoch (a number the
// host never reuses) in its own flag and waits until every flag shows it, with the usual
// time limit; a wait that runs out sets the status word and stops the CTA.
// ---------------------------------------------------------------------------------------------
constexpr int kFusedThreads = 512;
constexpr int kFusedBufs = 6;
constexpr int kFusedSmem = kFusedBufs * kQTileBytes + 1024 + 1024;

__device__ __forceinline__ bool grid_barrier(volatile unsigned long long* flags, int G, unsigned long long epoch,
                                             uint64_t wait_ns, int* abort_sh) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    flags[blockIdx.x] = epoch;
  }
  const uint64_t t0 = globaltimer_ns();
  bool ok = true;
  for (int i = threadIdx.x; i < G && ok; i += blockDim.x) {
    while (flags[i] != epoch) {
      if (globaltimer_ns() - t0 > wait_ns) {
        ok = false;
        break;
      }
      __nanosleep(64);
    }
  }
  if (!ok) {
    set_status(kStatusTimeout);
    *reinterpret_cast<volatile int*>(abort_sh) = 1;
  }
  __threadfence();
  __syncthreads();
  return *reinterpret_cast<volatile int*>(abort_sh) == 0;
}

struct FusedArgs {
  int tiles_k, ntiles;
  int do_amax;                  // phase 1 runs (dynamic scale without RMSNorm)
  uint32_t* partials;           // [gridDim.x] written by phase 1
  unsigned long long* flags;    // [2 * gridDim.x] barrier flags
  unsigned long long epoch;     // this call's barrier epochs: epoch and epoch + 1
  uint64_t wait_ns;
  int mpad;                     // rows rounded up to 128 (scale padding rows)
};

template <bool RMS>
__device__ __forceinline__ void code_tile(const QuantArgs& a, const uint8_t* tile, uint32_t tbase, int tm, int tk,
                                          float s, float rcp_s, float rcp6, uint32_t* sf_tile, uint32_t* omask,
                                          int16_t* ocol) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = tm * 128, k0 = tk * 128;
  const int b = lane & 7, rsub = lane >> 3;
  const int kcol = k0 + 16 * b;
  const bool colok = kcol < a.K;
  const uint32_t obits = (omask[b >> 1] >> ((b & 1) * 16)) & 0xFFFFu;
  const int64_t cpitch = a.kpad >> 1;
  uint8_t* sfb = reinterpret_cast<uint8_t*>(sf_tile);
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
  // 16 warps x 4 rows per step = 64 rows; two steps cover the 128-row tile
#pragma unroll 1
  for (int rg = 0; rg < 2; ++rg) {
    const int mm = rg * 64 + warp * 4 + rsub;
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
        const uint32_t hv =
            *reinterpret_cast<const uint16_t*>(tile + (qtile_chunk(tbase, mm, 2 * b + (e >> 3)) - tbase) + 2 * (e & 7));
        float v = __uint_as_float(hv << 16);
        if (RMS) v = rms_apply(v, inv, __bfloat162float(a.gain[kcol + e]));
        const uint32_t c = ((e < 8 ? codes.x : codes.y) >> (4 * (e & 7))) & 15u;
        const float deq = __fmul_rn(e2m1_value(c), d);
        a.stash[static_cast<int64_t>(m) * a.r + ocol[16 * b + e]] = a.dup ? v : __fsub_rn(v, deq);
      }
    }
  }
}

// The appended residual blocks (from the stash) and zero padding up to K_pad of one row.
__device__ __forceinline__ void tail_row(const QuantArgs& a, int m, float s, float rcp_s, float rcp6, int lane) {
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

template <bool RMS>
__global__ void __launch_bounds__(kFusedThreads, 1) k_quant_fused(const __grid_constant__ CUtensorMap tmX,
                                                                  QuantArgs a, FusedArgs f) {
  extern __shared__ uint8_t fsmem_raw[];
  uint8_t* qs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fsmem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* sf_tile = reinterpret_cast<uint32_t*>(qs + kFusedBufs * kQTileBytes);
  __shared__ uint64_t bar[kFusedBufs];
  __shared__ uint32_t omask[4];
  __shared__ int16_t ocol[128];
  __shared__ int abort_sh;
  __shared__ int issued_sh;  // slots whose loads thread 0 has issued
  __shared__ float s_sh;
  const int tid = threadIdx.x;
  const int G = gridDim.x;
  const int n_c = (f.ntiles > static_cast<int>(blockIdx.x)) ? (f.ntiles - blockIdx.x + G - 1) / G : 0;
  const uint32_t xbase = smem_u32(qs);
  auto tile_of = [&](int i) { return static_cast<int>(blockIdx.x) + i * G; };  // CTA-local index -> tile
  auto issue = [&](int slot, int i) {
    const int t = tile_of(i);
    const int tm = t / f.tiles_k, tk = t - (t / f.tiles_k) * f.tiles_k;
    const int buf = slot % kFusedBufs;
    mbar_arrive_expect_tx(&bar[buf], kQTileBytes);
    uint8_t* dst = qs + buf * kQTileBytes;
    tma_load_2d(dst, &tmX, &bar[buf], tk * 128, tm * 128);
    tma_load_2d(dst + 128 * 128, &tmX, &bar[buf], tk * 128 + 64, tm * 128);
    issued_sh = slot + 1;
  };
  auto wait_slot = [&](int slot) -> bool {
    if (!mbar_wait(&bar[slot % kFusedBufs], static_cast<uint32_t>((slot / kFusedBufs) & 1), f.wait_ns, &abort_sh))
      abort_sh = 1;
    __syncthreads();
    return abort_sh == 0;
  };
  // after an abort: let every load still in flight land (bounded) before the CTA exits
  auto teardown = [&](int from_slot) {
    if (tid == 0) {
      const uint64_t t0 = globaltimer_ns();
      for (int sl = from_slot; sl < issued_sh; ++sl)
        while (!mbar_test(&bar[sl % kFusedBufs], static_cast<uint32_t>((sl / kFusedBufs) & 1)) &&
               globaltimer_ns() - t0 < f.wait_ns) {
        }
    }
  };
  if (tid == 0) {
    for (int i = 0; i < kFusedBufs; ++i) mbar_init(&bar[i], 1);
    abort_sh = 0;
    issued_sh = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    for (int i = 0; i < min(n_c, kFusedBufs); ++i) issue(i, i);
  }
  __syncthreads();
  int slot = 0;     // next slot to consume
  int resident = 0;  // tiles left in the ring by phase 1 (CTA-local indices n_c-resident .. n_c-1)
  if (f.do_amax) {
    // ------------------------------------------------------------------ phase 1: max |x|
    uint32_t mx = 0;
    for (int i = 0; i < n_c; ++i, ++slot) {
      if (!wait_slot(slot)) {
        teardown(slot);
        return;
      }
      const uint32_t tb = xbase + (slot % kFusedBufs) * kQTileBytes;
      // 512 threads x 4 chunks of 16 bytes = the 32 KB tile
#pragma unroll
      for (int j = 0; j < 4; ++j) mx = absmax_bf16x2(mx, lds_v4(tb + (tid + j * kFusedThreads) * 16));
      __syncthreads();
      if (tid == 0 && i + kFusedBufs < n_c) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(slot + kFusedBufs, i + kFusedBufs);
      }
    }
    cta_max_to(max(mx & 0xFFFFu, mx >> 16) << 16, &f.partials[blockIdx.x]);
    resident = min(n_c, kFusedBufs);
    if (!grid_barrier(f.flags, G, f.epoch, f.wait_ns, &abort_sh)) return;
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
  // processing order: the resident tiles (slots n_c-resident .. n_c-1), then the rest
  const int first_slot = f.do_amax ? n_c - resident : 0;
  const int nproc = n_c;
  for (int q = 0; q < nproc; ++q) {
    const int cur = first_slot + q;  // slot of this tile
    const int i = f.do_amax ? (q < resident ? n_c - resident + q : q - resident) : q;
    const int t = tile_of(i);
    const int tm = t / f.tiles_k, tk = t - tm * f.tiles_k;
    const int k0 = tk * 128;
    __syncthreads();
    for (int j = tid; j < 256; j += kFusedThreads) sf_tile[j] = 0;
    if (tid < 4) omask[tid] = 0;
    __syncthreads();
    for (int j = tid; j < a.r; j += kFusedThreads) {
      const int c = a.idx[j];
      if (c >= k0 && c < k0 + 128) {
        ocol[c - k0] = static_cast<int16_t>(j);
        atomicOr(&omask[(c - k0) >> 5], 1u << ((c - k0) & 31));
      }
    }
    const bool loaded = f.do_amax && q < resident;  // already waited for in phase 1
    if (!loaded) {
      if (!wait_slot(cur)) {
        teardown(cur);
        return;
      }
    } else {
      __syncthreads();
    }
    const int buf = cur % kFusedBufs;
    code_tile<RMS>(a, qs + buf * kQTileBytes, xbase + buf * kQTileBytes, tm, tk, s, rcp_s, rcp6, sf_tile, omask,
                   ocol);
    __syncthreads();
    // the next load into this buffer: the tile kFusedBufs slots later, if any
    const int next = q + kFusedBufs;
    if (tid == 0 && next < nproc) {
      const int inext = f.do_amax ? (next < resident ? -1 : next - resident) : next;
      if (inext >= 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(cur + kFusedBufs, inext);
      }
    }
    const int natoms = min(2, (a.K - k0 + 63) >> 6);
    uint4* dst = reinterpret_cast<uint4*>(a.sf + (static_cast<int64_t>(tm) * a.katoms + (k0 >> 6)) * 512);
    const uint4* src = reinterpret_cast<const uint4*>(sf_tile);
    for (int j = tid; j < natoms * 32; j += kFusedThreads) dst[j] = src[j];
  }
  if (a.kpad == a.K) return;
  // ---------------------------------------------------------------------- phase 3: tail
  if (!grid_barrier(f.flags + G, G, f.epoch + 1, f.wait_ns, &abort_sh)) return;
  const int warp = tid >> 5, lane = tid & 31;
  for (int m = blockIdx.x * (kFusedThreads / 32) + warp; m < f.mpad; m += G * (kFusedThreads / 32))
    tail_row(a, m, s, rcp_s, rcp6, lane);
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
