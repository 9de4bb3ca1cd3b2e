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
//   k_amax        whole-tensor max |x| (16-byte loads, integer max on |bf16| bit patterns,
//                 one atomicMax per CTA) -> workspace word
//   k_row_stats   one warp per row: exact sum of squares -> 1/rms (double), and with a dynamic
//                 scale the max |RMSNorm(x)| as well
//   k_quant_main  CTA tile 128 rows x 256 channels: 8 warps x 16 rows, one 16-byte load per
//                 lane per row (a lane pair owns a block), codes stored as 4 bytes per lane
//                 (128 contiguous bytes per warp), scale bytes staged in shared memory and
//                 written as whole 512-byte atoms; outlier channels leave x (weights) or
//                 x - deq (activations) in a [rows, r] fp32 stash
//   k_quant_tail  one warp per row: the r/16 appended blocks from the stash plus zero padding
//                 up to K_pad, including the zero scale bytes of padding rows
#pragma once

#include "arc_device.cuh"

namespace arc {

struct QuantArgs {
  const __nv_bfloat16* x;
  int64_t ldx;
  int M, K, r, kpad, katoms;
  const int32_t* idx;
  const __nv_bfloat16* gain;  // RMSNorm prologue gain, or nullptr
  const double* inv_rms;      // [M] from k_row_stats when gain != nullptr
  const float* static_scale;  // or nullptr (dynamic)
  const uint32_t* amax_word;  // fp32 bits of max |x| (dynamic)
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

__device__ __forceinline__ float tensor_scale_of(const QuantArgs& a) {
  if (a.static_scale) return *a.static_scale;
  const float am = __uint_as_float(*a.amax_word);
  return am > 0.0f ? __fdiv_rn(am, 2688.0f) : 1.0f;
}

// Byte offset of scale (row m, scale column kb) in the swizzled layout.
__device__ __forceinline__ int64_t sf_offset(int64_t m, int64_t kb, int katoms) {
  return ((m >> 7) * katoms + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

// Codes of up to 8 values against decode scale d (d > 0): E2M1 of the correctly rounded
// quotient, sign bit taken from the value.
__device__ __forceinline__ uint32_t encode8(const float (&v)[8], float d) {
  float q[8];
  if (d >= 7.888609052210118e-31f && d <= 1.2676506002282294e30f) {  // [2^-100, 2^100]
    const float rcp = __frcp_rn(d);
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = div_rn_from_rcp(v[e], d, rcp);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = __fdiv_rn(v[e], d);
  }
  uint32_t c = e2m1x8_rn_sat(q) & 0x77777777u;
#pragma unroll
  for (int e = 0; e < 8; ++e) c |= (__float_as_uint(v[e]) >> 31) << (4 * e + 3);
  return c;
}

// Scale byte and decode scale of a block with abs-max `amax` under tensor scale s.
__device__ __forceinline__ uint32_t block_scale(float amax, float s, float* d) {
  const float t = __fdiv_rn(__fdiv_rn(amax, 6.0f), s);
  const uint32_t sfb = e4m3_rn_sat(t);
  *d = __fmul_rn(e4m3_value(sfb), s);
  return sfb;
}

// RMSNorm of one bf16 value: bf16( fp32( (h * inv) * g ) ), products in double.
__device__ __forceinline__ float rms_apply(float h, double inv, float g) {
  const double t = __dmul_rn(__dmul_rn(static_cast<double>(h), inv), static_cast<double>(g));
  return __bfloat162float(__float2bfloat16_rn(__double2float_rn(t)));
}

// ---------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256) k_amax(const __nv_bfloat16* __restrict__ x, int64_t ldx, int M, int K,
                                              uint32_t* amax_word) {
  const int vpr = K >> 3;  // 16-byte vectors per row
  const int64_t total = static_cast<int64_t>(M) * vpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t mx = 0;
  int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (ldx == K) {
    const uint4* p = reinterpret_cast<const uint4*>(x);
    for (; v + 3 * stride < total; v += 4 * stride) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = ld_nc_v4(p + v + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mx = __vmaxu2(mx, w[u].x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, w[u].y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, w[u].z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, w[u].w & 0x7FFF7FFFu);
      }
    }
    for (; v < total; v += stride) {
      const uint4 w = ld_nc_v4(p + v);
      mx = __vmaxu2(mx, w.x & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.y & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.z & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.w & 0x7FFF7FFFu);
    }
  } else {
    for (; v < total; v += stride) {
      const int64_t m = v / vpr, c = v - m * vpr;
      const uint4 w = ld_nc_v4(x + m * ldx + 8 * c);
      mx = __vmaxu2(mx, w.x & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.y & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.z & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, w.w & 0x7FFF7FFFu);
    }
  }
  uint32_t m16 = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o; o >>= 1) m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m16;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b = max(b, red[i]);
    if (b) atomicMax(amax_word, b << 16);
  }
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
#pragma unroll
  for (int o = 16; o; o >>= 1) emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
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

// One warp per row: inv_rms[m]; with amax_word != nullptr also max |RMSNorm(h) * g|.
__global__ void __launch_bounds__(256) k_row_stats(const __nv_bfloat16* __restrict__ h, int64_t ldh, int M, int K,
                                                   const __nv_bfloat16* __restrict__ gain, double eps,
                                                   double* inv_rms, uint32_t* amax_word) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  uint32_t mx = 0;
  if (m < M) {
    const __nv_bfloat16* row = h + static_cast<int64_t>(m) * ldh;
    const double inv = warp_row_inv_rms(row, K, eps, lane);
    if (lane == 0) inv_rms[m] = inv;
    if (amax_word) {
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
  if (amax_word) {
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0 && mx) atomicMax(amax_word, mx);
  }
}

// ---------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256) k_quant_main(QuantArgs a) {
  __shared__ __align__(16) uint32_t sf_tile[4 * 128];
  __shared__ uint32_t omask[8];
  __shared__ int16_t ocol[256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * 128, k0 = blockIdx.y * 256;
  for (int i = tid; i < 4 * 128; i += 256) sf_tile[i] = 0;
  if (tid < 8) omask[tid] = 0;
  __syncthreads();
  for (int j = tid; j < a.r; j += 256) {
    const int c = a.idx[j];
    if (c >= k0 && c < k0 + 256) {
      ocol[c - k0] = static_cast<int16_t>(j);
      atomicOr(&omask[(c - k0) >> 5], 1u << ((c - k0) & 31));
    }
  }
  const float s = tensor_scale_of(a);
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *a.scale_out = s;
  __syncthreads();

  const int kcol = k0 + 8 * lane;
  const bool colok = kcol < a.K;
  const uint32_t obits = (omask[lane >> 2] >> ((lane & 3) * 8)) & 0xFFu;
  float g[8];
  if (a.gain) {
    uint4 gw = make_uint4(0, 0, 0, 0);
    if (colok) gw = ld_nc_v4(a.gain + kcol);
    const uint32_t gs[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = (i & 1) ? bf16_hi(gs[i >> 1]) : bf16_lo(gs[i >> 1]);
  }
  uint8_t* sfb = reinterpret_cast<uint8_t*>(sf_tile);
  const int blk = lane >> 1;  // block index inside the tile (0..15)
  const int64_t cpitch = a.kpad >> 1;

#pragma unroll 1
  for (int i = 0; i < 16; i += 4) {
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int m = m0 + warp * 16 + i + u;
      w[u] = make_uint4(0, 0, 0, 0);
      if (m < a.M && colok) w[u] = ld_nc_v4(a.x + static_cast<int64_t>(m) * a.ldx + kcol);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int mm = warp * 16 + i + u;  // row inside the tile
      const int m = m0 + mm;
      const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = (e & 1) ? bf16_hi(ws[e >> 1]) : bf16_lo(ws[e >> 1]);
      if (a.gain && m < a.M) {
        const double inv = a.inv_rms[m];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = rms_apply(v[e], inv, g[e]);
      }
      float am = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(v[e]));
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
      float d;
      const uint32_t sfv = block_scale(am, s, &d);
      const uint32_t codes = (d == 0.0f) ? 0u : encode8(v, d);
      if (m < a.M && colok) {
        *reinterpret_cast<uint32_t*>(a.codes + static_cast<int64_t>(m) * cpitch + (kcol >> 1)) = codes;
        if ((lane & 1) == 0) sfb[(blk >> 2) * 512 + (mm & 31) * 16 + (mm >> 5) * 4 + (blk & 3)] = static_cast<uint8_t>(sfv);
        if (obits) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if ((obits >> e) & 1u) {
              const int j = ocol[8 * lane + e];
              const float deq = __fmul_rn(e2m1_value((codes >> (4 * e)) & 15u), d);
              a.stash[static_cast<int64_t>(m) * a.r + j] = a.dup ? v[e] : __fsub_rn(v[e], deq);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  // whole atoms that hold primary blocks (a partly residual atom is finished by k_quant_tail)
  const int natoms = min(4, (a.K - k0 + 63) >> 6);
  uint4* dst = reinterpret_cast<uint4*>(a.sf + (static_cast<int64_t>(blockIdx.x) * a.katoms + (k0 >> 6)) * 512);
  const uint4* src = reinterpret_cast<const uint4*>(sf_tile);
  for (int t = tid; t < natoms * 32; t += 256) dst[t] = src[t];
}

// One warp per row (rows up to the 128-padded count): appended residual blocks and padding.
__global__ void __launch_bounds__(256) k_quant_tail(QuantArgs a, int mpad) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  if (m >= mpad) return;
  const float s = (a.static_scale) ? *a.static_scale : *a.scale_out;
  const int nres = a.r >> 4;
  const int ntail = (a.kpad - a.K) >> 4;
  const int64_t cpitch = a.kpad >> 1;
  for (int b = lane; b < ntail; b += 32) {
    uint32_t sfv = 0, c0 = 0, c1 = 0;
    if (m < a.M && b < nres) {
      const float4* p = reinterpret_cast<const float4*>(a.stash + static_cast<int64_t>(m) * a.r + 16 * b);
      float v0[8], v1[8];
      const float4 q0 = p[0], q1 = p[1], q2 = p[2], q3 = p[3];
      v0[0] = q0.x; v0[1] = q0.y; v0[2] = q0.z; v0[3] = q0.w;
      v0[4] = q1.x; v0[5] = q1.y; v0[6] = q1.z; v0[7] = q1.w;
      v1[0] = q2.x; v1[1] = q2.y; v1[2] = q2.z; v1[3] = q2.w;
      v1[4] = q3.x; v1[5] = q3.y; v1[6] = q3.z; v1[7] = q3.w;
      float am = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) am = fmaxf(am, fmaxf(fabsf(v0[e]), fabsf(v1[e])));
      float d;
      sfv = block_scale(am, s, &d);
      if (d != 0.0f) {
        c0 = encode8(v0, d);
        c1 = encode8(v1, d);
      }
    }
    if (m < a.M)
      *reinterpret_cast<uint2*>(a.codes + static_cast<int64_t>(m) * cpitch + ((a.K + 16 * b) >> 1)) = make_uint2(c0, c1);
    a.sf[sf_offset(m, (a.K >> 4) + b, a.katoms)] = static_cast<uint8_t>(sfv);
  }
}

}  // namespace arc
