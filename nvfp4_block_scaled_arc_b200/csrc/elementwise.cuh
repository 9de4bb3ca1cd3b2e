// elementwise.cuh -- the small kernels around the GEMMs: the BF16 path's RMSNorm, the SwiGLU
// gate, and the offline outlier calibration.
#pragma once

#include "quant.cuh"

namespace arc {

// One warp per row: out = RMSNorm(h) * gain, same arithmetic as the fused quantizer prologue.
__global__ void __launch_bounds__(256) k_rmsnorm(const __nv_bfloat16* __restrict__ h, int64_t ldh, int M, int K,
                                                 const __nv_bfloat16* __restrict__ gain, double eps,
                                                 __nv_bfloat16* __restrict__ out, int64_t ldo) {
  pdl_launch_dependents();  // the GEMM that follows may set itself up meanwhile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  if (m >= M) return;
  const __nv_bfloat16* row = h + static_cast<int64_t>(m) * ldh;
  const double inv = warp_row_inv_rms(row, K, eps, lane);
  for (int k = 8 * lane; k < K; k += 256) {
    const uint4 w = ld_nc_v4(row + k);
    const uint4 g = ld_nc_v4(gain + k);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, gs[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = rms_apply(bf16_lo(ws[i]), inv, bf16_lo(gs[i]));
      const float b = rms_apply(bf16_hi(ws[i]), inv, bf16_hi(gs[i]));
      o[i] = (__float_as_uint(a) >> 16) | (__float_as_uint(b) & 0xFFFF0000u);  // already bf16-exact
    }
    *reinterpret_cast<uint4*>(out + static_cast<int64_t>(m) * ldo + k) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// out[m, j] = bf16( silu(g) * u ), g = gu[m, j], u = gu[m, F + j]; silu(g) = g / (1 + exp(-g))
// in fp32 (expf, IEEE divide and multiply). 8 columns per thread, F % 8 == 0.
__global__ void __launch_bounds__(256) k_silu_mul(const __nv_bfloat16* __restrict__ gu, int64_t ld, int M, int F,
                                                  __nv_bfloat16* __restrict__ out, int64_t ldo) {
  pdl_launch_dependents();  // the GEMM that follows may set itself up meanwhile
  const int vpr = F >> 3;
  const int64_t total = static_cast<int64_t>(M) * vpr;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = v / vpr;
    const int j = static_cast<int>(v - m * vpr) * 8;
    const uint4 gw = ld_nc_v4(gu + m * ld + j);
    const uint4 uw = ld_nc_v4(gu + m * ld + F + j);
    const uint32_t gs[4] = {gw.x, gw.y, gw.z, gw.w}, us[4] = {uw.x, uw.y, uw.z, uw.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float r[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float gv = h ? bf16_hi(gs[i]) : bf16_lo(gs[i]);
        const float uv = h ? bf16_hi(us[i]) : bf16_lo(us[i]);
        const float s = __fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv)));
        r[h] = __fmul_rn(s, uv);
      }
      o[i] = pack_bf16x2_rn(r[0], r[1]);
    }
    *reinterpret_cast<uint4*>(out + m * ldo + j) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// h[m, k] = bf16(fp32(beta * h[m, k]) + e[m, k]) in place (e optional), 8 values per thread
// (d % 8 == 0): the damped residual (with input injection) of a contractive recurrent block,
// applied before the sublayer's residual add.
__global__ void __launch_bounds__(256) k_damp_bf16(__nv_bfloat16* __restrict__ h, int64_t ldh, int M, int d,
                                                   float beta, const __nv_bfloat16* __restrict__ e) {
  const int vpr = d >> 3;
  const int64_t total = static_cast<int64_t>(M) * vpr;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = v / vpr;
    const int j = static_cast<int>(v - m * vpr) * 8;
    uint4* p = reinterpret_cast<uint4*>(h + m * ldh + j);
    const uint4 w = *p;
    const uint4 ew = e ? ld_nc_v4(e + m * d + j) : make_uint4(0, 0, 0, 0);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, es[4] = {ew.x, ew.y, ew.z, ew.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __fmul_rn(beta, bf16_lo(ws[i])), hi = __fmul_rn(beta, bf16_hi(ws[i]));
      o[i] = e ? pack_bf16x2_rn(__fadd_rn(lo, bf16_lo(es[i])), __fadd_rn(hi, bf16_hi(es[i]))) : pack_bf16x2_rn(lo, hi);
    }
    *p = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Per-channel max |x| over rows (fp32 bit patterns, atomicMax), channel pairs per thread.
__global__ void __launch_bounds__(256) k_colmax(const __nv_bfloat16* __restrict__ x, int64_t ldx, int M, int K,
                                                int rows_per_cta, uint32_t* colmax) {
  const int kp = blockIdx.x * 256 + threadIdx.x;  // channel pair index
  if (2 * kp >= K) return;
  const int r0 = blockIdx.y * rows_per_cta, r1 = min(M, r0 + rows_per_cta);
  uint32_t mx = 0;
  for (int m = r0; m < r1; ++m) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(x + static_cast<int64_t>(m) * ldx + 2 * kp);
    mx = __vmaxu2(mx, w & 0x7FFF7FFFu);
  }
  if (mx & 0xFFFFu) atomicMax(&colmax[2 * kp], (mx & 0xFFFFu) << 16);
  if (mx >> 16) atomicMax(&colmax[2 * kp + 1], mx & 0xFFFF0000u);
}

// Full calibration order (the channel reorder of ARCQuant's adaptive outlier identification):
// channel c goes to position rank(c) = #{c' : key(c') > key(c)}, key = (abs-max bits << 32) |
// (2^32 - 1 - c), i.e. larger abs-max first and ties by ascending channel. The keys are distinct,
// so the ranks form a permutation and no two threads write the same slot. O(K^2) comparisons
// through shared-memory tiles that every thread of the CTA reads in the same order (broadcast);
// a calibration step, not part of the per-batch path.
__global__ void __launch_bounds__(256) k_order(const uint32_t* colmax, int K, int32_t* perm_out) {
  __shared__ uint64_t tile[2048];
  const int c = blockIdx.x * 256 + threadIdx.x;
  const uint64_t mine = c < K ? (static_cast<uint64_t>(colmax[c]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(c)) : 0;
  int rank = 0;
  for (int t0 = 0; t0 < K; t0 += 2048) {
    const int n = min(2048, K - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += 256)
      tile[i] = (static_cast<uint64_t>(colmax[t0 + i]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(t0 + i));
    __syncthreads();
#pragma unroll 8
    for (int i = 0; i < n; ++i) rank += tile[i] > mine ? 1 : 0;
  }
  if (c < K) perm_out[rank] = c;
}

// Top-r channels by abs-max (descending), ties by ascending index, r rounds of a block-wide
// argmax over 64-bit keys (abs-max bits << 32 | ~index).
__global__ void __launch_bounds__(1024) k_topk(const uint32_t* colmax, int K, int r, uint64_t* keys, int32_t* idx_out) {
  __shared__ uint64_t red[32];
  const int tid = threadIdx.x;
  for (int k = tid; k < K; k += 1024) keys[k] = (static_cast<uint64_t>(colmax[k]) << 32) | (0xFFFFFFFFu - k);
  __syncthreads();
  for (int j = 0; j < r; ++j) {
    uint64_t b = 0;
    for (int k = tid; k < K; k += 1024) b = max(b, keys[k]);
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const uint64_t t = __shfl_xor_sync(0xFFFFFFFFu, b, o);
      b = max(b, t);
    }
    if ((tid & 31) == 0) red[tid >> 5] = b;
    __syncthreads();
    if (tid < 32) {
      uint64_t c = red[tid];
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const uint64_t t = __shfl_xor_sync(0xFFFFFFFFu, c, o);
        c = max(c, t);
      }
      if (tid == 0) {
        const int k = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(c));
        idx_out[j] = k;
        keys[k] = 0;  // taken
      }
    }
    __syncthreads();
  }
}

}  // namespace arc
