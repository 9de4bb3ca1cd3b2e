// libarc.cu -- the C ABI declared in include/arc.h: argument checks, launch configuration,
// TMA tensor-map encoding, the device status word, and the recurrent prefill driver.
// Single translation unit: every kernel of the library is included here.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/arc.h"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "quant.cuh"

namespace {

using arc::GemmArgs;
using arc::QuantArgs;

uint64_t g_wait_ns = 2000000000ull;  // 2 s
int g_inject = 0;
std::mutex g_mu;

struct DeviceInfo {
  bool ok = false;
  int sms = 0;
  bool attrs_set = false;
};
DeviceInfo g_dev[64];

inline cudaStream_t S(arc_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

arc_status device_check(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARC_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ok) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return ARC_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return ARC_ERR_CUDA;
    if (major != 10 || minor != 0) return ARC_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ARC_ERR_CUDA;
    d.ok = true;
  }
  if (!d.attrs_set) {
    if (cudaFuncSetAttribute(arc::k_gemm<arc::kGemmFP4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmFP4>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmFP4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmFP4>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmBF16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmBF16>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmBF16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmBF16>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmFP8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmFP8>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmFP8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmFP8>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_quant_rows<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::kQRowsSmemMax) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_quant_rows<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::kQRowsSmemMax) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmMX4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmMX4>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_gemm<arc::kGemmMX4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::gemm_smem_bytes<arc::kGemmMX4>()) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_quant_mx_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::kQRowsSmemMax) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_quant_reordered<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::kQReoSmemMax) != cudaSuccess ||
        cudaFuncSetAttribute(arc::k_quant_reordered<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             arc::kQReoSmemMax) != cudaSuccess)
      return ARC_ERR_CUDA;
    d.attrs_set = true;
  }
  if (sms) *sms = d.sms;
  return ARC_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }
inline arc_status launch_status() { return cudaGetLastError() == cudaSuccess ? ARC_OK : ARC_ERR_CUDA; }

// ---------------------------------------------------------------------------------------------
// Tensor maps
// ---------------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] with a row pitch in bytes, box [box_outer, box_inner],
// 128-byte swizzle (box_inner * element size == 128 bytes), zero fill out of bounds.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Y [outer, inner] bf16, row pitch in bytes, as the target of 32-row x 16-column TMA stores
// (no swizzle; the staging chunk is 32 rows of 32 bytes).
bool make_store_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {16, 32};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The armed failure injection if it is of this kind (it is then disarmed), else 0.
int take_inject(int kind) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_inject != kind) return 0;
  g_inject = 0;
  return kind;
}

// ---------------------------------------------------------------------------------------------
// Quantization driver shared by activations and weights
// ---------------------------------------------------------------------------------------------

// Quantizer workspace: per-CTA abs-max partials | 1/rms per row (double, RMSNorm prologue only).
// Nothing in it needs to be initialised.
struct QuantWs {
  uint32_t* partials;
  double* inv_rms;
};

constexpr int64_t kPartialBytes = arc::kMaxPartials * 4;

QuantWs carve_quant_ws(void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  QuantWs w;
  w.partials = reinterpret_cast<uint32_t*>(b);
  w.inv_rms = reinterpret_cast<double*>(b + kPartialBytes);
  return w;
}

// Quantization driver shared by activations and weights, in the natural channel order (idx lists
// the outlier channels) or reordered (perm != nullptr: primary channel p is input channel perm[p]
// and the outlier channels are perm[0 .. r)).
// The checks of the quantizer's arguments that need neither the workspace nor the device, in the
// order every quantizer entry point reports them.
arc_status quantize_check(const void* x, int64_t M, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                          const void* gain, uint8_t* codes, uint8_t* sf, float* scale_out,
                          const int32_t* perm) {
  if (!x || !codes || !sf || !scale_out) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 16 || r < 0 || r % 16 || r > K || ldx < K) return ARC_ERR_INVALID_ARG;
  if (!perm && r > 0 && !idx) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || K > (1ll << 20) || r > 32767) return ARC_ERR_UNSUPPORTED;
  if (perm ? arc::qreo_smem_bytes(static_cast<int>(K)) > static_cast<size_t>(arc::kQReoSmemMax)
           : arc::qrows_warps(static_cast<int>(K), r) < 1)
    return ARC_ERR_UNSUPPORTED;
  if (!al16(x) || (ldx * 2) % 16 || !al16(codes) || !al16(sf) || (gain && !al16(gain)) || (perm && !al16(perm)))
    return ARC_ERR_ALIGNMENT;
  return ARC_OK;
}

arc_status quantize_common(const void* x, int64_t M, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                           const void* gain, float eps, const float* static_scale, uint8_t* codes, uint8_t* sf,
                           float* scale_out, void* workspace, size_t ws_bytes, arc_stream_t stream, int dup,
                           const int32_t* perm = nullptr) {
  arc_status st = quantize_check(x, M, K, ldx, idx, r, gain, codes, sf, scale_out, perm);
  if (st != ARC_OK) return st;
  const int qwarps = arc::qrows_warps(static_cast<int>(K), r);
  const size_t smem = perm ? arc::qreo_smem_bytes(static_cast<int>(K))
                           : arc::qrows_smem_bytes(static_cast<int>(K), r, qwarps);
  if (!workspace || ws_bytes < arc_quantize_workspace_bytes(M, r)) return ARC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  st = device_check(&sms);
  if (st != ARC_OK) return st;
  cudaStream_t s = S(stream);
  QuantWs w = carve_quant_ws(workspace);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(gain);
  int npartials = 0;
  bool first = false;
  if (gain) {
    // RMSNorm statistics (and, with a dynamic scale, the abs-max of the normalised rows) first
    npartials = static_cast<int>(std::min<int64_t>((M + 7) / 8, arc::kMaxPartials));
    arc::k_row_stats<<<static_cast<unsigned>(npartials), 256, 0, s>>>(xb, ldx, static_cast<int>(M),
                                                                     static_cast<int>(K), gb, static_cast<double>(eps),
                                                                     w.inv_rms, static_scale ? nullptr : w.partials);
    if ((st = launch_status()) != ARC_OK) return st;
    first = true;
  } else if (!static_scale) {
    // a persistent streaming grid: four 256-thread CTAs per SM, each thread many 16-byte loads
    const int64_t items = M * ((K + arc::kAmaxSeg - 1) / arc::kAmaxSeg);
    npartials = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>({(items + 7) / 8, static_cast<int64_t>(sms) * 4, arc::kMaxPartials})));
    arc::k_amax<<<static_cast<unsigned>(npartials), 256, 0, s>>>(xb, ldx, static_cast<int>(M), static_cast<int>(K),
                                                                w.partials);
    if ((st = launch_status()) != ARC_OK) return st;
    first = true;
  }
  QuantArgs a;
  a.x = xb;
  a.ldx = ldx;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.r = r;
  a.kpad = static_cast<int>(arc_kpad(K + r));
  a.katoms = a.kpad / 64;
  a.idx = idx;
  a.gain = gb;
  a.inv_rms = w.inv_rms;
  a.static_scale = static_scale;
  a.partials = w.partials;
  a.npartials = npartials;
  a.scale_out = scale_out;
  a.codes = codes;
  a.sf = sf;
  a.dup = dup;
  a.wait_ns = g_wait_ns;
  a.inject = perm ? take_inject(2) : 0;
  const int mpad = static_cast<int>((M + 127) / 128 * 128);
  // the second launch may begin while the first one runs; it waits for the first one's results
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  if (perm) {
    const void* rk = gain ? reinterpret_cast<const void*>(arc::k_quant_reordered<true>)
                          : reinterpret_cast<const void*>(arc::k_quant_reordered<false>);
    int rper_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&rper_sm, rk, arc::kQReoThreads, smem) != cudaSuccess ||
        rper_sm < 1)
      return ARC_ERR_CUDA;
    cudaLaunchConfig_t rc = {};
    rc.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(mpad, static_cast<int64_t>(sms) * rper_sm)));
    rc.blockDim = dim3(arc::kQReoThreads);
    rc.dynamicSmemBytes = smem;
    rc.stream = s;
    rc.attrs = pdl;
    rc.numAttrs = first ? 1 : 0;
    const cudaError_t re = gain ? cudaLaunchKernelEx(&rc, arc::k_quant_reordered<true>, a, perm, mpad)
                                : cudaLaunchKernelEx(&rc, arc::k_quant_reordered<false>, a, perm, mpad);
    return re == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
  }
  const void* kern = gain ? reinterpret_cast<const void*>(arc::k_quant_rows<true>)
                          : reinterpret_cast<const void*>(arc::k_quant_rows<false>);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, qwarps * 32, smem) != cudaSuccess || per_sm < 1)
    return ARC_ERR_CUDA;
  // one warp per row at a time, rows dealt round-robin over one resident wave of CTAs (every SM
  // then holds the same number of rows to within one per CTA)
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(mpad, static_cast<int64_t>(sms) * per_sm));
  // the second launch may begin while the first one runs; it waits for the first one's results
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(static_cast<unsigned>(qwarps * 32));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = first ? 1 : 0;
  const cudaError_t e = gain ? cudaLaunchKernelEx(&cfg, arc::k_quant_rows<true>, a, mpad)
                             : cudaLaunchKernelEx(&cfg, arc::k_quant_rows<false>, a, mpad);
  return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

// MXFP4 quantization driver (activations: residuals appended; weights: channels duplicated).
arc_status quantize_mx(const void* x, int64_t M, int64_t K, int64_t ldx, const int32_t* idx, int32_t r,
                       uint8_t* codes, uint8_t* sf, arc_stream_t stream, int dup) {
  if (!x || !codes || !sf) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 32 || r < 0 || r % 32 || r > K || ldx < K || (r > 0 && !idx)) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || K > (1ll << 20) || r > 32767) return ARC_ERR_UNSUPPORTED;
  const int warps = arc::qmx_warps(static_cast<int>(K), r);
  if (warps < 1) return ARC_ERR_UNSUPPORTED;
  if (!al16(x) || (ldx * 2) % 16 || !al16(codes) || !al16(sf)) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  const size_t smem = arc::qmx_smem_bytes(static_cast<int>(K), r, warps);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, arc::k_quant_mx_rows, warps * 32, smem) != cudaSuccess ||
      per_sm < 1)
    return ARC_ERR_CUDA;
  arc::QuantMxArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.ldx = ldx;
  a.M = static_cast<int>(M);
  a.K = static_cast<int>(K);
  a.r = r;
  a.kpad = static_cast<int>(arc_kpad(K + r));
  a.katoms = (a.kpad + 127) / 128;
  a.idx = idx;
  a.codes = codes;
  a.sf = sf;
  a.dup = dup;
  const int mpad = static_cast<int>((M + 127) / 128 * 128);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(mpad, static_cast<int64_t>(sms) * per_sm));
  arc::k_quant_mx_rows<<<grid, warps * 32, smem, S(stream)>>>(a, mpad);
  return launch_status();
}

// ---------------------------------------------------------------------------------------------
// GEMM driver
// ---------------------------------------------------------------------------------------------

template <int KIND>
arc_status gemm_launch(const CUtensorMap& ta, const CUtensorMap& tb, GemmArgs g, int sms, bool add,
                       cudaStream_t s) {
  const int ntiles = g.tiles_m * g.tiles_n;
  const unsigned grid = static_cast<unsigned>(std::min(ntiles, sms));
  // raster groups: as many 128-row blocks of A as fit in about 36 MB (well inside the 126 MB L2,
  // beside the streaming B block and output), split into groups of equal size; B is then read
  // from HBM once per group
  {
    const int64_t a_row_bytes = static_cast<int64_t>(g.ksteps) * (KIND == arc::kGemmFP4 ? 36 : KIND == arc::kGemmMX4 ? 34 : 32);
    const int64_t gm_max = std::max<int64_t>(1, (36ll << 20) / (128 * a_row_bytes));
    const int64_t ngroups = (g.tiles_m + gm_max - 1) / gm_max;
    g.group_m = static_cast<int>((g.tiles_m + ngroups - 1) / ngroups);
  }
  const int smem = arc::gemm_smem_bytes<KIND>();
  CUtensorMap ty;
  std::memset(&ty, 0, sizeof(ty));
  if (!add && !make_store_map(&ty, g.y, static_cast<uint64_t>(g.N), static_cast<uint64_t>(g.M),
                              static_cast<uint64_t>(g.ldy) * 2))
    return ARC_ERR_CUDA;
  // programmatic dependent launch: the set-up (tensor memory, barriers, descriptor prefetch)
  // overlaps the tail of the kernel before it; the kernel waits for it before any other work
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(arc::kGemmThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = add ? cudaLaunchKernelEx(&cfg, arc::k_gemm<KIND, true>, ta, tb, ty, g)
                            : cudaLaunchKernelEx(&cfg, arc::k_gemm<KIND, false>, ta, tb, ty, g);
  return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

}  // namespace

// =============================================================================================
// C ABI
// =============================================================================================

extern "C" {

const char* arc_status_str(arc_status s) {
  switch (s) {
    case ARC_OK: return "ARC_OK";
    case ARC_ERR_INVALID_ARG: return "ARC_ERR_INVALID_ARG";
    case ARC_ERR_ALIGNMENT: return "ARC_ERR_ALIGNMENT";
    case ARC_ERR_UNSUPPORTED: return "ARC_ERR_UNSUPPORTED";
    case ARC_ERR_CUDA: return "ARC_ERR_CUDA";
    case ARC_ERR_TIMEOUT: return "ARC_ERR_TIMEOUT";
    case ARC_ERR_WORKSPACE: return "ARC_ERR_WORKSPACE";
  }
  return "ARC_ERR_UNKNOWN";
}

int64_t arc_kpad(int64_t k_aug) { return (k_aug + 63) / 64 * 64; }

size_t arc_nvfp4_codes_bytes(int64_t rows, int64_t k_aug) {
  if (rows <= 0 || k_aug <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(arc_kpad(k_aug) / 2);
}

size_t arc_nvfp4_sf_bytes(int64_t rows, int64_t k_aug) {
  if (rows <= 0 || k_aug <= 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>(arc_kpad(k_aug) / 64) * 512u;
}

size_t arc_mxfp4_sf_bytes(int64_t rows, int64_t k_aug) {
  if (rows <= 0 || k_aug <= 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((arc_kpad(k_aug) + 127) / 128) * 512u;
}

size_t arc_quantize_workspace_bytes(int64_t rows, int32_t r) {
  if (rows < 0 || r < 0) return 0;
  return static_cast<size_t>(kPartialBytes + align256(rows * 8));
}

size_t arc_calibrate_workspace_bytes(int64_t K) {
  if (K <= 0) return 0;
  return static_cast<size_t>(align256(K * 4) + align256(K * 8));
}

arc_status arc_quantize_act_nvfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const int32_t* d_idx,
                                  int32_t r, const void* rms_gain_bf16, float rms_eps, const float* d_static_scale,
                                  uint8_t* codes, uint8_t* sf, float* d_scale_out, void* workspace, size_t ws_bytes,
                                  arc_stream_t stream) {
  return quantize_common(x_bf16, M, K, ldx, d_idx, r, rms_gain_bf16, rms_eps, d_static_scale, codes, sf,
                         d_scale_out, workspace, ws_bytes, stream, 0);
}

arc_status arc_pack_weight_nvfp4(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, const int32_t* d_idx,
                                 int32_t r, uint8_t* codes, uint8_t* sf, float* d_scale_out, void* workspace,
                                 size_t ws_bytes, arc_stream_t stream) {
  return quantize_common(w_bf16, N, K, ldw, d_idx, r, nullptr, 0.0f, nullptr, codes, sf, d_scale_out, workspace,
                         ws_bytes, stream, 1);
}

arc_status arc_calibrate_outliers(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int32_t r,
                                  int32_t* d_idx_out, void* workspace, size_t ws_bytes, arc_stream_t stream) {
  if (!x_bf16 || !d_idx_out) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 2 || ldx < K || r <= 0 || r > K || r > 1024) return ARC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 3u) || ldx % 2) return ARC_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < arc_calibrate_workspace_bytes(K)) return ARC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  cudaStream_t s = S(stream);
  uint32_t* colmax = static_cast<uint32_t*>(workspace);
  uint64_t* keys = reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(workspace) + align256(K * 4));
  if (cudaMemsetAsync(colmax, 0, static_cast<size_t>(K) * 4, s) != cudaSuccess) return ARC_ERR_CUDA;
  const int rows_per_cta = 64;
  dim3 grid(static_cast<unsigned>((K / 2 + 255) / 256), static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
  arc::k_colmax<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x_bf16), ldx, static_cast<int>(M),
                                     static_cast<int>(K), rows_per_cta, colmax);
  if ((st = launch_status()) != ARC_OK) return st;
  arc::k_topk<<<1, 1024, 0, s>>>(colmax, static_cast<int>(K), r, keys, d_idx_out);
  return launch_status();
}

arc_status arc_calibrate_order(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int32_t* d_perm_out,
                               void* workspace, size_t ws_bytes, arc_stream_t stream) {
  if (!x_bf16 || !d_perm_out) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 2 || ldx < K) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || K > (1ll << 20)) return ARC_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 3u) || ldx % 2) return ARC_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < arc_calibrate_workspace_bytes(K)) return ARC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  cudaStream_t s = S(stream);
  uint32_t* colmax = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(colmax, 0, static_cast<size_t>(K) * 4, s) != cudaSuccess) return ARC_ERR_CUDA;
  const int rows_per_cta = 64;
  dim3 grid(static_cast<unsigned>((K / 2 + 255) / 256), static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
  arc::k_colmax<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x_bf16), ldx, static_cast<int>(M),
                                     static_cast<int>(K), rows_per_cta, colmax);
  if ((st = launch_status()) != ARC_OK) return st;
  arc::k_order<<<static_cast<unsigned>((K + 255) / 256), 256, 0, s>>>(colmax, static_cast<int>(K), d_perm_out);
  return launch_status();
}

arc_status arc_quantize_act_nvfp4_reordered(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                            const int32_t* d_perm, int32_t r, const void* rms_gain_bf16,
                                            float rms_eps, const float* d_static_scale, uint8_t* codes, uint8_t* sf,
                                            float* d_scale_out, void* workspace, size_t ws_bytes,
                                            arc_stream_t stream) {
  if (!d_perm) return ARC_ERR_INVALID_ARG;
  return quantize_common(x_bf16, M, K, ldx, nullptr, r, rms_gain_bf16, rms_eps, d_static_scale, codes, sf,
                         d_scale_out, workspace, ws_bytes, stream, 0, d_perm);
}

arc_status arc_pack_weight_nvfp4_reordered(const void* w_bf16, int64_t N, int64_t K, int64_t ldw,
                                           const int32_t* d_perm, int32_t r, uint8_t* codes, uint8_t* sf,
                                           float* d_scale_out, void* workspace, size_t ws_bytes,
                                           arc_stream_t stream) {
  if (!d_perm) return ARC_ERR_INVALID_ARG;
  return quantize_common(w_bf16, N, K, ldw, nullptr, r, nullptr, 0.0f, nullptr, codes, sf, d_scale_out, workspace,
                         ws_bytes, stream, 1, d_perm);
}

arc_status arc_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sf, const float* d_a_scale,
                          const uint8_t* b_codes, const uint8_t* b_sf, const float* d_b_scale, int64_t M, int64_t N,
                          int64_t k_aug, void* y_bf16, int64_t ldy, const void* add_bf16, int64_t ld_add,
                          arc_stream_t stream) {
  if (!a_codes || !a_sf || !d_a_scale || !b_codes || !b_sf || !d_b_scale || !y_bf16) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || k_aug <= 0 || N % 8 || ldy < N || ldy % 8) return ARC_ERR_INVALID_ARG;
  if (add_bf16 && (ld_add < N || ld_add % 8)) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || k_aug > (1ll << 24)) return ARC_ERR_UNSUPPORTED;
  if (!al16(a_codes) || !al16(a_sf) || !al16(b_codes) || !al16(b_sf) || !al16(y_bf16) ||
      (add_bf16 && !al16(add_bf16)))
    return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  const int64_t kpad = arc_kpad(k_aug);
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.ksteps = static_cast<int>(kpad / 64);
  g.kstages = (g.ksteps + 3) / 4;
  g.katoms = g.ksteps;
  g.nblk128 = static_cast<int>((N + 127) / 128);
  g.tiles_m = static_cast<int>((M + 127) / 128);
  g.tiles_n = static_cast<int>((N + 255) / 256);
  g.box_rows_a = static_cast<int>(std::min<int64_t>(128, M));
  g.box_rows_b = static_cast<int>(std::min<int64_t>(256, N));
  g.sfa = a_sf;
  g.sfb = b_sf;
  g.a_scale = d_a_scale;
  g.b_scale = d_b_scale;
  g.y = static_cast<__nv_bfloat16*>(y_bf16);
  g.ldy = ldy;
  g.add = static_cast<const __nv_bfloat16*>(add_bf16);
  g.ld_add = ld_add;
  g.wait_ns = g_wait_ns;
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(kpad / 2),
                static_cast<uint64_t>(M), static_cast<uint64_t>(kpad / 2), 128, g.box_rows_a) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, static_cast<uint64_t>(kpad / 2),
                static_cast<uint64_t>(N), static_cast<uint64_t>(kpad / 2), 128, g.box_rows_b))
    return ARC_ERR_CUDA;
  g.inject = take_inject(1);
  return gemm_launch<arc::kGemmFP4>(ta, tb, g, sms, add_bf16 != nullptr, S(stream));
}

arc_status arc_quantize_act_mxfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const int32_t* d_idx,
                                  int32_t r, uint8_t* codes, uint8_t* sf, arc_stream_t stream) {
  return quantize_mx(x_bf16, M, K, ldx, d_idx, r, codes, sf, stream, 0);
}

arc_status arc_pack_weight_mxfp4(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, const int32_t* d_idx,
                                 int32_t r, uint8_t* codes, uint8_t* sf, arc_stream_t stream) {
  return quantize_mx(w_bf16, N, K, ldw, d_idx, r, codes, sf, stream, 1);
}

arc_status arc_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes, const uint8_t* b_sf,
                          int64_t M, int64_t N, int64_t k_aug, void* y_bf16, int64_t ldy, const void* add_bf16,
                          int64_t ld_add, arc_stream_t stream) {
  if (!a_codes || !a_sf || !b_codes || !b_sf || !y_bf16) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || k_aug <= 0 || N % 8 || ldy < N || ldy % 8) return ARC_ERR_INVALID_ARG;
  if (add_bf16 && (ld_add < N || ld_add % 8)) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || k_aug > (1ll << 24)) return ARC_ERR_UNSUPPORTED;
  if (!al16(a_codes) || !al16(a_sf) || !al16(b_codes) || !al16(b_sf) || !al16(y_bf16) ||
      (add_bf16 && !al16(add_bf16)))
    return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  const int64_t kpad = arc_kpad(k_aug);
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.ksteps = static_cast<int>(kpad / 64);
  g.kstages = (g.ksteps + 3) / 4;
  g.katoms = static_cast<int>((kpad + 127) / 128);
  g.nblk128 = static_cast<int>((N + 127) / 128);
  g.tiles_m = static_cast<int>((M + 127) / 128);
  g.tiles_n = static_cast<int>((N + 255) / 256);
  g.box_rows_a = static_cast<int>(std::min<int64_t>(128, M));
  g.box_rows_b = static_cast<int>(std::min<int64_t>(256, N));
  g.sfa = a_sf;
  g.sfb = b_sf;
  g.y = static_cast<__nv_bfloat16*>(y_bf16);
  g.ldy = ldy;
  g.add = static_cast<const __nv_bfloat16*>(add_bf16);
  g.ld_add = ld_add;
  g.wait_ns = g_wait_ns;
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(kpad / 2),
                static_cast<uint64_t>(M), static_cast<uint64_t>(kpad / 2), 128, g.box_rows_a) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, static_cast<uint64_t>(kpad / 2),
                static_cast<uint64_t>(N), static_cast<uint64_t>(kpad / 2), 128, g.box_rows_b))
    return ARC_ERR_CUDA;
  g.inject = take_inject(1);
  return gemm_launch<arc::kGemmMX4>(ta, tb, g, sms, add_bf16 != nullptr, S(stream));
}

arc_status arc_gemm_bf16(const void* x_bf16, int64_t ldx, const void* w_bf16, int64_t ldw, int64_t M, int64_t N,
                         int64_t K, void* y_bf16, int64_t ldy, const void* add_bf16, int64_t ld_add,
                         arc_stream_t stream) {
  if (!x_bf16 || !w_bf16 || !y_bf16) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 || N % 8 || ldx < K || ldw < K || ldy < N) return ARC_ERR_INVALID_ARG;
  if (ldx % 8 || ldw % 8 || ldy % 8) return ARC_ERR_INVALID_ARG;
  if (add_bf16 && (ld_add < N || ld_add % 8)) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 24)) return ARC_ERR_UNSUPPORTED;
  if (!al16(x_bf16) || !al16(w_bf16) || !al16(y_bf16) || (add_bf16 && !al16(add_bf16))) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.kstages = static_cast<int>((K + 63) / 64);
  g.ksteps = g.kstages * 4;
  g.tiles_m = static_cast<int>((M + 127) / 128);
  g.tiles_n = static_cast<int>((N + 255) / 256);
  g.box_rows_a = static_cast<int>(std::min<int64_t>(128, M));
  g.box_rows_b = static_cast<int>(std::min<int64_t>(256, N));
  g.y = static_cast<__nv_bfloat16*>(y_bf16);
  g.ldy = ldy;
  g.add = static_cast<const __nv_bfloat16*>(add_bf16);
  g.ld_add = ld_add;
  g.wait_ns = g_wait_ns;
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x_bf16, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                static_cast<uint64_t>(ldx * 2), 64, g.box_rows_a) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_bf16, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                static_cast<uint64_t>(ldw * 2), 64, g.box_rows_b))
    return ARC_ERR_CUDA;
  g.inject = take_inject(1);
  return gemm_launch<arc::kGemmBF16>(ta, tb, g, sms, add_bf16 != nullptr, S(stream));
}

arc_status arc_quantize_fp8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const float* d_static_scale,
                            uint8_t* codes, int64_t ldc, float* d_scale_out, void* workspace, size_t ws_bytes,
                            arc_stream_t stream) {
  if (!x_bf16 || !codes || !d_scale_out) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 16 || ldx < K || ldc < K) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || K > (1ll << 24)) return ARC_ERR_UNSUPPORTED;
  if (!al16(x_bf16) || (ldx * 2) % 16 || !al16(codes) || ldc % 16) return ARC_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < arc_quantize_workspace_bytes(M, 0)) return ARC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  cudaStream_t s = S(stream);
  QuantWs w = carve_quant_ws(workspace);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x_bf16);
  int npartials = 0;
  if (!d_static_scale) {
    const int64_t items = M * ((K + arc::kAmaxSeg - 1) / arc::kAmaxSeg);
    npartials = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>({(items + 7) / 8, static_cast<int64_t>(sms) * 4, arc::kMaxPartials})));
    arc::k_amax<<<static_cast<unsigned>(npartials), 256, 0, s>>>(xb, ldx, static_cast<int>(M), static_cast<int>(K),
                                                                w.partials);
    if ((st = launch_status()) != ARC_OK) return st;
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(M, static_cast<int64_t>(sms) * 8)));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = d_static_scale ? 0 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, arc::k_quant_fp8, xb, ldx, static_cast<int>(M), static_cast<int>(K),
                                           d_static_scale, static_cast<const uint32_t*>(w.partials), npartials,
                                           d_scale_out, codes, ldc);
  return e == cudaSuccess ? ARC_OK : ARC_ERR_CUDA;
}

arc_status arc_gemm_fp8(const uint8_t* a_codes, int64_t lda, const float* d_a_scale, const uint8_t* b_codes,
                        int64_t ldb, const float* d_b_scale, int64_t M, int64_t N, int64_t K, void* y_bf16,
                        int64_t ldy, const void* add_bf16, int64_t ld_add, arc_stream_t stream) {
  if (!a_codes || !b_codes || !d_a_scale || !d_b_scale || !y_bf16) return ARC_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || K % 16 || N % 8 || lda < K || ldb < K || ldy < N || ldy % 8)
    return ARC_ERR_INVALID_ARG;
  if (add_bf16 && (ld_add < N || ld_add % 8)) return ARC_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 24)) return ARC_ERR_UNSUPPORTED;
  if (!al16(a_codes) || !al16(b_codes) || lda % 16 || ldb % 16 || !al16(y_bf16) || (add_bf16 && !al16(add_bf16)))
    return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.ksteps = static_cast<int>((K + 31) / 32);  // one MMA per 32 values; the map zero-fills past K
  g.kstages = (g.ksteps + 3) / 4;
  g.tiles_m = static_cast<int>((M + 127) / 128);
  g.tiles_n = static_cast<int>((N + 255) / 256);
  g.box_rows_a = static_cast<int>(std::min<int64_t>(128, M));
  g.box_rows_b = static_cast<int>(std::min<int64_t>(256, N));
  g.a_scale = d_a_scale;
  g.b_scale = d_b_scale;
  g.y = static_cast<__nv_bfloat16*>(y_bf16);
  g.ldy = ldy;
  g.add = static_cast<const __nv_bfloat16*>(add_bf16);
  g.ld_add = ld_add;
  g.wait_ns = g_wait_ns;
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                static_cast<uint64_t>(lda), 128, g.box_rows_a) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                static_cast<uint64_t>(ldb), 128, g.box_rows_b))
    return ARC_ERR_CUDA;
  g.inject = take_inject(1);
  return gemm_launch<arc::kGemmFP8>(ta, tb, g, sms, add_bf16 != nullptr, S(stream));
}

arc_status arc_rmsnorm_bf16(const void* h_bf16, int64_t S_, int64_t d, int64_t ldh, const void* gain_bf16, float eps,
                            void* out_bf16, int64_t ldo, arc_stream_t stream) {
  if (!h_bf16 || !gain_bf16 || !out_bf16) return ARC_ERR_INVALID_ARG;
  if (S_ <= 0 || d <= 0 || d % 8 || ldh < d || ldo < d || ldh % 8 || ldo % 8) return ARC_ERR_INVALID_ARG;
  if (!al16(h_bf16) || !al16(gain_bf16) || !al16(out_bf16)) return ARC_ERR_ALIGNMENT;
  arc_status st = device_check(nullptr);
  if (st != ARC_OK) return st;
  arc::k_rmsnorm<<<static_cast<unsigned>((S_ + 7) / 8), 256, 0, S(stream)>>>(
      static_cast<const __nv_bfloat16*>(h_bf16), ldh, static_cast<int>(S_), static_cast<int>(d),
      static_cast<const __nv_bfloat16*>(gain_bf16), static_cast<double>(eps), static_cast<__nv_bfloat16*>(out_bf16),
      ldo);
  return launch_status();
}

arc_status arc_silu_mul_bf16(const void* gu_bf16, int64_t S_, int64_t F, int64_t ld_gu, void* out_bf16, int64_t ldo,
                             arc_stream_t stream) {
  if (!gu_bf16 || !out_bf16) return ARC_ERR_INVALID_ARG;
  if (S_ <= 0 || F <= 0 || F % 8 || ld_gu < 2 * F || ldo < F || ld_gu % 8 || ldo % 8) return ARC_ERR_INVALID_ARG;
  if (!al16(gu_bf16) || !al16(out_bf16)) return ARC_ERR_ALIGNMENT;
  int sms = 0;
  arc_status st = device_check(&sms);
  if (st != ARC_OK) return st;
  const int64_t vecs = S_ * (F / 8);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((vecs + 255) / 256, static_cast<int64_t>(sms) * 16));
  arc::k_silu_mul<<<static_cast<unsigned>(blocks), 256, 0, S(stream)>>>(
      static_cast<const __nv_bfloat16*>(gu_bf16), ld_gu, static_cast<int>(S_), static_cast<int>(F),
      static_cast<__nv_bfloat16*>(out_bf16), ldo);
  return launch_status();
}

// Workspace of the recurrent driver: activation codes/scales (the larger of the NVFP4 and FP8
// quantizations), two tensor scales, gate|up output, SwiGLU output, normed hidden state,
// quantizer workspace.
static void recurrent_layout(int64_t S_, const arc_swiglu_block* blk, size_t off[7]) {
  int32_t rmax_gu = 0, rmax_d = 0;
  for (int i = 0; i < blk->n_sublayers; ++i) {
    rmax_gu = std::max(rmax_gu, blk->sublayers[i].r_gateup);
    rmax_d = std::max(rmax_d, blk->sublayers[i].r_down);
  }
  const size_t codes = std::max({arc_nvfp4_codes_bytes(S_, blk->d + rmax_gu), arc_nvfp4_codes_bytes(S_, blk->ffn + rmax_d),
                                 static_cast<size_t>(S_) * static_cast<size_t>(std::max(blk->d, blk->ffn))});
  const size_t sf = std::max(arc_nvfp4_sf_bytes(S_, blk->d + rmax_gu), arc_nvfp4_sf_bytes(S_, blk->ffn + rmax_d));
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  off[0] = 0;                                                       // codes
  off[1] = off[0] + a256(codes);                                    // sf
  off[2] = off[1] + a256(sf);                                       // 2 scales
  off[3] = off[2] + 256;                                            // gate|up [S, 2F]
  off[4] = off[3] + a256(static_cast<size_t>(S_) * 2 * blk->ffn * 2);  // act [S, F]
  off[5] = off[4] + a256(static_cast<size_t>(S_) * blk->ffn * 2);      // normed [S, d]
  off[6] = off[5] + a256(static_cast<size_t>(S_) * blk->d * 2);        // quant workspace
}

size_t arc_recurrent_workspace_bytes(int64_t S_, const arc_swiglu_block* blk) {
  if (!blk || S_ <= 0 || blk->n_sublayers <= 0 || !blk->sublayers) return 0;
  size_t off[7];
  recurrent_layout(S_, blk, off);
  int32_t rmax = 0;
  for (int i = 0; i < blk->n_sublayers; ++i)
    rmax = std::max(rmax, std::max(blk->sublayers[i].r_gateup, blk->sublayers[i].r_down));
  return off[6] + arc_quantize_workspace_bytes(S_, rmax);
}

// h = bf16(beta * h + e), the damped residual (with input injection) of a contractive block.
static arc_status damp_bf16(void* h, int64_t S_, int64_t d, float beta, const void* e, arc_stream_t stream, int sms) {
  const int64_t vecs = S_ * (d / 8);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((vecs + 255) / 256, static_cast<int64_t>(sms) * 8));
  arc::k_damp_bf16<<<static_cast<unsigned>(blocks), 256, 0, S(stream)>>>(
      static_cast<__nv_bfloat16*>(h), d, static_cast<int>(S_), static_cast<int>(d), beta,
      static_cast<const __nv_bfloat16*>(e));
  return launch_status();
}

// The recurrence with a per-step format: step t runs as fmt(t) (ARC_STEP_BF16, ARC_STEP_NVFP4 or
// ARC_STEP_FP8).
extern "C++" {
template <class Fmt>
arc_status recurrent_run(void* h_bf16, int64_t S_, const arc_swiglu_block* blk, int32_t T, Fmt fmt,
                         void* workspace, size_t ws_bytes, arc_stream_t stream) {
  if (!h_bf16 || !blk || !blk->sublayers || blk->n_sublayers <= 0 || S_ <= 0 || T < 0) return ARC_ERR_INVALID_ARG;
  const int64_t d = blk->d, F = blk->ffn;
  if (d <= 0 || F <= 0 || d % 16 || F % 16) return ARC_ERR_INVALID_ARG;
  const float beta = blk->residual_scale == 0.0f ? 1.0f : blk->residual_scale;
  if (!(beta > 0.0f && beta <= 1.0f)) return ARC_ERR_INVALID_ARG;
  for (int32_t t = 0; t < T; ++t) {
    const int f = fmt(t);
    if (f != ARC_STEP_BF16 && f != ARC_STEP_NVFP4 && f != ARC_STEP_FP8) return ARC_ERR_INVALID_ARG;
    if (f == ARC_STEP_FP8)
      for (int i = 0; i < blk->n_sublayers; ++i) {
        const arc_swiglu_sublayer& L = blk->sublayers[i];
        if (!L.gateup_fp8 || !L.gateup_fp8_scale || !L.down_fp8 || !L.down_fp8_scale) return ARC_ERR_INVALID_ARG;
      }
  }
  const void* inj = blk->inject_bf16;
  if (inj && (reinterpret_cast<uintptr_t>(inj) & 15u)) return ARC_ERR_ALIGNMENT;
  const bool damp = beta != 1.0f || inj != nullptr;
  int sms = 0;
  if (damp) {
    const arc_status dc = device_check(&sms);
    if (dc != ARC_OK) return dc;
  }
  const size_t need = arc_recurrent_workspace_bytes(S_, blk);
  if (!workspace || ws_bytes < need) return ARC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ARC_ERR_ALIGNMENT;
  size_t off[7];
  recurrent_layout(S_, blk, off);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* codes = ws + off[0];
  uint8_t* sf = ws + off[1];
  float* sA = reinterpret_cast<float*>(ws + off[2]);
  void* gu = ws + off[3];
  void* act = ws + off[4];
  void* nrm = ws + off[5];
  void* qws = ws + off[6];
  const size_t qws_bytes = ws_bytes - off[6];
  arc_status st;
  for (int32_t t = 0; t < T; ++t) {
    const int f = fmt(t);
    for (int i = 0; i < blk->n_sublayers; ++i) {
      const arc_swiglu_sublayer& L = blk->sublayers[i];
      if (f == ARC_STEP_NVFP4) {
        if ((st = arc_quantize_act_nvfp4(h_bf16, S_, d, d, L.idx_gateup, L.r_gateup, L.rms_gain_bf16, blk->eps,
                                         nullptr, codes, sf, sA, qws, qws_bytes, stream)) != ARC_OK)
          return st;
        if ((st = arc_gemm_nvfp4(codes, sf, sA, L.gateup_codes, L.gateup_sf, L.gateup_scale, S_, 2 * F,
                                 d + L.r_gateup, gu, 2 * F, nullptr, 0, stream)) != ARC_OK)
          return st;
        if ((st = arc_silu_mul_bf16(gu, S_, F, 2 * F, act, F, stream)) != ARC_OK) return st;
        if ((st = arc_quantize_act_nvfp4(act, S_, F, F, L.idx_down, L.r_down, nullptr, 0.0f, nullptr, codes, sf,
                                         sA + 1, qws, qws_bytes, stream)) != ARC_OK)
          return st;
        if (damp && (st = damp_bf16(h_bf16, S_, d, beta, inj, stream, sms)) != ARC_OK) return st;
        if ((st = arc_gemm_nvfp4(codes, sf, sA + 1, L.down_codes, L.down_sf, L.down_scale, S_, d, F + L.r_down,
                                 h_bf16, d, h_bf16, d, stream)) != ARC_OK)
          return st;
      } else if (f == ARC_STEP_FP8) {
        if ((st = arc_rmsnorm_bf16(h_bf16, S_, d, d, L.rms_gain_bf16, blk->eps, nrm, d, stream)) != ARC_OK) return st;
        if ((st = arc_quantize_fp8(nrm, S_, d, d, nullptr, codes, d, sA, qws, qws_bytes, stream)) != ARC_OK) return st;
        if ((st = arc_gemm_fp8(codes, d, sA, L.gateup_fp8, d, L.gateup_fp8_scale, S_, 2 * F, d, gu, 2 * F, nullptr, 0,
                               stream)) != ARC_OK)
          return st;
        if ((st = arc_silu_mul_bf16(gu, S_, F, 2 * F, act, F, stream)) != ARC_OK) return st;
        if ((st = arc_quantize_fp8(act, S_, F, F, nullptr, codes, F, sA + 1, qws, qws_bytes, stream)) != ARC_OK)
          return st;
        if (damp && (st = damp_bf16(h_bf16, S_, d, beta, inj, stream, sms)) != ARC_OK) return st;
        if ((st = arc_gemm_fp8(codes, F, sA + 1, L.down_fp8, F, L.down_fp8_scale, S_, d, F, h_bf16, d, h_bf16, d,
                               stream)) != ARC_OK)
          return st;
      } else {
        if ((st = arc_rmsnorm_bf16(h_bf16, S_, d, d, L.rms_gain_bf16, blk->eps, nrm, d, stream)) != ARC_OK) return st;
        if ((st = arc_gemm_bf16(nrm, d, L.w_gateup_bf16, d, S_, 2 * F, d, gu, 2 * F, nullptr, 0, stream)) != ARC_OK)
          return st;
        if ((st = arc_silu_mul_bf16(gu, S_, F, 2 * F, act, F, stream)) != ARC_OK) return st;
        if (damp && (st = damp_bf16(h_bf16, S_, d, beta, inj, stream, sms)) != ARC_OK) return st;
        if ((st = arc_gemm_bf16(act, F, L.w_down_bf16, F, S_, d, F, h_bf16, d, h_bf16, d, stream)) != ARC_OK)
          return st;
      }
    }
  }
  return ARC_OK;
}
}  // extern "C++"

arc_status arc_recurrent_prefill(void* h_bf16, int64_t S_, const arc_swiglu_block* blk, int32_t T, int32_t k_low,
                                 void* workspace, size_t ws_bytes, arc_stream_t stream) {
  if (k_low < 0) return ARC_ERR_INVALID_ARG;
  return recurrent_run(h_bf16, S_, blk, T, [k_low](int32_t t) { return t < k_low ? ARC_STEP_NVFP4 : ARC_STEP_BF16; },
                       workspace, ws_bytes, stream);
}

arc_status arc_recurrent_prefill_schedule(void* h_bf16, int64_t S_, const arc_swiglu_block* blk, int32_t T,
                                          const uint8_t* low_steps, void* workspace, size_t ws_bytes,
                                          arc_stream_t stream) {
  if (T > 0 && !low_steps) return ARC_ERR_INVALID_ARG;
  return recurrent_run(h_bf16, S_, blk, T, [low_steps](int32_t t) { return static_cast<int>(low_steps[t]); },
                       workspace, ws_bytes, stream);
}

arc_status arc_last_device_status(arc_stream_t stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return ARC_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, arc::g_status, sizeof(int)) != cudaSuccess) return ARC_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(arc::g_status, &zero, sizeof(int)) != cudaSuccess) return ARC_ERR_CUDA;
  }
  return static_cast<arc_status>(v);
}

arc_status arc_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return ARC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_wait_ns = ns;
  return ARC_OK;
}

}  // extern "C"

// Temporary space of arc_quantize_act_nvfp4_static_scratch: one fixed array per device, for
// callers that cannot allocate. Host code only ever passes the address that
// cudaGetSymbolAddress returns for the current device, looked up once per device.
static __device__ __align__(256) uint8_t g_static_scratch[ARC_STATIC_SCRATCH_BYTES];

namespace {
arc_status static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARC_ERR_CUDA;
  static void* addr[64] = {};
  std::lock_guard<std::mutex> lk(g_mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return ARC_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return ARC_OK;
}
}  // namespace

extern "C" {

arc_status arc_quantize_act_nvfp4_static_scratch(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                                 const int32_t* d_idx, int32_t r, const void* rms_gain_bf16,
                                                 float rms_eps, const float* d_static_scale, uint8_t* codes,
                                                 uint8_t* sf, float* d_scale_out, arc_stream_t stream) {
  // argument errors first, in the order of the workspace entry point, then the array's limit
  arc_status st = quantize_check(x_bf16, M, K, ldx, d_idx, r, rms_gain_bf16, codes, sf, d_scale_out, nullptr);
  if (st != ARC_OK) return st;
  if (arc_quantize_workspace_bytes(M, r) > static_cast<size_t>(ARC_STATIC_SCRATCH_BYTES)) return ARC_ERR_WORKSPACE;
  void* ws = nullptr;
  st = static_scratch_address(&ws);
  if (st != ARC_OK) return st;
  return quantize_common(x_bf16, M, K, ldx, d_idx, r, rms_gain_bf16, rms_eps, d_static_scale, codes, sf,
                         d_scale_out, ws, ARC_STATIC_SCRATCH_BYTES, stream, 0);
}

arc_status arc_debug_inject(int32_t kind) {
  if (kind < 0 || kind > 2) return ARC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_inject = kind;
  return ARC_OK;
}

}  // extern "C"
