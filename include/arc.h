/*
 * arc.h -- C ABI of the B200 (sm_100a) NVFP4 + augmented-residual-channel (ARC) library.
 *
 * The method (sources by page title and section):
 *   "ARCQuant: Boosting NVFP4 Quantization with Augmented Residual Channels for LLMs"
 *     (Technische Samenvatting, Methodologie): NVFP4 blocks of 16 E2M1 values; outlier channels
 *     identified offline by calibration abs-max (optionally all channels reordered by it before
 *     the primary stage); primary block-wise quantization; the residual
 *     x - dequant(Q(x)) of the outlier channels quantized again as a second set of NVFP4
 *     channels and appended along K; the matching weight columns duplicated; one unified GEMM
 *     of depth K + r whose linear accumulation adds the correction; one fused kernel for
 *     RMSNorm + primary + residual quantization writing a GEMM-ready layout.
 *   "Day 0 LLM Inference Support: Hierarchical Quantization and Memory Access Optimization
 *     Practices" (section V): scale = amax / FMT_MAX with an all-zero guard, clipping to the
 *     format range, scale factors laid out for vectorised loads, quantization fused into the
 *     producing operator, block-scaled tensor-core instructions consuming the scales directly.
 *   "RAMP: Recurrent Adaptive Mixed Precision for Efficient Prefill in Recurrent-Depth
 *     Language Models" (sections 2.1, 4.1, 4.2): a shared block applied T times; low-precision
 *     weight-and-activation steps before step k_low (or on any schedule of steps),
 *     reference-precision (BF16) steps after; hidden state kept in BF16; FP8 weights and
 *     activations as the pages' own low-precision format.
 *
 * Number formats (the pages name E2M1 and block size 16; the rest is this library's reading):
 *   element   E2M1 code, 4 bits, magnitudes {0,.5,1,1.5,2,3,4,6}, bit 3 = sign
 *   block     16 consecutive K-elements share one unsigned E4M3 scale byte (bias 7, max 448)
 *   tensor    one fp32 tensor scale s = amax / 2688 (2688 = 6 * 448; amax == 0 gives s = 1)
 *   decode    value = E2M1(code) * E4M3(sf) * s
 *   encode    sf = E4M3_rne_sat((amax_block / 6) / s); d = E4M3(sf) * s;
 *             code = E2M1_rne_sat(x / d) with the sign of x kept, or 0 when d == 0
 *             (every operation fp32 round-to-nearest-even, no fused multiply-add)
 *
 * Layouts:
 *   K_aug = K + r, K_pad = K_aug rounded up to a multiple of 64.
 *   codes  [rows, K_pad/2] bytes, row-major; element k of a row is byte k/2, low nibble for
 *          even k. Columns K..K+r-1 hold the r appended channels, K+r..K_pad-1 are zero.
 *   sf     scale bytes in 512-byte atoms of 128 rows x 4 scales: the atom of rows 128i..
 *          and scale columns 4j.. sits at byte (i * (K_pad/64) + j) * 512; inside it, row m
 *          and scale column kb are at (m%32)*16 + ((m/32)%4)*4 + kb%4. Rows are padded to a
 *          multiple of 128 with zero bytes. This is the order the tensor cores read scale
 *          factors in, so one 512-byte atom feeds one K=64 step of a 128-row tile.
 *   bf16   row-major with an explicit leading dimension (elements); rows 16-byte aligned.
 *
 * Conventions:
 *   - The caller owns every buffer (device memory unless a parameter says "host"). The library
 *     allocates no device memory. Temporary space is the caller's `workspace`, sized by the
 *     matching *_workspace_bytes query.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream) and returns at once.
 *     Per-tensor scales stay in device memory, so no call synchronises with the host.
 *   - Errors that the host can see are returned before any launch: NULL pointers, sizes,
 *     K % 16 != 0, r % 16 != 0, r > K, leading dimensions, pointer alignment (16 bytes), a
 *     workspace that is too small, a device that is not sm_100.
 *   - Errors on the device (a pipeline wait that ran out, a device-side check) set a status
 *     word that arc_last_device_status() reads.
 *   - idx must hold r distinct channels in [0, K) (checked by the calibration routine that
 *     produces it, not on every call). Inputs are assumed finite: NaN/Inf give unspecified
 *     codes.
 */
#ifndef ARC_H_
#define ARC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* arc_stream_t;

typedef enum {
  ARC_OK = 0,
  ARC_ERR_INVALID_ARG = 1,  /* NULL pointer, bad size or leading dimension */
  ARC_ERR_ALIGNMENT = 2,    /* a pointer or row pitch is not 16-byte aligned */
  ARC_ERR_UNSUPPORTED = 3,  /* device is not sm_100, or a shape outside the supported range */
  ARC_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, tensor-map encoding) */
  ARC_ERR_TIMEOUT = 5,      /* a bounded pipeline wait on the device ran out */
  ARC_ERR_WORKSPACE = 6     /* workspace NULL or smaller than the size query returned */
} arc_status;

/* Human-readable name of a status code (static string). */
const char* arc_status_str(arc_status s);

/* ----------------------------------------------------------------------------------------- */
/* Size queries (host, pure functions)                                                        */
/* ----------------------------------------------------------------------------------------- */

/* K_aug rounded up to a multiple of 64. */
int64_t arc_kpad(int64_t k_aug);
/* Bytes of the packed E2M1 codes for `rows` rows of K_aug channels: rows * K_pad / 2. */
size_t arc_nvfp4_codes_bytes(int64_t rows, int64_t k_aug);
/* Bytes of the swizzled scale bytes: ceil(rows/128) * (K_pad/64) * 512. */
size_t arc_nvfp4_sf_bytes(int64_t rows, int64_t k_aug);
/* Workspace of arc_quantize_act_nvfp4 / arc_pack_weight_nvfp4 for `rows` rows and r channels:
 * 8 KiB of per-CTA abs-max partials plus 8 bytes per row (RMSNorm statistics). */
size_t arc_quantize_workspace_bytes(int64_t rows, int32_t r);
/* Workspace of arc_calibrate_outliers for K channels. */
size_t arc_calibrate_workspace_bytes(int64_t K);

/* ----------------------------------------------------------------------------------------- */
/* Quantization ("ARCQuant", Dual-Stage Quantisatie and Kernel Implementatie)                  */
/* ----------------------------------------------------------------------------------------- */

/*
 * Quantize bf16 activations X [M, K] (leading dimension ldx elements) to NVFP4 and append the
 * r residual channels: for j < r and c = d_idx[j], R[m, j] = x[m, c] - E2M1(q) * d_block(c)
 * (fp32), quantized in blocks of 16 (in idx order) with the same tensor scale and written at
 * columns K + j.
 *   d_idx           device int32[r]; may be NULL when r == 0.
 *   rms_gain_bf16   device bf16[K] or NULL. Non-NULL fuses an RMSNorm prologue: x is replaced
 *                   by bf16((h * inv) * g) with inv = 1/sqrt(sum(h^2)/K + eps) in double and the
 *                   sum of squares exact (order-independent).
 *   d_static_scale  device fp32 scalar, or NULL for a dynamic scale s = amax(|x|)/2688 taken
 *                   over the whole tensor (an extra read pass over X).
 *   codes, sf       outputs, arc_nvfp4_codes_bytes(M, K+r) / arc_nvfp4_sf_bytes(M, K+r) bytes,
 *                   16-byte aligned.
 *   d_scale_out     device fp32 scalar receiving the tensor scale used (may equal d_static_scale).
 *   workspace       device scratch of arc_quantize_workspace_bytes(M, r) bytes, 256-byte aligned;
 *                   contents need not be initialised; calls sharing a workspace must be ordered.
 * Requires K % 16 == 0, r % 16 == 0, 0 <= r <= K, ldx >= K, x rows 16-byte aligned. The
 * residuals are staged in shared memory (56 bytes per outlier channel plus K/8 bytes of block
 * table, at most 200 KB), which accepts r <= 3504 for any K <= 65536 and r <= 1312 up to
 * K = 2^20; larger requests return ARC_ERR_UNSUPPORTED.
 */
arc_status arc_quantize_act_nvfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const int32_t* d_idx,
                                  int32_t r, const void* rms_gain_bf16, float rms_eps, const float* d_static_scale,
                                  uint8_t* codes, uint8_t* sf, float* d_scale_out, void* workspace, size_t ws_bytes,
                                  arc_stream_t stream);

/*
 * Pack weights W [N, K] (nn.Linear layout, Y = X W^T) as the augmented W_aug = [W | W[:, idx]]
 * ("de bijbehorende gewichten gedupliceerd"): the r duplicated columns are quantized as ordinary
 * NVFP4 blocks of W_aug, with one tensor scale s_W = amax(|W|)/2688 written to d_scale_out.
 * Same layouts, requirements and workspace as arc_quantize_act_nvfp4 (rows = N).
 */
arc_status arc_pack_weight_nvfp4(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, const int32_t* d_idx,
                                 int32_t r, uint8_t* codes, uint8_t* sf, float* d_scale_out, void* workspace,
                                 size_t ws_bytes, arc_stream_t stream);

/*
 * Offline outlier identification ("Adaptieve Uitschieter-identificatie"): the r channels of the
 * calibration tensor X [M, K] with the largest abs-max, in descending order, ties by ascending
 * index, written to d_idx_out (device int32[r]). 0 < r <= K, r <= 1024, K even, ldx even and x
 * 4-byte aligned (else ARC_ERR_INVALID_ARG / ARC_ERR_ALIGNMENT); workspace of at least
 * arc_calibrate_workspace_bytes(K), 256-byte aligned (else ARC_ERR_WORKSPACE / ARC_ERR_ALIGNMENT).
 */
arc_status arc_calibrate_outliers(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int32_t r,
                                  int32_t* d_idx_out, void* workspace, size_t ws_bytes, arc_stream_t stream);

/*
 * Channel reorder ("Adaptieve Uitschieter-identificatie": the channels are reordered by their
 * absolute maxima and a top-S subset is selected): all K channels of the calibration tensor
 * X [M, K] in descending abs-max order, ties by ascending index, written to d_perm_out (device
 * int32[K]); its first r entries are what arc_calibrate_outliers returns for r. Workspace as
 * arc_calibrate_outliers. The ranking does O(K^2) comparisons on the device (a calibration
 * step, run once per model). 0 < K <= 2^20, K even, x 4-byte aligned.
 */
arc_status arc_calibrate_order(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int32_t* d_perm_out,
                               void* workspace, size_t ws_bytes, arc_stream_t stream);

/*
 * Reordered dual-stage quantization ("Primaire Fase: de input-activatiematrix wordt geherordend
 * en gekwantiseerd"; Kernel Implementatie: reordering, RMSNorm, primary and residual
 * quantization in one kernel). Primary channel p of the output is input channel d_perm[p]; the
 * r outlier channels are d_perm[0 .. r), so appended block j (columns K + 16 j ..) holds the
 * residuals x - E2M1(code) * d of primary block j's channels, coded with the same tensor scale.
 * The result equals arc_quantize_act_nvfp4 applied to X[:, perm] with idx = 0 .. r-1.
 *   d_perm          device int32[K], a permutation of 0 .. K-1, 16-byte aligned (entries outside
 *                   [0, K) are read as channel K-1; a repeated entry repeats that channel).
 * Other arguments, layouts and workspace as arc_quantize_act_nvfp4 (the RMSNorm gain is indexed
 * by input channel). Each row is staged in shared memory twice over: K <= 51200, else
 * ARC_ERR_UNSUPPORTED.
 */
arc_status arc_quantize_act_nvfp4_reordered(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                            const int32_t* d_perm, int32_t r, const void* rms_gain_bf16,
                                            float rms_eps, const float* d_static_scale, uint8_t* codes, uint8_t* sf,
                                            float* d_scale_out, void* workspace, size_t ws_bytes,
                                            arc_stream_t stream);

/*
 * Weights of the reordered augmented GEMM: W_aug = [W[:, perm] | W[:, perm[0 .. r)]] packed as
 * NVFP4 with one tensor scale s_W = amax(|W|)/2688; the appended blocks repeat primary blocks
 * 0 .. r/16 - 1. Same requirements as arc_quantize_act_nvfp4_reordered (rows = N).
 */
arc_status arc_pack_weight_nvfp4_reordered(const void* w_bf16, int64_t N, int64_t K, int64_t ldw,
                                           const int32_t* d_perm, int32_t r, uint8_t* codes, uint8_t* sf,
                                           float* d_scale_out, void* workspace, size_t ws_bytes,
                                           arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* GEMMs ("Unified GEMM Executie"; RAMP's BF16 reference path)                                 */
/* ----------------------------------------------------------------------------------------- */

/*
 * Y [M, N] bf16 = bf16_rn( (s_A * s_B) * sum_{k < K_pad} E2M1(a)*sfA * E2M1(b)*sfB )
 *                 [ + add, as bf16_rn(fp32(alpha*acc) + fp32(add)) ]
 * One block-scaled tcgen05 GEMM of depth K_aug over NVFP4 operands laid out as above (A from
 * arc_quantize_act_nvfp4, B from arc_pack_weight_nvfp4 with the same idx), fp32 accumulation
 * in tensor memory.
 *   d_a_scale, d_b_scale   device fp32 tensor scales.
 *   add_bf16               NULL, or [M, N] bf16 with leading dimension ld_add; may alias y.
 * Requires N % 8 == 0, ldy % 8 == 0, ld_add % 8 == 0, 16-byte aligned pointers.
 */
arc_status arc_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sf, const float* d_a_scale,
                          const uint8_t* b_codes, const uint8_t* b_sf, const float* d_b_scale, int64_t M, int64_t N,
                          int64_t k_aug, void* y_bf16, int64_t ldy, const void* add_bf16, int64_t ld_add,
                          arc_stream_t stream);

/*
 * BF16 switch: Y [M, N] = bf16_rn(X W^T [+ add]) with X [M, K], W [N, K] bf16 and fp32
 * accumulation (tcgen05 kind::f16). Requires K % 8 == 0, N % 8 == 0, leading dimensions
 * multiples of 8, 16-byte aligned pointers. add may alias y.
 */
arc_status arc_gemm_bf16(const void* x_bf16, int64_t ldx, const void* w_bf16, int64_t ldw, int64_t M, int64_t N,
                         int64_t K, void* y_bf16, int64_t ldy, const void* add_bf16, int64_t ld_add,
                         arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* FP8 W8A8 ("RAMP…" §4.1: the low-precision steps run with FP8 weights and activations)        */
/* ----------------------------------------------------------------------------------------- */

/*
 * Quantize X [M, K] bf16 (leading dimension ldx) to E4M3 codes [M, K] (leading dimension ldc
 * bytes) with one per-tensor scale: s = amax(|x|)/448 (1 for an all-zero tensor), or
 * *d_static_scale; code = signed E4M3 of the correctly rounded fp32 quotient x / s (ties to
 * even, saturating at 448, the sign kept on a quotient that rounds to zero). The scale used is
 * written to d_scale_out. Workspace: arc_quantize_workspace_bytes(M, 0) bytes, 256-byte aligned.
 * Requires K % 16 == 0, ldx >= K with rows 16-byte aligned, ldc >= K, ldc % 16 == 0.
 */
arc_status arc_quantize_fp8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const float* d_static_scale,
                            uint8_t* codes, int64_t ldc, float* d_scale_out, void* workspace, size_t ws_bytes,
                            arc_stream_t stream);

/*
 * Y [M, N] bf16 = bf16_rn( (s_A * s_B) * sum_k E4M3(a) E4M3(b) [+ add] ) with A [M, K] and
 * B [N, K] E4M3 codes (leading dimensions lda, ldb bytes), fp32 tensor-core accumulation
 * (tcgen05 kind::f8f6f4). Requires K % 16 == 0, lda, ldb multiples of 16, N % 8 == 0,
 * ldy % 8 == 0, 16-byte aligned pointers; add may alias y.
 */
arc_status arc_gemm_fp8(const uint8_t* a_codes, int64_t lda, const float* d_a_scale, const uint8_t* b_codes,
                        int64_t ldb, const float* d_b_scale, int64_t M, int64_t N, int64_t K, void* y_bf16,
                        int64_t ldy, const void* add_bf16, int64_t ld_add, arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* MXFP4 with augmented residual channels ("ARCQuant", Resultaten / Generaliseerbaarheid: the    */
/* approach extends to MXFP4)                                                                   */
/* ----------------------------------------------------------------------------------------- */
/*
 * Format (this library's reading, the OCP microscaling MXFP4): 32 consecutive K-elements share
 * one power-of-two scale X = 2^(floor(log2 amax) - 2) stored as an E8M0 byte (exponent + 127,
 * clamped to [0, 254]; 0 for an all-zero block); elements are E2M1_rne_sat(x / X) with the sign
 * of x kept (zero codes for an all-zero block). No tensor scale.
 * Layouts: codes as for NVFP4, [rows, K_pad/2] with K_pad = K + r rounded up to 64. Scale bytes
 * in 512-byte atoms of 128 rows x 4 scales (128 K-elements): the atom of rows 128i.. and scale
 * columns 4j.. at byte (i * ceil(K_pad/128) + j) * 512, row m / column kb inside at
 * (m%32)*16 + ((m/32)%4)*4 + kb%4; padding rows and columns are zero.
 */

/* Bytes of the MXFP4 scale layout: ceil(rows/128) * ceil(K_pad/128) * 512. */
size_t arc_mxfp4_sf_bytes(int64_t rows, int64_t k_aug);

/*
 * Quantize bf16 X [M, K] to MXFP4 and append r residual channels: for j < r and c = d_idx[j],
 * R[m, j] = x[m, c] - E2M1(code) * X_block(c) (exact product, fp32 subtract), coded in blocks of
 * 32 in idx order at columns K + j. One kernel, one read of X, no workspace.
 * Requires K % 32 == 0, r % 32 == 0, 0 <= r <= K, ldx >= K, 16-byte aligned rows and outputs.
 * Per warp the kernel keeps K/32 + 4r bytes of shared memory (at most 200 KB in all): larger
 * requests return ARC_ERR_UNSUPPORTED.
 */
arc_status arc_quantize_act_mxfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const int32_t* d_idx,
                                  int32_t r, uint8_t* codes, uint8_t* sf, arc_stream_t stream);

/* Weights W [N, K] as W_aug = [W | W[:, idx]] in MXFP4 (the r duplicated channels re-blocked
 * among themselves in blocks of 32). Requirements as arc_quantize_act_mxfp4. */
arc_status arc_pack_weight_mxfp4(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, const int32_t* d_idx,
                                 int32_t r, uint8_t* codes, uint8_t* sf, arc_stream_t stream);

/*
 * Y [M, N] bf16 = bf16_rn( sum_{k < K_pad} E2M1(a) X_A * E2M1(b) X_B ) [ + add ] over MXFP4
 * operands of depth K_aug (tcgen05 kind::mxf4nvf4 with scale_vec::2X and UE8M0 scales, fp32
 * accumulation in tensor memory). Requirements as arc_gemm_nvfp4.
 */
arc_status arc_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes, const uint8_t* b_sf,
                          int64_t M, int64_t N, int64_t k_aug, void* y_bf16, int64_t ldy, const void* add_bf16,
                          int64_t ld_add, arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* Elementwise pieces of the recurrent SwiGLU block                                            */
/* ----------------------------------------------------------------------------------------- */

/* out [S, d] = RMSNorm(h) * gain, with the same arithmetic as the fused prologue above. */
arc_status arc_rmsnorm_bf16(const void* h_bf16, int64_t S, int64_t d, int64_t ldh, const void* gain_bf16,
                            float eps, void* out_bf16, int64_t ldo, arc_stream_t stream);

/* out [S, F] = bf16( silu(g) * u ), g = gu[:, :F], u = gu[:, F:2F], silu in fp32. */
arc_status arc_silu_mul_bf16(const void* gu_bf16, int64_t S, int64_t F, int64_t ld_gu, void* out_bf16,
                             int64_t ldo, arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* Recurrent-depth prefill with a RAMP precision schedule                                     */
/* ----------------------------------------------------------------------------------------- */

/*
 * One pre-norm SwiGLU residual sublayer: h <- beta h + e + W_down (silu(W_g n) * (W_u n)),
 * n = RMSNorm(h)*g, beta and e = the block's residual_scale and inject_bf16 (1 and none for the
 * plain block); beta h + e is rounded to bf16 before the down projection adds to it. All pointers are device pointers. The
 * NVFP4 fields are the arc_pack_weight_nvfp4 outputs of the same weights augmented with
 * idx_gateup (channels of n, in [0, d)) and idx_down (channels of the SwiGLU output, in
 * [0, ffn)). The FP8 fields are the arc_quantize_fp8 outputs of the same weights (codes with row
 * strides d and ffn bytes, and their tensor scales); they are read only by FP8 steps and may be
 * NULL when no step runs in FP8.
 */
typedef struct {
  const void* rms_gain_bf16;  /* [d] */
  const void* w_gateup_bf16;  /* [2*ffn, d]: gate rows 0..ffn-1, up rows ffn..2ffn-1 */
  const void* w_down_bf16;    /* [d, ffn] */
  const uint8_t* gateup_codes;
  const uint8_t* gateup_sf;
  const float* gateup_scale;
  const uint8_t* down_codes;
  const uint8_t* down_sf;
  const float* down_scale;
  const int32_t* idx_gateup;
  int32_t r_gateup;
  const int32_t* idx_down;
  int32_t r_down;
  const uint8_t* gateup_fp8;      /* [2*ffn, d] E4M3 */
  const float* gateup_fp8_scale;
  const uint8_t* down_fp8;        /* [d, ffn] E4M3 */
  const float* down_fp8_scale;
} arc_swiglu_sublayer;

typedef struct {
  int64_t d;      /* hidden size */
  int64_t ffn;    /* SwiGLU width */
  float eps;      /* RMSNorm epsilon */
  int32_t n_sublayers;
  const arc_swiglu_sublayer* sublayers; /* host array of n_sublayers entries */
  float residual_scale; /* beta in (0, 1] of the damped residual h <- beta h + e + F(h); 0 or 1 is
                           the plain residual block */
  const void* inject_bf16; /* e: device bf16 [S, d] (row stride d) added to the damped residual of
                              every sublayer, or NULL. With beta < 1 and a small F the step map
                              contracts towards a fixed point that e keeps away from zero: the
                              regime of RAMP's error analysis (section 3, local contraction of a
                              recurrence that re-reads its input at every step). */
} arc_swiglu_block;

/* Workspace of arc_recurrent_prefill for S tokens. */
size_t arc_recurrent_workspace_bytes(int64_t S, const arc_swiglu_block* blk);

/*
 * Apply the shared block T times to h [S, d] bf16 (in place, leading dimension d): steps
 * t < k_low run every linear layer in NVFP4 + ARC (fused RMSNorm+quantize, block-scaled GEMM,
 * SwiGLU, quantize, block-scaled GEMM with the residual add in its epilogue); steps t >= k_low
 * run the same sublayers in BF16. k_low = 0 is all-BF16, k_low = T all-NVFP4. Asynchronous;
 * no host synchronisation inside the loop.
 */
arc_status arc_recurrent_prefill(void* h_bf16, int64_t S, const arc_swiglu_block* blk, int32_t T, int32_t k_low,
                                 void* workspace, size_t ws_bytes, arc_stream_t stream);

/*
 * The same recurrence with any per-step precision schedule (for schedule studies: RAMP's
 * matched-budget comparison of where the BF16 steps go, "RAMP…" §6 and its Early-BF16 and
 * random-schedule baselines; and RAMP's own FP8-BF16 instantiation, §4.2): low_steps is a host
 * array of T bytes, read during the call, one format per step:
 *   ARC_STEP_BF16 (0)   BF16 (RMSNorm, BF16 GEMMs);
 *   ARC_STEP_NVFP4 (1)  NVFP4 + ARC (as arc_recurrent_prefill's steps before k_low);
 *   ARC_STEP_FP8 (2)    FP8 W8A8 with per-tensor scales: RMSNorm, arc_quantize_fp8 (dynamic
 *                       scale), arc_gemm_fp8 with the sublayer's FP8 weights, SwiGLU,
 *                       arc_quantize_fp8, arc_gemm_fp8 with the residual add.
 * Any other value, or an FP8 step with NULL FP8 weights, returns ARC_ERR_INVALID_ARG before any
 * launch. arc_recurrent_prefill with k_low is the schedule low_steps[t] = (t < k_low).
 */
#define ARC_STEP_BF16 0
#define ARC_STEP_NVFP4 1
#define ARC_STEP_FP8 2
arc_status arc_recurrent_prefill_schedule(void* h_bf16, int64_t S, const arc_swiglu_block* blk, int32_t T,
                                          const uint8_t* low_steps, void* workspace, size_t ws_bytes,
                                          arc_stream_t stream);

/* ----------------------------------------------------------------------------------------- */
/* Device status and failure detection                                                        */
/* ----------------------------------------------------------------------------------------- */

/*
 * Synchronise `stream`, then return and clear the device status word of the current device:
 * ARC_OK, ARC_ERR_TIMEOUT (a bounded wait in a pipelined kernel ran out; the kernel stopped
 * cleanly and released its tensor memory) or ARC_ERR_CUDA (a CUDA error is pending).
 */
arc_status arc_last_device_status(arc_stream_t stream);

/* Upper bound, in nanoseconds, of every pipeline wait in the GEMM kernels (default 2 s). */
arc_status arc_set_wait_limit_ns(uint64_t ns);

/*
 * Failure-injection switch for tests (0 = off). 1: the next arc_gemm_* launch withholds its
 * first operand load, so its consumer's bounded wait must run out and report ARC_ERR_TIMEOUT.
 * 2: the next reordered quantization (arc_quantize_act_nvfp4_reordered or
 * arc_pack_weight_nvfp4_reordered) withholds the first row copy of its first CTA, with the same
 * outcome. The switch resets itself after the launch it applies to.
 */
arc_status arc_debug_inject(int32_t kind);

/* ----------------------------------------------------------------------------------------- */
/* Quantization without a workspace argument                                                  */
/* ----------------------------------------------------------------------------------------- */

/* Bytes of the fixed device array the call below uses (about 4.5 MiB). */
#define ARC_STATIC_SCRATCH_BYTES 4726784

/*
 * The pages have no counterpart of this call: it changes where temporary memory comes from, not
 * what is computed. It is for callers that cannot call cudaMalloc (or any allocator) while they
 * run: a process that reserves all the device memory it will ever use when it starts and forbids
 * allocation afterwards, or a plug-in hosted by a framework that owns the GPU's memory pool and
 * gives its plug-ins no way to borrow from it. Such a caller cannot provide the workspace that
 * arc_quantize_act_nvfp4 asks for.
 *
 * Same computation, arguments and outputs as arc_quantize_act_nvfp4 without `workspace` and
 * `ws_bytes`; the call allocates nothing. Its temporary space is one array of
 * ARC_STATIC_SCRATCH_BYTES bytes of device memory compiled into this library, so every GPU that
 * loads the library holds that array until the process exits.
 *   Limit: arc_quantize_workspace_bytes(M, r) <= ARC_STATIC_SCRATCH_BYTES, that is 8 KiB plus
 *          8 bytes per row: up to about 580 000 rows; larger requests return ARC_ERR_WORKSPACE
 *          before any launch.
 *   Set-up: the first call on a device looks up the array's device address on that device (it
 *          must be the current device) and keeps it for the life of the process; make that first
 *          call before any stream capture. The kept address is not looked up again, so it is not
 *          valid after cudaDeviceReset (or any other teardown of the device's primary context):
 *          do not call this entry point on a device after resetting it.
 *   Errors: argument, shape and alignment errors are reported first, in the same order as
 *          arc_quantize_act_nvfp4 reports them; ARC_ERR_WORKSPACE (request beyond the array)
 *          comes after them.
 *   Sharing: every call uses the same array and leaves its last contents in it; nothing in the
 *          array needs to start at zero. Calls whose work overlaps on the GPU (other streams,
 *          other host threads) race on the array and must be ordered by the caller.
 */
arc_status arc_quantize_act_nvfp4_static_scratch(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                                 const int32_t* d_idx, int32_t r, const void* rms_gain_bf16,
                                                 float rms_eps, const float* d_static_scale, uint8_t* codes,
                                                 uint8_t* sf, float* d_scale_out, arc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ARC_H_ */
