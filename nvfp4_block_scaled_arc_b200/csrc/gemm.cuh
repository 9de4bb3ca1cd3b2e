// gemm.cuh -- the compute-bound half of the hot path: one persistent, warp-specialised
// tcgen05 GEMM skeleton instantiated for three operand kinds.
//   FP4:         block-scaled NVFP4 GEMM of depth K_aug (tcgen05.mma kind::mxf4nvf4,
//                scale_vec::4X: one E4M3 scale per 16 elements of A and of B), the unified
//                GEMM of "ARCQuant ... Augmented Residual Channels" (Unified GEMM Executie:
//                one GEMM over K_in + S absorbs the residual correction by linearity), epilogue
//                Y = bf16(s_A s_B acc [+ add]).
//   BF16:        BF16 GEMM (tcgen05.mma kind::f16), the reference-precision switch of RAMP
//                (section 4.1: the recurrent steps after the switch run in BF16).
//   FP8:         E4M3 x E4M3 GEMM (tcgen05.mma kind::f8f6f4) with per-tensor scales, epilogue
//                Y = bf16(s_A s_B acc [+ add]): RAMP's own low-precision format (FP8 W8A8).
//
// CTA = 15 warps, one CTA per SM, persistent over 128 x 256 output tiles (grouped raster):
//   warp 0       TMA producer: per stage an A tile of 128 rows x 128 bytes and a B tile of 256
//                rows x 128 bytes (128-byte swizzle), plus A's scale atoms of the stage as a 1-D
//                bulk copy (up to 4 atoms of its 128-row block); it arms the stage's barrier with
//                all of the stage's bytes, B's scale atoms (warp 2) included; no multicast.
//   warp 1       MMA issue, one thread, every pipeline stage in order: the fp32 accumulation
//                order is fixed, so results are reproducible bit for bit. The issuing thread
//                does no release/acquire memory operation: one such pair per stage in this
//                thread costs about 40% of the tensor pipe's throughput (measured with the MMA
//                issue loop alone, 7.1 against 5.1 PFLOP/s), while tcgen05 fences cost nothing.
//                Warp 1 also owns the TMEM allocation.
//   warp 2       (FP4) issues each stage's bulk copies of B's scale atoms, beside the producer's
//                operand and A-scale copies: two small copies fewer in the producer's sequence
//                make the stages land sooner (7 % on gateup). Its position also keeps the scale
//                writers and epilogue warps on the TMEM lane quarters their warp index selects.
//   warps 3..6   (FP4) scale writers, one per TMEM lane quarter: they read the stage's scale
//                bytes from shared memory and store them into the stage's set of TMEM scale
//                columns with tcgen05.st, in the cell order the block-scaled MMA reads
//                (A: row m at lane m, column base + m/32; B: column n at lane 32q + n%32 of
//                every quarter q, column base + n/32). Register stores keep the tensor pipe free
//                for MMAs; tcgen05.cp of the same bytes costs the pipe ~70 cycles per copy.
//   warps 7..14  epilogue: tcgen05.ld of the fp32 accumulator (warp w owns TMEM lane quarter
//                w%4 = tile rows 32*(w%4)..+31, and one 128-column half), scale by alpha; bf16
//                output staged 32 x 16 at a time in shared memory and written by TMA stores (the
//                residual-add form reads the add term and stores directly).
// TMEM (512 columns): fp32 accumulator 128 lanes x 256 columns (two of them for bf16); fp4
// keeps one and uses columns 256..511 as four 64-column scale sets, one per pipeline stage
// (B scales at +0..31, 8 columns per K=64 step; A scales at +32 + 4k + quarter).
// Every wait is bounded (wait_ns); a wait that runs out raises the CTA's abort flag and the
// device status word, and the CTA drains what it issued and frees its tensor memory before it
// returns.
#pragma once

#include "arc_device.cuh"

namespace arc {

// GEMM kinds: the BF16 reference GEMM, the block-scaled NVFP4 GEMM, the per-tensor-scaled FP8 GEMM.
constexpr int kGemmBF16 = 0, kGemmFP4 = 1, kGemmFP8 = 2, kGemmMX4 = 3;

template <int KIND>
struct GemmTraits;

template <>
struct GemmTraits<kGemmFP4> {
  static constexpr int BM = 128, BN = 256, STAGES = 4, ACC_STAGES = 1;
  static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 4 * 512, SFB_BYTES = 2 * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr uint32_t IDESC = idesc_nvf4(BM, BN);
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 256, SF_SET_COLS = 64;
};

template <>
struct GemmTraits<kGemmBF16> {
  static constexpr int BM = 128, BN = 256, STAGES = 4, ACC_STAGES = 2;
  static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 0, SFB_BYTES = 0;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN);
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 0, SF_SET_COLS = 0;
};

// MXFP4: the FP4 geometry with one UE8M0 scale per 32 elements; a stage's 256 K-elements per row
// are 8 scales, two 512-byte atoms per 128-row block.
template <>
struct GemmTraits<kGemmMX4> {
  static constexpr int BM = 128, BN = 256, STAGES = 4, ACC_STAGES = 1;
  static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 2 * 512, SFB_BYTES = 2 * 2 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr uint32_t IDESC = idesc_mxf4(BM, BN);
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 256, SF_SET_COLS = 64;
};

// FP8: the BF16 geometry (128 bytes of K per row and stage = 128 E4M3 values, 4 MMAs of K = 32)
template <>
struct GemmTraits<kGemmFP8> {
  static constexpr int BM = 128, BN = 256, STAGES = 4, ACC_STAGES = 2;
  static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 0, SFB_BYTES = 0;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t IDESC = idesc_f8(BM, BN);
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 0, SF_SET_COLS = 0;
};

// Output staging for the TMA-store epilogue: per epilogue warp one 32-row x 16-column bf16 chunk.
constexpr int kEpiStageBytes = 32 * 16 * 2;

template <int KIND>
constexpr int gemm_smem_bytes() {
  return GemmTraits<KIND>::STAGES * GemmTraits<KIND>::STAGE_BYTES + 8 * kEpiStageBytes + 1024 + 256;
}

// TMA tensor store of a box from shared memory (bulk-group completion), and its waits.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(m),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct GemmArgs {
  int M, N;
  int ksteps;   // MMA K-steps over the whole depth
  int kstages;  // pipeline stages per tile (4 K-steps each)
  int katoms;   // fp4: 512-byte scale atoms per 128-row block (K_pad / 64)
  int nblk128;  // fp4: 128-row blocks of B's scales (ceil(N / 128))
  int tiles_m, tiles_n;
  int group_m;  // raster: consecutive tiles walk group_m row blocks before the next column block
  int box_rows_a, box_rows_b;  // TMA box heights (min(128, M), min(256, N))
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* a_scale;
  const float* b_scale;
  __nv_bfloat16* y;
  int64_t ldy;
  const __nv_bfloat16* add;
  int64_t ld_add;
  uint64_t wait_ns;
  int inject;
};

// Grouped raster: tiles t = 0, 1, ... walk GM row blocks of one column block, then the same row
// blocks of the next column block, and so on; then the next group of row blocks. A group's A
// rows stay in L2 while B streams through it once per group.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int GM, int& tm, int& tn) {
  const int per_group = GM * tiles_n;
  const int group = t / per_group;
  const int first_m = group * GM;
  const int gm = min(GM, tiles_m - first_m);
  const int rr = t - group * per_group;
  tm = first_m + rr % gm;
  tn = rr / gm;
}


__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds_u32x4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// One MMA of a pipeline stage: K-step k of the stage, operand descriptors already offset to it
// (32 bytes of K per step = 2 descriptor units), scales (block-scaled kinds) from the stage's set:
// A's at sf + 32 + 4k, B's at sf + 8k.
template <int KIND>
__device__ __forceinline__ void mma_step(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t sf, int k,
                                         uint32_t accum) {
  using T = GemmTraits<KIND>;
  if constexpr (KIND == kGemmFP4)
    tc_mma_nvf4(d_tmem, da, db, T::IDESC, sf + 32 + 4 * k, sf + 8 * k, accum);
  else if constexpr (KIND == kGemmMX4)
    tc_mma_mxf4(d_tmem, da, db, T::IDESC, sf + 32 + 4 * k, sf + 8 * k, accum);
  else if constexpr (KIND == kGemmFP8)
    tc_mma_f8(d_tmem, da, db, T::IDESC, accum);
  else
    tc_mma_bf16(d_tmem, da, db, T::IDESC, accum);
}

constexpr int kGemmThreads = 480;  // producer, MMA issuer, idle warp, 4 scale writers, 8 epilogue warps
constexpr int kGemmEpiWarp0 = 7;

template <int KIND, bool ADD>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmY, const GemmArgs g) {
  using T = GemmTraits<KIND>;
  constexpr bool NV4 = KIND == kGemmFP4, MX4 = KIND == kGemmMX4, FP8 = KIND == kGemmFP8;
  constexpr bool FP4 = NV4 || MX4;  // block-scaled E2M1 operands, scales in tensor memory
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + T::STAGES * T::STAGE_BYTES;  // 8 x 1 KB, one per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + 8 * kEpiStageBytes);
  uint64_t* empty = full + T::STAGES;
  uint64_t* ready = empty + T::STAGES;  // fp4: the stage's scales are in TMEM
  uint64_t* acc_full = ready + T::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;  // the MMA thread's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 4);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);   // one commit per tile
      mbar_init(&acc_empty[a], 8);  // one arrival from each epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!ADD) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // everything above overlaps the previous kernel's tail; nothing below runs before it is done
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = g.tiles_m * g.tiles_n;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
      bool skip = (g.inject == 1) && blockIdx.x == 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, g.tiles_m, g.tiles_n, g.group_m, tm, tn);
        for (int ks = 0; ks < g.kstages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * T::STAGE_BYTES;
          uint8_t* sB = sA + T::A_BYTES;
          if (skip) {
            skip = false;  // failure injection: this stage's loads are never issued
          } else {
            uint32_t bytes = static_cast<uint32_t>(g.box_rows_a + g.box_rows_b) * 128u;
            int natoms = 0, nb = 0;
            constexpr int APS = MX4 ? 2 : 4;  // scale atoms per stage and 128-row block
            if (FP4) {
              natoms = min(APS, g.katoms - APS * ks);
              nb = min(2, g.nblk128 - 2 * tn);
              bytes += static_cast<uint32_t>(natoms * 512 * (1 + nb));
            }
            mbar_arrive_expect_tx(&full[stage], bytes);
            const int kx = (FP4 || FP8) ? ks * 128 : ks * 64;  // byte maps for FP4 / FP8, bf16 map
            tma_load_2d(sA, &tmA, &full[stage], kx, tm * T::BM);
            tma_load_2d(sB, &tmB, &full[stage], kx, tn * T::BN);
            if (FP4) {
              uint8_t* sSFA = sB + T::B_BYTES;
              uint8_t* sSFB = sSFA + T::SFA_BYTES;
              bulk_load(sSFA, g.sfa + (static_cast<int64_t>(tm) * g.katoms + APS * ks) * 512, natoms * 512, &full[stage]);
              (void)sSFB;  // B's scale atoms: warp 2
            }
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == T::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let every load this thread issued land before the CTA goes away
        for (int s = 0; s < T::STAGES; ++s)
          if ((armed >> s) & 1u) mbar_wait_teardown(&full[s], (armed_par >> s) & 1u, g.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issue
      // Each tcgen05.mma is accepted only about as fast as the tensor pipe runs them, so every
      // instruction between two MMAs lengthens the pipe's idle time at a stage boundary: the
      // stage's descriptors and scale columns are advanced by one add each, and the four MMAs of
      // a full stage are unrolled (5 % on the llama8b projections against recomputing them).
      uint32_t acc = 0, acc_phase = 0;
      uint32_t stage = 0, phase = 0;  // the same stage sequence the producer walks
      bool ok = true;
      constexpr uint64_t kStageDesc = static_cast<uint64_t>(T::STAGE_BYTES >> 4);  // descriptor units
      constexpr uint64_t kBDesc = static_cast<uint64_t>(T::A_BYTES >> 4);
      const uint64_t da0 = desc_kmajor_sw128(smem_u32(smem));
      uint64_t da = da0;                 // stage's A tile; its B tile at da + kBDesc
      uint32_t sf = tmem + T::SF_COL0;   // stage's scale set
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        // the accumulator must have been drained by the epilogue
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, g.wait_ns, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * T::BN;
        for (int ks = 0; ks < g.kstages; ++ks) {
          if (!mbar_wait(FP4 ? &ready[stage] : &full[stage], phase, g.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = da + kBDesc;
          const uint32_t acc0 = ks > 0 ? 1u : 0u;  // the tile's first MMA overwrites
          // MMAs in this stage: 4 of K = 64 (FP4) / K = 32 (FP8) / K = 16 (BF16), fewer at the end
          const int nk = (FP4 || FP8) ? min(4, g.ksteps - 4 * ks) : 4;
          if (nk == 4) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_step<KIND>(d_tmem, da + 2 * k, db + 2 * k, sf, k, k > 0 ? 1u : acc0);
          } else {
            for (int k = 0; k < nk; ++k) mma_step<KIND>(d_tmem, da + 2 * k, db + 2 * k, sf, k, k > 0 ? 1u : acc0);
          }
          tc_commit(&empty[stage]);
          if (++stage == T::STAGES) {
            stage = 0;
            phase ^= 1u;
            da = da0;
            sf = tmem + T::SF_COL0;
          } else {
            da += kStageDesc;
            sf += T::SF_SET_COLS;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == T::ACC_STAGES) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // nothing issued may still be running when the tensor memory is released
      tc_commit(drain);
      mbar_wait_teardown(drain, 0, g.wait_ns);
    }
  } else if (warp == 2) {
    if (FP4 && lane == 0) {
      // B's scale atoms of every stage, issued beside the producer's copies
      constexpr int APS = MX4 ? 2 : 4;
      uint32_t stage = 0, phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, g.tiles_m, g.tiles_n, g.group_m, tm, tn);
        (void)tm;
        for (int ks = 0; ks < g.kstages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          const int natoms = min(APS, g.katoms - APS * ks);
          const int nb = min(2, g.nblk128 - 2 * tn);
          uint8_t* sSFB = smem + stage * T::STAGE_BYTES + T::A_BYTES + T::B_BYTES + T::SFA_BYTES;
          for (int b = 0; b < nb; ++b)
            bulk_load(sSFB + b * APS * 512, g.sfb + (static_cast<int64_t>(2 * tn + b) * g.katoms + APS * ks) * 512,
                      natoms * 512, &full[stage]);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == T::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < T::STAGES; ++s)
          if ((armed >> s) & 1u) mbar_wait_teardown(&full[s], (armed_par >> s) & 1u, g.wait_ns);
      }
    }
  } else if (warp < kGemmEpiWarp0) {
    if (FP4) {
      // ------------------------------------------------------------------ scale writers
      const int q = warp & 3;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        for (int ks = 0; ks < g.kstages; ++ks) {
          const bool got = mbar_wait(&full[stage], phase, g.wait_ns, abort_flag);
          if (!__all_sync(0xFFFFFFFFu, got)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sSFA = smem_u32(smem + stage * T::STAGE_BYTES + T::A_BYTES + T::B_BYTES);
          const uint32_t sSFB = sSFA + T::SFA_BYTES;
          const uint32_t set = lane_base + T::SF_COL0 + T::SF_SET_COLS * stage;
          uint32_t v[32];
          if (NV4) {
            // one atom per K = 64 step: a row's 4 scales are one 32-bit cell
            const int natoms = min(4, g.katoms - 4 * ks);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
              if (k < natoms) {
                b0 = lds_u32x4(sSFB + k * 512 + lane * 16);
                b1 = lds_u32x4(sSFB + 2048 + k * 512 + lane * 16);
              }
              v[8 * k + 0] = b0.x, v[8 * k + 1] = b0.y, v[8 * k + 2] = b0.z, v[8 * k + 3] = b0.w;
              v[8 * k + 4] = b1.x, v[8 * k + 5] = b1.y, v[8 * k + 6] = b1.z, v[8 * k + 7] = b1.w;
            }
            tmem_st_32x32b_x32(set, v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t a = (k < natoms) ? lds_u32(sSFA + k * 512 + lane * 16 + 4 * q) : 0u;
              tmem_st_32x32b_x1(set + 32 + 4 * k + q, a);
            }
          } else {
            // MXFP4: one atom per two K = 64 steps; step k's two scales are half k % 2 of the
            // atom's 32-bit word, stored in bytes 0 and 1 of the step's cell
            const int natoms = min(2, g.katoms - 2 * ks);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int at = k >> 1, sh = 16 * (k & 1);
              uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
              if (at < natoms) {
                b0 = lds_u32x4(sSFB + at * 512 + lane * 16);
                b1 = lds_u32x4(sSFB + 1024 + at * 512 + lane * 16);
              }
              v[8 * k + 0] = (b0.x >> sh) & 0xFFFFu, v[8 * k + 1] = (b0.y >> sh) & 0xFFFFu;
              v[8 * k + 2] = (b0.z >> sh) & 0xFFFFu, v[8 * k + 3] = (b0.w >> sh) & 0xFFFFu;
              v[8 * k + 4] = (b1.x >> sh) & 0xFFFFu, v[8 * k + 5] = (b1.y >> sh) & 0xFFFFu;
              v[8 * k + 6] = (b1.z >> sh) & 0xFFFFu, v[8 * k + 7] = (b1.w >> sh) & 0xFFFFu;
            }
            tmem_st_32x32b_x32(set, v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int at = k >> 1, sh = 16 * (k & 1);
              const uint32_t a = (at < natoms) ? (lds_u32(sSFA + at * 512 + lane * 16 + 4 * q) >> sh) & 0xFFFFu : 0u;
              tmem_st_32x32b_x1(set + 32 + 4 * k + q, a);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ready[stage]);
          if (++stage == T::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // 8 warps: warp w reads TMEM lane quarter w%4 (tile rows 32*(w%4)..+31) and column half
    // (w-7)/4 (128 columns). Without a residual add the warp converts its 32 x 128 block to
    // bf16 chunk by chunk as it leaves TMEM, releases the accumulator, then stores; with an add,
    // the residual block is prefetched into registers and the accumulator is read, combined and
    // stored 32 columns at a time.
    const int q = warp & 3;
    const int half = (warp - kGemmEpiWarp0) >> 2;
    const float alpha = (NV4 || FP8) ? __fmul_rn(*g.a_scale, *g.b_scale) : 1.0f;  // MXFP4: no tensor scales
    const uint64_t alpha2 = f2_pack(alpha, alpha);
    constexpr int HB = T::BN / 2;  // columns per warp
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int tm, tn;
      tile_coords(t, g.tiles_m, g.tiles_n, g.group_m, tm, tn);
      const int row = tm * T::BM + q * 32 + lane;
      const bool row_ok = row < g.M;
      const int col0 = tn * T::BN + half * HB;
      __nv_bfloat16* yrow = g.y + static_cast<int64_t>(row) * g.ldy;
      uint32_t addv[ADD ? HB / 2 : 1];
      if (ADD) {
#pragma unroll
        for (int j = 0; j < HB / 8; ++j) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (row_ok && col0 + 8 * j < g.N)
            v = *reinterpret_cast<const uint4*>(g.add + static_cast<int64_t>(row) * g.ld_add + col0 + 8 * j);
          addv[4 * j + 0] = v.x;
          addv[4 * j + 1] = v.y;
          addv[4 * j + 2] = v.z;
          addv[4 * j + 3] = v.w;
        }
      }
      // every lane waits; the warp goes on only if all of them saw the accumulator (the TMEM
      // loads below are warp-collective, so the decision must be uniform)
      const bool got = mbar_wait(&acc_full[acc], acc_phase, g.wait_ns, abort_flag, 64);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * T::BN + half * HB;
      if (!ADD) {
        uint32_t pk[HB / 2];
#pragma unroll
        for (int c = 0; c < HB / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), alpha2), a0, a1);
            pk[16 * c + e] = pack_bf16x2_rn(a0, a1);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        // stores through the warp's staging chunk: thread i writes row i's 16 columns, one TMA
        // store moves the 32 x 16 box to Y (clipped at the matrix edges)
        uint8_t* stg = staging + (warp - kGemmEpiWarp0) * kEpiStageBytes;
        const int row0 = tm * T::BM + q * 32;
#pragma unroll
        for (int c = 0; c < HB / 16; ++c) {
          uint4* dst = reinterpret_cast<uint4*>(stg + lane * 32);
          dst[0] = make_uint4(pk[8 * c], pk[8 * c + 1], pk[8 * c + 2], pk[8 * c + 3]);
          dst[1] = make_uint4(pk[8 * c + 4], pk[8 * c + 5], pk[8 * c + 6], pk[8 * c + 7]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, stg, col0 + 16 * c, row0);
            bulk_commit_group();
            bulk_wait_read_all();  // the chunk may be overwritten once the TMA has read it
          }
          __syncwarp();
        }
        (void)row_ok;
        (void)yrow;
      } else {
#pragma unroll
        for (int c = 0; c < HB / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c * 32, r);
          tmem_ld_wait();
          if (c == HB / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
          }
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = col0 + c * 32 + 8 * j;
              if (col < g.N) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const uint32_t w = addv[(c * 32 + 8 * j + e) >> 1];
                  f[e] = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[8 * j + e])), (e & 1) ? bf16_hi(w) : bf16_lo(w));
                }
                uint4 o;
                o.x = pack_bf16x2_rn(f[0], f[1]);
                o.y = pack_bf16x2_rn(f[2], f[3]);
                o.z = pack_bf16x2_rn(f[4], f[5]);
                o.w = pack_bf16x2_rn(f[6], f[7]);
                *reinterpret_cast<uint4*>(yrow + col) = o;
              }
            }
          }
        }
      }
      if (++acc == T::ACC_STAGES) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (!ADD && lane == 0) bulk_wait_all();  // every output store has completed
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

}  // namespace arc
