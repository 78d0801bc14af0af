// Block-scaled W4A4 GEMM mainloop for sm_100a (tcgen05 + TMA + TMEM).
//
// C = (ga*gb) * sum_k (sa*qa)(sb*qb): E2M1 operands with one UE4M3 scale per
// 16 elements of K, FP32 accumulation in tensor memory -- the FP4 tensor-core
// GEMM that "Why W4A4 rather than W4A16" ("Model-Optimizer in practice:
// recovering Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD") says W4A4 unlocks.
//
// One CTA per SM, persistent over output tiles of 128 x 256. Warp roles:
//   warp 0      TMA producer: codes of A (128 rows) and B (two boxes of 128
//               rows) and the matching 512-byte scale tiles, 4-stage ring of
//               256 K-elements per stage, mbarrier transaction counts;
//   warp 1      allocates tensor memory; one lane copies the scale tiles
//               shared -> tensor memory (tcgen05.cp) and issues the
//               block-scaled MMAs (kind::mxf4nvf4, M=128, N=256, K=64);
//   warps 2..9  epilogue: drain the 128 x 256 FP32 accumulator from tensor
//               memory into registers, release it to the MMA warp, then scale,
//               round and store (policy-specific; the dense store stages
//               32 x 16 boxes in shared memory and writes them with TMA, so C
//               leaves as whole 32-byte rows instead of 16-byte pieces of 32
//               rows that would compete with the operand loads).
// Tensor memory: columns [0,256) accumulator; from column 256 each pipeline
// stage owns 48 columns of scales -- 16 for A (4 per MMA) then 32 for B (8 per
// MMA) -- so the scale copy of one stage never overwrites columns that MMAs of
// the previous stages may still read.
// Every mbarrier wait is bounded; on expiry the CTA records
// NVFP4_ERR_TIMEOUT, drains its in-flight copies and MMAs (bounded) and
// returns with its tensor memory freed. With `skip_first_stage` set (a test
// hook), the producer of CTA 0 leaves the first stage of its first tile
// unissued -- no copy is in flight for it -- so the MMA warp's wait on that
// stage runs out and the drain path above is taken.
#pragma once

#include "common.cuh"

namespace nvfp4 {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 256;                       // K elements per stage
constexpr uint32_t kABytes = kBM * kBK / 2;    // 16 KB of codes
constexpr uint32_t kBHalfBytes = 128 * kBK / 2;
constexpr uint32_t kBBytes = kBN * kBK / 2;    // 32 KB
constexpr uint32_t kSFAtom = 512;              // 128 rows x 4 scales
constexpr uint32_t kSFABytes = 4 * kSFAtom;
constexpr uint32_t kSFBBytes = 8 * kSFAtom;
constexpr int kGemmThreads = 320;
constexpr int kEpiCols = 16;                   // dense output columns per TMA store box
constexpr uint32_t kEpiBytes = 32 * kEpiCols * 2;  // one epilogue warp's BF16 staging box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSF = 256;         // first scale column
constexpr uint32_t kTmemSFStage = 48;     // scale columns per stage
constexpr uint32_t kTmemSFBOff = 16;      // B scales after A scales inside a stage

// Shared-memory layout of one CTA for a problem with `kStagesT` pipeline
// stages and `kEpiWarpBytesT` bytes of epilogue staging per epilogue warp.
template <int kStagesT, uint32_t kEpiWarpBytesT>
struct GemmSmem {
  static constexpr int kStages = kStagesT;
  static constexpr uint32_t kA = 0;
  static constexpr uint32_t kB = kA + kStages * kABytes;
  static constexpr uint32_t kSFA = kB + kStages * kBBytes;
  static constexpr uint32_t kSFB = kSFA + kStages * kSFABytes;
  static constexpr uint32_t kEpi = kSFB + kStages * kSFBBytes;  // 8 warps x kEpiWarpBytesT
  static constexpr uint32_t kEpiWarp = kEpiWarpBytesT;
  static constexpr uint32_t kBar = kEpi + 8 * kEpiWarpBytesT;
  static constexpr uint32_t kNumBars = 2 * kStages + 3;   // full, empty, acc_full, acc_empty, drain
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 16 + 1024;  // + alignment slack
  static_assert(kTmemSF + kStages * kTmemSFStage <= kTmemCols, "tensor memory budget");
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Dynamic shared memory of nvf4_gemm_kernel<Prob>.
template <class Prob>
constexpr uint32_t gemm_smem_bytes() {
  return GemmSmem<Prob::kPipeStages, Prob::kEpiWarpBytes>::kBytes;
}

// Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// UE4M3 scales (scale format 0), N >> 3 in bits [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t make_idesc_nvf4(int m, int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// What the producer needs to fetch for one output tile.
struct TileJob {
  int32_t a_row;          // first row of A in A's tensor map
  int32_t b_row0;         // B rows for accumulator columns [0,128)
  int32_t b_row1;         // B rows for accumulator columns [128,256)
  const uint8_t* sfa;     // A scale tiles of this 128-row tile, K-group 0
  const uint8_t* sfb0;    // B scale tiles for b_row0
  const uint8_t* sfb1;    // B scale tiles for b_row1 (nullptr: none)
  int32_t expert;
  int32_t m0, n0;
};

template <class Prob>
__global__ void __launch_bounds__(kGemmThreads, 1)
    nvf4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const Prob prob, int* status,
                     uint64_t timeout_ns, int skip_first_stage) {
  using Lay = GemmSmem<Prob::kPipeStages, Prob::kEpiWarpBytes>;
  constexpr int kStages = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);  // one arrive per epilogue warp
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int K = prob.K;
  const int nkt = (K + kBK - 1) / kBK;
  const int kgroups = K / 64;
  const int ntiles = prob.num_tiles();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (warp-uniform state); elect.sync issues.
    // Launched as a programmatic dependent of the kernel that wrote A, the
    // set-up above overlapped that kernel's tail; its outputs are read only
    // after this wait (a no-op for an ordinary launch).
    grid_dependency_wait();
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0;  // bit s: stage s armed; bit 8+s: its phase
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      const TileJob job = prob.job(t);
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        if (skip_first_stage && blockIdx.x == 0 && t == 0 && kt == 0) {
          // test hook: nothing armed, nothing in flight for this stage
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          continue;
        }
        const int nkb = min(4, kgroups - 4 * kt);
        const uint32_t sf_bytes = (uint32_t)nkb * kSFAtom;
        const uint32_t tx = kABytes + kBBytes + sf_bytes * (job.sfb1 ? 3u : 2u);
        mbar_arrive_expect_tx_elect(&full[stage], tx);
        armed = (armed & ~(0x101u << stage)) | (1u << stage) | (phase << (8 + stage));
        uint8_t* sA = smem + Lay::kA + stage * kABytes;
        uint8_t* sB = smem + Lay::kB + stage * kBBytes;
        tma_load_2d_elect(sA, &tmA, kt * (kBK / 2), job.a_row, &full[stage]);
        tma_load_2d_elect(sB, &tmB, kt * (kBK / 2), job.b_row0, &full[stage]);
        tma_load_2d_elect(sB + kBHalfBytes, &tmB, kt * (kBK / 2), job.b_row1, &full[stage]);
        const uint8_t* pa = job.sfa + (size_t)kt * kSFABytes;
        const uint8_t* pb0 = job.sfb0 + (size_t)kt * kSFABytes;
        const uint8_t* pb1 = job.sfb1 ? job.sfb1 + (size_t)kt * kSFABytes : nullptr;
#ifdef NVFP4_DEBUG_BOUNDS
        // scale tiles outside their buffers: reported, and read from the
        // buffer's start instead so that the stage still completes
        if (pa < prob.sfa_lo || pa + sf_bytes > prob.sfa_hi) {
          if (lane == 0) record_status(status, NVFP4_ERR_BOUNDS);
          pa = prob.sfa_lo;
        }
        if (pb0 < prob.sfb_lo || pb0 + sf_bytes > prob.sfb_hi) {
          if (lane == 0) record_status(status, NVFP4_ERR_BOUNDS);
          pb0 = prob.sfb_lo;
        }
        if (pb1 && (pb1 < prob.sfb_lo || pb1 + sf_bytes > prob.sfb_hi)) {
          if (lane == 0) record_status(status, NVFP4_ERR_BOUNDS);
          pb1 = prob.sfb_lo;
        }
#endif
        bulk_load_elect(smem + Lay::kSFA + stage * kSFABytes, pa, sf_bytes, &full[stage]);
        uint8_t* sSFB = smem + Lay::kSFB + stage * kSFBBytes;
        bulk_load_elect(sSFB, pb0, sf_bytes, &full[stage]);
        if (pb1) bulk_load_elect(sSFB + kSFABytes, pb1, sf_bytes, &full[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      // let copies already in flight land before the CTA exits
      record_status(status, NVFP4_ERR_TIMEOUT);
      for (int s = 0; s < kStages; ++s) {
        if (!((armed >> s) & 1u)) continue;
        const uint32_t ph = (armed >> (8 + s)) & 1u;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[s], ph) && globaltimer_ns() - t0 < 1000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // Warp-converged loop; scale copies, MMAs and commits issued by one
    // elected lane (the same lane each time, so they stay in issue order).
    constexpr uint32_t idesc = make_idesc_nvf4(kBM, kBN);
    uint32_t stage = 0, phase = 0, acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      if (!mbar_wait_warp(acc_empty, acc_phase ^ 1, abort_flag, timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait_warp(&full[stage], phase, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nkb = min(4, kgroups - 4 * kt);
        const uint32_t sA = smem_u32(smem + Lay::kA + stage * kABytes);
        const uint32_t sB = smem_u32(smem + Lay::kB + stage * kBBytes);
        const uint32_t sSFA = smem_u32(smem + Lay::kSFA + stage * kSFABytes);
        const uint32_t sSFB = smem_u32(smem + Lay::kSFB + stage * kSFBBytes);
        const uint64_t adesc = smem_desc(sA, 16, 1024, 2);
        const uint64_t bdesc = smem_desc(sB, 16, 1024, 2);
        const uint32_t tsfa = tmem + kTmemSF + stage * kTmemSFStage;
        const uint32_t tsfb = tsfa + kTmemSFBOff;
        // All of the stage's scale copies first, then its MMAs: an MMA issued
        // right behind the copies it reads waited for them each time
        // (measured: 146 -> 137 us on 4096 x 17408 x 5120).
        if (nkb == 4) {
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tc_copy_scales_elect(tsfa + 4 * kb, smem_desc(sSFA + kb * kSFAtom, 0, 128, 0));
            tc_copy_scales_elect(tsfb + 8 * kb, smem_desc(sSFB + kb * kSFAtom, 0, 128, 0));
            tc_copy_scales_elect(tsfb + 8 * kb + 4, smem_desc(sSFB + kSFABytes + kb * kSFAtom, 0, 128, 0));
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)  // K advance inside the 128-byte swizzle atom: 32 bytes per MMA
            tc_mma_nvf4_elect(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb), idesc, tsfa + 4 * kb,
                              tsfb + 8 * kb, (kt | kb) != 0);
        } else {
          for (int kb = 0; kb < nkb; ++kb) {
            tc_copy_scales_elect(tsfa + 4 * kb, smem_desc(sSFA + kb * kSFAtom, 0, 128, 0));
            tc_copy_scales_elect(tsfb + 8 * kb, smem_desc(sSFB + kb * kSFAtom, 0, 128, 0));
            tc_copy_scales_elect(tsfb + 8 * kb + 4, smem_desc(sSFB + kSFABytes + kb * kSFAtom, 0, 128, 0));
          }
          for (int kb = 0; kb < nkb; ++kb)
            tc_mma_nvf4_elect(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb), idesc, tsfa + 4 * kb,
                              tsfb + 8 * kb, (kt | kb) != 0);
        }
        tc_commit_elect(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit_elect(acc_full);
      acc_phase ^= 1;
    }
    if (!ok) {
      tc_commit_elect(drain);  // wait (bounded) for MMAs already issued
      if (lane == 0) {
        record_status(status, NVFP4_ERR_TIMEOUT);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000ull) {
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();          // global scales written by the previous kernel
    const int q = warp & 3;          // tensor-memory lane quarter of this warp
    const int h = (warp - 2) >> 2;   // which half of the tile's columns
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      if (!mbar_wait_warp(acc_full, acc_phase, abort_flag, timeout_ns)) {
        if (lane == 0) record_status(status, NVFP4_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      uint32_t acc[4][32];
      const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(lane_addr + Prob::tmem_col(h, j), acc[j]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const TileJob job = prob.job(t);
      prob.store(job, q, h, lane, acc, smem + Lay::kEpi + (warp - 2) * Lay::kEpiWarp, &tmC);
      acc_phase ^= 1;
    }
    bulk_wait_all();  // bulk stores / reductions issued by this lane complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace nvfp4
