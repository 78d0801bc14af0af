// Device helpers shared by the NVFP4 kernels: format conversions, the
// library status word, and thin wrappers over the sm_100a PTX the GEMM uses
// (mbarrier, TMA, tcgen05).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

#define NVFP4_DEVINL __device__ __forceinline__

namespace nvfp4 {

// Programmatic dependent launch: wait until the preceding grid has completed
// and its memory operations are visible (returns at once when this grid was
// not launched as a programmatic dependent); let the next grid, launched as a
// programmatic dependent of this one, start its set-up.
NVFP4_DEVINL void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
NVFP4_DEVINL void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------------------
// Status word. Kernels get its device address as a parameter and record the
// first non-OK condition with atomicCAS (later conditions do not overwrite).
// ----------------------------------------------------------------------------
NVFP4_DEVINL void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Index check of the bounds-checking build (-DNVFP4_DEBUG_BOUNDS): true when
// i < n; otherwise records NVFP4_ERR_BOUNDS and returns false so that the
// caller skips the access. In the regular build it is the constant true.
NVFP4_DEVINL bool bounds_ok(uint64_t i, uint64_t n, int* status) {
  if (i < n) return true;
  record_status(status, NVFP4_ERR_BOUNDS);
  return false;
}
#ifdef NVFP4_DEBUG_BOUNDS
#define NVFP4_IN_BOUNDS(i, n, status) ::nvfp4::bounds_ok((uint64_t)(i), (uint64_t)(n), (status))
#else
#define NVFP4_IN_BOUNDS(i, n, status) true
#endif

// ----------------------------------------------------------------------------
// Format conversions.
// Round-to-nearest-even, saturating conversions of the NVFP4 format: E2M1
// elements saturate at +-6 and E4M3 block scales at 448 ("Core: W4A4
// two-level scaling", num_bits [2,1] and scale_bits [4,3]).
// ----------------------------------------------------------------------------

// One FP32 value -> E2M1 code in the low nibble.
NVFP4_DEVINL uint32_t e2m1_code(float v) {
  uint16_t out;
  asm("{\n\t"
      ".reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
      "cvt.u16.u8 %0, q;\n\t"
      "}"
      : "=h"(out)
      : "f"(v), "f"(0.0f));
  return out & 0xFu;
}

// Value of an E2M1 magnitude code 0..7: exponent field e (bias 1), mantissa m;
// e == 0 is subnormal (m * 0.5).
NVFP4_DEVINL float e2m1_magnitude(uint32_t k) {
  const uint32_t e = (k >> 1) & 3u, m = k & 1u;
  const float normal = __uint_as_float(((e + 126u) << 23) | (m << 22));
  return e ? normal : (m ? 0.5f : 0.0f);
}

// Non-negative FP32 -> E4M3 code (RNE, satfinite at 448).
NVFP4_DEVINL uint32_t e4m3_code(float t) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(t), "f"(0.0f));
  return out & 0xFFu;
}

// Global scale from amax: g = amax / (6 * 448), FP32, correctly rounded;
// amax == 0 gives g = 1.
NVFP4_DEVINL float global_scale_from_amax(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// E4M3 block-scale code for target magnitude mt (6 or 4): E4M3(bmax / (mt*g)),
// floored at code 1 (2^-9) so that every stored scale is positive.
NVFP4_DEVINL uint32_t block_scale_code(float bmax, float g, float mt) {
  const float t = __fdiv_rn(bmax, __fmul_rn(mt, g));
  const uint32_t c = e4m3_code(t);
  return c > 1u ? c : 1u;
}

NVFP4_DEVINL uint32_t f32x2_to_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // x -> low half
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Nanosecond clock for bounded waits.
NVFP4_DEVINL uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bulk copies (TMA).
// ----------------------------------------------------------------------------
NVFP4_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

NVFP4_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

NVFP4_DEVINL void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

NVFP4_DEVINL void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

NVFP4_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

NVFP4_DEVINL bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Contiguous bulk copy global -> shared (16-byte aligned, size % 16 == 0).
NVFP4_DEVINL void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tiled TMA store of a shared-memory box to global memory (bulk-group
// completion), and the bulk-group bookkeeping around it.
NVFP4_DEVINL void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}
// out[i] += shared[i] for `bytes` / 4 FP32 values (each an atomic add in the
// memory system), from a 16-byte-aligned shared address to a 16-byte-aligned
// global address; bytes a multiple of 16. Bulk-group completion.
NVFP4_DEVINL void bulk_reduce_add_f32(float* dst, uint32_t smem_src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;"
               ::"l"(dst), "r"(smem_src), "r"(bytes) : "memory");
}
NVFP4_DEVINL void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the bulk stores issued by this thread have finished reading shared memory.
NVFP4_DEVINL void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until at most the latest bulk group of this thread may still be reading its source.
NVFP4_DEVINL void bulk_wait_read_but_one() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Wait until the bulk stores issued by this thread are complete.
NVFP4_DEVINL void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
NVFP4_DEVINL void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
NVFP4_DEVINL void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Barrier `id` (1..15; 0 is __syncthreads) over `nthreads` threads (a
// multiple of 32) of the CTA.
NVFP4_DEVINL void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

NVFP4_DEVINL void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, tensor memory).
// ----------------------------------------------------------------------------
NVFP4_DEVINL void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

NVFP4_DEVINL void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

NVFP4_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

NVFP4_DEVINL void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

NVFP4_DEVINL void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

NVFP4_DEVINL void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive FP32 columns of this warp's 32 tensor-memory lanes.
NVFP4_DEVINL void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (16-byte units), descriptor version 1 for sm_100, and
// the swizzle mode (0 none, 2 = 128-byte swizzle).
NVFP4_DEVINL uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                uint32_t swizzle) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)(swizzle & 7u) << 61;
  return d;
}

// ----------------------------------------------------------------------------
// Warp-converged issue. The producer and MMA roles run their loops on all 32
// lanes (so loop state and descriptors stay warp-uniform) and each issuing
// instruction is predicated on elect.sync, which picks the same single lane
// every time for a full mask.
// ----------------------------------------------------------------------------
// Issue helpers for a converged warp: elect.sync picks one lane, which
// issues the operation (the same lane every time, so issue order holds).
#define NVFP4_ELECT_BEGIN "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
#define NVFP4_ELECT_END "\n\t}"

NVFP4_DEVINL void mbar_arrive_expect_tx_elect(uint64_t* bar, uint32_t bytes) {
  asm volatile(NVFP4_ELECT_BEGIN "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" NVFP4_ELECT_END
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// 2-D tiled TMA load into shared memory, completion on an mbarrier.
NVFP4_DEVINL void tma_load_2d_elect(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(NVFP4_ELECT_BEGIN
               "@e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3}], [%4];" NVFP4_ELECT_END
               ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
               : "memory");
}

// Contiguous bulk copy global -> shared, completion on an mbarrier.
NVFP4_DEVINL void bulk_load_elect(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(NVFP4_ELECT_BEGIN
               "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               NVFP4_ELECT_END
               ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Shared -> tensor memory copy of one 512-byte scale tile (32 rows of 16
// bytes), replicated into the four 32-lane quarters of tensor memory.
NVFP4_DEVINL void tc_copy_scales_elect(uint32_t taddr, uint64_t sdesc) {
  asm volatile(NVFP4_ELECT_BEGIN "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" NVFP4_ELECT_END
               ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16-element UE4M3 scales read from
// tensor memory: the block-scaled FP4 MMA (kind::mxf4nvf4, M=128, K=64).
NVFP4_DEVINL void tc_mma_nvf4_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                    uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(NVFP4_ELECT_BEGIN ".reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
               NVFP4_ELECT_END
               ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
               : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far has completed.
NVFP4_DEVINL void tc_commit_elect(uint64_t* bar) {
  asm volatile(NVFP4_ELECT_BEGIN
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" NVFP4_ELECT_END
               ::"r"(smem_u32(bar)) : "memory");
}

// Warp-converged bounded wait: every lane observes the phase; the timeout
// decision is lane 0's, broadcast, so the warp leaves the loop together.
NVFP4_DEVINL bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  uint64_t t0 = 0;
  uint32_t spins = 0;
  const int lane = threadIdx.x & 31;
  while (true) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xFFFFFFFFu, done)) return true;
    if (((++spins) & 63u) == 0) {
      int stop = 0;
      if (lane == 0) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        stop = (*abort != 0) || (now - t0 > limit_ns);
        if (stop) *abort = 1;
      }
      if (__shfl_sync(0xFFFFFFFFu, stop, 0)) return false;
    }
  }
}

}  // namespace nvfp4
