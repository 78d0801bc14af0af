// FP4 tensor-core issue-rate probe: the dense block-scaled MMA
// (tcgen05.mma kind::mxf4nvf4, M=128, N=256, K=64, 16-element UE4M3 scale
// vectors) -- the instruction the W4A4 GEMM of "Why W4A4 rather than W4A16"
// runs -- issued back to back on operands that stay in shared memory, with no
// global-memory traffic. One CTA per SM; the achieved FLOP rate is the
// measured FP4 peak the GEMM's roofline is reported against.
//
// Each CTA: warp 0 fills one stage of operands (A 16 KB, B 32 KB, 12 scale
// tiles) with a fixed non-zero pattern, warp 1 allocates tensor memory,
// copies the scale tiles into it and issues `iters` groups of four MMAs (one
// 256-element K step, as in the GEMM mainloop) into one FP32 accumulator,
// then commits and waits (bounded) for them to finish before the tensor
// memory is freed.
#include "common.cuh"
#include "gemm_kernel.cuh"
#include "kernels.h"

namespace nvfp4 {

// operands need ~55 KB; asking for 120 KB keeps the launch at one CTA per SM
constexpr uint32_t kPeakSmem = 120 * 1024;
static_assert(kABytes + kBBytes + 12 * kSFAtom + 64 + 1024 <= kPeakSmem, "probe shared memory");

__global__ void __launch_bounds__(64, 1) mma_peak_kernel(int iters, int* status, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kABytes;
  uint8_t* sSF = sB + kBBytes;                        // 4 A tiles, then 8 B tiles
  uint64_t* done = reinterpret_cast<uint64_t*>(sSF + 12 * kSFAtom);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5;

  // operands: E2M1 codes of +-0.5..6 in a fixed pattern, scales 1.0 (0x38)
  for (uint32_t i = threadIdx.x; i < (kABytes + kBBytes) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sA)[i] = 0x2A3B4C5Du ^ (i * 0x9E3779B9u & 0x77777777u);
  for (uint32_t i = threadIdx.x; i < 12 * kSFAtom / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sSF)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_barrier_init();
  }
  fence_proxy_async_smem();  // the generic-proxy writes above are read by the tensor cores
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 1) {
    constexpr uint32_t idesc = make_idesc_nvf4(kBM, kBN);
    const uint32_t a = smem_u32(sA), b = smem_u32(sB), sf = smem_u32(sSF);
    const uint64_t adesc = smem_desc(a, 16, 1024, 2);
    const uint64_t bdesc = smem_desc(b, 16, 1024, 2);
    const uint32_t tsfa = tmem + kTmemSF, tsfb = tsfa + kTmemSFBOff;
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      tc_copy_scales_elect(tsfa + 4 * kb, smem_desc(sf + kb * kSFAtom, 0, 128, 0));
      tc_copy_scales_elect(tsfb + 8 * kb, smem_desc(sf + (4 + kb) * kSFAtom, 0, 128, 0));
      tc_copy_scales_elect(tsfb + 8 * kb + 4, smem_desc(sf + (8 + kb) * kSFAtom, 0, 128, 0));
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
        tc_mma_nvf4_elect(tmem, adesc + (uint64_t)(2 * kb), bdesc + (uint64_t)(2 * kb), idesc, tsfa + 4 * kb,
                          tsfb + 8 * kb, (it | kb) != 0);
    }
    tc_commit_elect(done);
    if ((threadIdx.x & 31) == 0) {
      const uint64_t t0 = globaltimer_ns();
      bool ok = true;
      while (!mbar_try_wait(done, 0)) {
        if (globaltimer_ns() - t0 > timeout_ns) {
          ok = false;
          break;
        }
      }
      if (!ok) record_status(status, NVFP4_ERR_TIMEOUT);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_mma_peak(int iters, int ctas, int* status, cudaStream_t s) {
  static cudaError_t attr = cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kPeakSmem);
  if (attr != cudaSuccess) return attr;
  note_launch();
  mma_peak_kernel<<<ctas, 64, kPeakSmem, s>>>(iters, status, 2000000000ull);
  return cudaGetLastError();
}

}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_probe_mma_peak(int iters, double* flops_per_launch, nvfp4_stream_t stream) {
  if (iters < 1 || iters > (1 << 20) || !flops_per_launch) return NVFP4_ERR_INVALID_ARG;
  int num_sms = 0;
  int* status = nullptr;
  const int st = nvfp4::current_device_context(&num_sms, &status);
  if (st != NVFP4_OK) return (nvfp4_status)st;
  *flops_per_launch = 2.0 * nvfp4::kBM * nvfp4::kBN * 256.0 * (double)iters * (double)num_sms;
  return nvfp4::launch_mma_peak(iters, num_sms, status, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? NVFP4_OK
             : NVFP4_ERR_CUDA;
}
