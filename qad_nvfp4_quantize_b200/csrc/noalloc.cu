// nvfp4_quantize_noalloc: nvfp4_quantize for callers that cannot allocate.
//
// Some callers cannot hand the library a workspace: an inference plugin whose
// enqueue step only receives input and output pointers, or code running where
// the device allocator is unavailable or forbidden (no cudaMalloc, no caching
// allocator). For them this entry point computes the dynamic global scale with
// a scratch array that the library owns for the life of the process, so the
// call itself allocates nothing.
//
// The scratch is a file-scope __device__ array of kNoallocSlots 32-bit slots
// (16 KiB). Every GPU that loads the library holds one copy until the process
// exits. The amax pass uses one slot per block of kNoallocElemsPerSlot input
// elements, so inputs of up to kNoallocSlots * kNoallocElemsPerSlot = 2^30
// elements (M * K) fit; larger inputs are rejected with NVFP4_ERR_TOO_LARGE
// before anything is launched.
//
// The array keeps the last call's contents. Nothing in it needs to start at
// zero: the amax pass writes every slot that the quantize pass then reads.
// All calls on a device share the array, so two calls whose kernels overlap on
// the GPU (different streams without ordering between them) race on it and
// may both produce wrong global scales; order such calls on one stream.
//
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress and caches it; in host
// code the array's name is only a host-side stand-in, never a device address.
// Make that first call before any stream capture on the device.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int64_t kNoallocSlots = 4096;
constexpr int64_t kNoallocElemsPerSlot = int64_t(1) << 18;
constexpr int kMaxDevicesNoalloc = 64;

static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoallocSlots];

uint32_t* g_scratch_addr[kMaxDevicesNoalloc] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once).
nvfp4_status scratch_address(uint32_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
  if (dev >= kMaxDevicesNoalloc) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return NVFP4_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t M, int64_t K, nvfp4_mode mode,
                                                const float* g_in, uint8_t* codes, uint8_t* scales,
                                                float* g_out, uint8_t* fos_choice, nvfp4_stream_t stream) {
  if (M < 0 || K <= 0 || K % 64 || (mode != NVFP4_MODE_MAX && mode != NVFP4_MODE_FOUR_OVER_SIX))
    return NVFP4_ERR_INVALID_ARG;
  if (M > kNoallocSlots * kNoallocElemsPerSlot / K) return NVFP4_ERR_TOO_LARGE;
  if (M > 0 && (!x || !codes || !scales || !al16(x) || !al16(codes) || !al16(scales)))
    return NVFP4_ERR_INVALID_ARG;
  int num_sms = 0;
  int* status = nullptr;
  const int st = nvfp4::current_device_context(&num_sms, &status);
  if (st != NVFP4_OK) return (nvfp4_status)st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = M * K;
  uint32_t* partial = nullptr;
  int np = 0;
  if (!g_in) {
    const nvfp4_status sst = scratch_address(&partial);
    if (sst != NVFP4_OK) return sst;
    // as many amax CTAs (one slot each) as the two-pass quantize uses for
    // its own partials, and at least one per 2^18 elements; never more than
    // the array holds (n <= 2^30 gives at most kNoallocSlots)
    int64_t want = (n + kNoallocElemsPerSlot - 1) / kNoallocElemsPerSlot;
    const int64_t grid = nvfp4::amax_partial_count(n, num_sms);
    if (want < grid) want = grid;
    if (want > kNoallocSlots) want = kNoallocSlots;
    np = (int)(want < 1 ? 1 : want);
    if (nvfp4::launch_amax_partial(x, n, partial, np, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return nvfp4::launch_quantize(x, M, K, (int)mode, partial, np, g_in, codes, scales,
                                g_out, fos_choice, status, num_sms, s) == cudaSuccess
             ? NVFP4_OK
             : NVFP4_ERR_CUDA;
}
