// C ABI entry points (include/nvfp4.h): argument validation, the sm_100
// hardware gate, the device status word, and dispatch to the kernels.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// Library-owned device status word (one per device: module globals are
// instantiated on every device that loads the library).
__device__ int g_device_status = 0;

struct DeviceInfo {
  int checked = 0;     // 0 unknown, 1 supported, -1 unsupported
  int num_sms = 0;
  int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

nvfp4_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
  if (dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) {
      d.checked = -1;
    } else {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return NVFP4_ERR_CUDA;
      d.status = static_cast<int*>(p);
      d.num_sms = sms;
      d.checked = 1;
    }
  }
  if (d.checked < 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return NVFP4_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvfp4_status launched(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Dynamic global scale: amax pass 1 into the workspace.
nvfp4_status run_amax(const void* x, int64_t n, void* ws, size_t ws_bytes, int num_sms, cudaStream_t s,
                      const uint32_t** partial, int* n_partial) {
  if (!ws || ws_bytes < nvfp4_quantize_workspace_bytes(1, 64) || !aligned16(ws)) return NVFP4_ERR_WORKSPACE;
  const int np = nvfp4::amax_partial_count(n, num_sms);
  uint32_t* part = static_cast<uint32_t*>(ws);
  if (nvfp4::launch_amax_partial(x, n, part, np, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  *partial = part;
  *n_partial = np;
  return NVFP4_OK;
}

std::atomic<uint64_t> g_launches{0};

}  // namespace

void nvfp4::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int nvfp4::current_device_context(int* num_sms, int** status) {
  DeviceInfo* d;
  const nvfp4_status st = current_device(&d);
  if (st == NVFP4_OK) {
    *num_sms = d->num_sms;
    *status = d->status;
  }
  return st;
}

extern "C" {

int nvfp4_version(void) { return 100; }

nvfp4_status nvfp4_check_device(void) {
  DeviceInfo* d;
  return current_device(&d);
}

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "unsupported device (NVFP4 needs sm_100)";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_NONFINITE_INPUT: return "non-finite input";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_TOO_LARGE: return "input larger than the no-alloc entry point's static scratch (M*K > 2^30)";
    case NVFP4_ERR_BOUNDS: return "a computed index fell outside its buffer (bounds-checking build)";
  }
  return "unknown status";
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 64) return 0;
  return (size_t)((rows + 127) / 128) * (size_t)(K / 64) * 512u;
}

size_t nvfp4_quantize_workspace_bytes(int64_t M, int64_t K) {
  (void)M;
  (void)K;
  // partial maxima, then the two grid-barrier words (padded to 256 bytes)
  return (size_t)nvfp4::kMaxPartials * sizeof(uint32_t) + 256;
}

nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t K, nvfp4_mode mode, const float* g_in,
                            uint8_t* codes, uint8_t* scales, float* g_out, uint8_t* fos_choice,
                            void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  if (M < 0 || K <= 0 || K % 64 ||
      (mode != NVFP4_MODE_MAX && mode != NVFP4_MODE_FOUR_OVER_SIX && mode != NVFP4_MODE_MSE))
    return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !codes || !scales || !aligned16(x) || !aligned16(codes) || !aligned16(scales)))
    return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t* partial = nullptr;
  int np = 0;
  const int m = (int)mode;
  if (!g_in) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_bytes(M, K) || !aligned16(workspace))
      return NVFP4_ERR_WORKSPACE;
    // one launch: amax, grid barrier and quantization with X kept on chip
    const cudaError_t e = nvfp4::launch_quantize_fused(x, M, K, m, static_cast<uint32_t*>(workspace), codes,
                                                       scales, g_out, fos_choice, d->status, d->num_sms, s);
    if (e != cudaErrorNotSupported) return launched(e);
    st = run_amax(x, M * K, workspace, workspace_bytes, d->num_sms, s, &partial, &np);
    if (st != NVFP4_OK) return st;
  }
  return launched(nvfp4::launch_quantize(x, M, K, m, partial, np, g_in, codes, scales, g_out, fos_choice,
                                         d->status, d->num_sms, s));
}

nvfp4_status nvfp4_fake_quant(const void* x, int64_t M, int64_t K, nvfp4_mode mode, const float* g_frozen,
                              const uint8_t* scales_frozen, void* y, void* workspace, size_t workspace_bytes,
                              nvfp4_stream_t stream) {
  if (M < 0 || K <= 0 || K % 64 || (mode != NVFP4_MODE_MAX && mode != NVFP4_MODE_FOUR_OVER_SIX))
    return NVFP4_ERR_INVALID_ARG;
  if (scales_frozen && !g_frozen) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y || !aligned16(x) || !aligned16(y) || x == y)) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t* partial = nullptr;
  int np = 0;
  const bool fos = mode == NVFP4_MODE_FOUR_OVER_SIX;
  if (!g_frozen) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_bytes(M, K) || !aligned16(workspace))
      return NVFP4_ERR_WORKSPACE;
    const cudaError_t e =
        nvfp4::launch_fake_quant_fused(x, M, K, fos, static_cast<uint32_t*>(workspace), y, d->status, d->num_sms, s);
    if (e != cudaErrorNotSupported) return launched(e);
    st = run_amax(x, M * K, workspace, workspace_bytes, d->num_sms, s, &partial, &np);
    if (st != NVFP4_OK) return st;
  }
  return launched(nvfp4::launch_fake_quant(x, M, K, fos, partial, np, g_frozen, scales_frozen, y, d->status,
                                           d->num_sms, s));
}

nvfp4_status nvfp4_gemm(const uint8_t* Aq, const uint8_t* As, const float* ga, const uint8_t* Bq,
                        const uint8_t* Bs, const float* gb, int64_t M, int64_t N, int64_t K, void* C,
                        nvfp4_stream_t stream) {
  if (M < 0 || N <= 0 || K <= 0 || K % 64 || N % 16 || M >= (1ll << 31) || N >= (1ll << 31))
    return NVFP4_ERR_INVALID_ARG;
  if (!Bq || !Bs || !gb || !aligned16(Bq) || !aligned16(Bs)) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!Aq || !As || !ga || !C || !aligned16(Aq) || !aligned16(As) || !aligned16(C)))
    return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return launched(nvfp4::launch_gemm(Aq, As, ga, Bq, Bs, gb, M, N, K, C, d->status, d->num_sms, s));
}

nvfp4_status nvfp4_convert_e2m1(const float* in, int64_t n, uint8_t* out, nvfp4_stream_t stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  if (n == 0) return NVFP4_OK;
  return launched(nvfp4::launch_convert(in, n, out, false, d->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_convert_e4m3(const float* in, int64_t n, uint8_t* out, nvfp4_stream_t stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  if (n == 0) return NVFP4_OK;
  return launched(nvfp4::launch_convert(in, n, out, true, d->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_topk_kl(const void* teacher, const void* student, int64_t rows, int64_t V, int k, float* loss,
                           int32_t* idx, float* grad, nvfp4_stream_t stream) {
  if (rows < 0 || V <= 0 || V % 8 || k < 1 || k > V || (grad && !idx)) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && (!teacher || !student || !loss || !aligned16(teacher) || !aligned16(student)))
    return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  return launched(nvfp4::launch_topk_kl(teacher, student, rows, V, k, loss, idx, grad, d->status, d->num_sms,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t M, int64_t K,
                              void* y, nvfp4_stream_t stream) {
  if (M < 0 || K <= 0 || K % 64) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!codes || !scales || !g || !y || !aligned16(codes) || !aligned16(y))) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  if (M == 0) return NVFP4_OK;
  return launched(nvfp4::launch_dequantize(codes, scales, g, M, K, y, d->status, d->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_fake_quant_backward(const void* x, const void* grad_y, int64_t M, int64_t K, nvfp4_mode mode,
                                       const float* g_frozen, const uint8_t* scales_frozen, void* grad_x,
                                       void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  if (M < 0 || K <= 0 || K % 64 || (mode != NVFP4_MODE_MAX && mode != NVFP4_MODE_FOUR_OVER_SIX))
    return NVFP4_ERR_INVALID_ARG;
  if (scales_frozen && !g_frozen) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !grad_y || !grad_x || !aligned16(x) || !aligned16(grad_y) || !aligned16(grad_x) ||
                grad_x == x || grad_x == grad_y))
    return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t* partial = nullptr;
  int np = 0;
  const bool fos = mode == NVFP4_MODE_FOUR_OVER_SIX;
  if (!g_frozen) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_bytes(M, K) || !aligned16(workspace))
      return NVFP4_ERR_WORKSPACE;
    const cudaError_t e = nvfp4::launch_fake_quant_bwd_fused(x, grad_y, M, K, fos, static_cast<uint32_t*>(workspace),
                                                             grad_x, d->status, d->num_sms, s);
    if (e != cudaErrorNotSupported) return launched(e);
    st = run_amax(x, M * K, workspace, workspace_bytes, d->num_sms, s, &partial, &np);
    if (st != NVFP4_OK) return st;
  }
  return launched(nvfp4::launch_fake_quant_bwd(x, grad_y, M, K, fos, partial, np, g_frozen, scales_frozen, grad_x,
                                               d->status, d->num_sms, s));
}

nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream, int clear, nvfp4_status* out) {
  if (!out) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (clear && cudaMemset(d->status, 0, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
  *out = static_cast<nvfp4_status>(v);
  return NVFP4_OK;
}

uint64_t nvfp4_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

nvfp4_status nvfp4_selftest_gemm_timeout(const uint8_t* Aq, const uint8_t* As, const float* ga, const uint8_t* Bq,
                                          const uint8_t* Bs, const float* gb, int64_t M, int64_t N, int64_t K,
                                          void* C, uint64_t timeout_ns, nvfp4_stream_t stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;  // (0, 10 s]
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 || N % 16 || M >= (1ll << 31) || N >= (1ll << 31))
    return NVFP4_ERR_INVALID_ARG;
  if (!Aq || !As || !ga || !Bq || !Bs || !gb || !C || !aligned16(Aq) || !aligned16(As) || !aligned16(Bq) ||
      !aligned16(Bs) || !aligned16(C))
    return NVFP4_ERR_INVALID_ARG;
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  return launched(nvfp4::launch_gemm(Aq, As, ga, Bq, Bs, gb, M, N, K, C, d->status, d->num_sms,
                                     reinterpret_cast<cudaStream_t>(stream), timeout_ns, 1));
}

nvfp4_status nvfp4_selftest_timeout(uint64_t timeout_ns, nvfp4_stream_t stream) {
  if (timeout_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARG;  // at most 10 s
  DeviceInfo* d;
  nvfp4_status st = current_device(&d);
  if (st != NVFP4_OK) return st;
  return launched(nvfp4::launch_selftest_timeout(timeout_ns, d->status, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
