// Host-side launchers of the NVFP4 kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

constexpr int kMaxPartials = 1024;  // amax pass-1 partial slots in a workspace

// ceil(2^64 / cpr) for the row division of 512-element chunk indices (cpr =
// chunks per row of K elements); unused (0) when cpr == 1.
inline uint64_t chunk_magic(int64_t K) {
  const uint64_t cpr = (uint64_t)((K + 511) / 512);
  return cpr > 1 ? ~uint64_t(0) / cpr + 1 : 0;
}

// ceil(2^32 / cpr) for the narrow (32-bit) chunk-row division; 0 when cpr == 1.
inline uint64_t chunk_magic_narrow(int64_t K) {
  const uint64_t cpr = (uint64_t)((K + 511) / 512);
  return cpr > 1 ? ((uint64_t(1) << 32) + cpr - 1) / cpr : 0;
}

// True when a tensor of M rows x K columns can be walked with 32-bit chunk
// arithmetic: element indices and scale-byte offsets below 2^31 and the
// 32-bit row division exact (chunks * cpr < 2^32).
inline bool narrow_chunks(int64_t M, int64_t K) {
  const int64_t cpr = (K + 511) / 512;
  return (M + 128) * (cpr * 512) < (int64_t(1) << 31) && M * cpr * cpr < (int64_t(1) << 32);
}

int amax_partial_count(int64_t n, int num_sms);
cudaError_t launch_amax_partial(const void* x, int64_t n, uint32_t* partial, int n_partial,
                                cudaStream_t s);
// mode: 0 max, 1 four_over_six, 2 MSE calibration (nvfp4_mode values).
cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, int mode, const uint32_t* partial,
                            int n_partial, const float* g_static, uint8_t* codes, uint8_t* scales,
                            float* g_out, uint8_t* choice, int* status, int num_sms, cudaStream_t s);
cudaError_t launch_fake_quant(const void* x, int64_t M, int64_t K, bool fos, const uint32_t* partial,
                              int n_partial, const float* g_static, const uint8_t* scales_frozen,
                              void* y, int* status, int num_sms, cudaStream_t s);
// Fused single-launch dynamic quantize / fake-quant (amax, grid barrier,
// quantization). ws: kMaxPartials partial slots followed by two barrier
// words that must be zero before the first use. Returns
// cudaErrorNotSupported when the cooperative launch is not possible.
cudaError_t launch_quantize_fused(const void* x, int64_t M, int64_t K, int mode, uint32_t* ws, uint8_t* codes,
                                  uint8_t* scales, float* g_out, uint8_t* choice, int* status, int num_sms,
                                  cudaStream_t s);
cudaError_t launch_fake_quant_fused(const void* x, int64_t M, int64_t K, bool fos, uint32_t* ws, void* y,
                                    int* status, int num_sms, cudaStream_t s);
// Top-k logit KL loss per row (idx / grad nullable; grad needs idx).
cudaError_t launch_topk_kl(const void* teacher, const void* student, int64_t rows, int64_t V, int k, float* loss,
                           int32_t* idx, float* grad, int* status, int num_sms, cudaStream_t s);
// y = BF16(g * s * q) from codes and tiled scales.
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t M, int64_t K,
                              void* y, int* status, int num_sms, cudaStream_t s);
// QAD backward (clipped straight-through estimator); scales as the forward.
cudaError_t launch_fake_quant_bwd(const void* x, const void* gy, int64_t M, int64_t K, bool fos,
                                  const uint32_t* partial, int n_partial, const float* g_static,
                                  const uint8_t* scales_frozen, void* gx, int* status, int num_sms, cudaStream_t s);
cudaError_t launch_fake_quant_bwd_fused(const void* x, const void* gy, int64_t M, int64_t K, bool fos, uint32_t* ws,
                                        void* gx, int* status, int num_sms, cudaStream_t s);
cudaError_t launch_convert(const float* in, int64_t n, uint8_t* out, bool e4m3, int num_sms,
                           cudaStream_t s);
cudaError_t launch_selftest_timeout(uint64_t timeout_ns, int* status, cudaStream_t s);

// Dense W4A4 GEMM (gemm.cu). Returns cudaErrorInvalidValue if a tensor map
// cannot be encoded. timeout_ns = 0 takes the library's 2 s wait bound;
// skip_first_stage != 0 is the bounded-wait test hook (nvf4_gemm_kernel).
cudaError_t launch_gemm(const uint8_t* Aq, const uint8_t* As, const float* ga, const uint8_t* Bq,
                        const uint8_t* Bs, const float* gb, int64_t M, int64_t N, int64_t K,
                        void* C, int* status, int num_sms, cudaStream_t s, uint64_t timeout_ns = 0,
                        int skip_first_stage = 0);

// Routed-expert pipeline (moe.cu).
struct MoeArgs {
  const void* x;
  int64_t T, H, I;
  const int32_t* topk_ids;
  const float* topk_w;
  int topk, E;
  const uint8_t *w13_q, *w13_s;
  const float* w13_g;
  const uint8_t *w2_q, *w2_s;
  const float* w2_g;
  float* out;
  uint8_t* ws;
};
int64_t moe_rows_capacity(int64_t T, int topk, int E);
cudaError_t launch_moe(const MoeArgs& a, int* status, int num_sms, cudaStream_t s);

// Current device: the sm_100 gate, SM count and the address of the device
// status word (api.cu). Returns NVFP4_OK or the gate's error code.
int current_device_context(int* num_sms, int** status);

// Host-side count of kernel launches issued by the library (every launch
// site calls note_launch() just before it launches).
void note_launch();

// Tensor-map encoder from the driver (resolved once through the runtime).
CUresult encode_tensor_map_2d(CUtensorMap* map, const void* base, uint64_t inner_bytes,
                              uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                              uint32_t box_rows);
// Row-major BF16 [rows][cols] written in 32-row x 16-column boxes from a
// 32-byte-swizzled staging box (cols * 2 a multiple of 16).
CUresult encode_store_map_bf16(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows);

}  // namespace nvfp4
