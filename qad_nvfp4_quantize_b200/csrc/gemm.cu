// Dense W4A4 GEMM: C[M x N] (BF16) = (ga*gb) * A_deq[M x K] * B_deq[N x K]^T.
// The mainloop is the tcgen05 block-scaled kernel of gemm_kernel.cuh; this
// file supplies the dense tile order and the epilogue (global-scale product
// and BF16 rounding fused, "Why W4A4 rather than W4A16").
#include <mutex>

#include "gemm_kernel.cuh"
#include "kernels.h"

namespace nvfp4 {

struct DenseProblem {
  static constexpr int kPipeStages = 4;
  static constexpr uint32_t kEpiWarpBytes = kEpiBytes;
  int M, N, K;
  int m_tiles, n_tiles;
  int kgroups;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* ga;
  const float* gb;
  __nv_bfloat16* C;
  const uint8_t *sfa_lo, *sfa_hi, *sfb_lo, *sfb_hi;  // scale buffers (bounds-checking build)

  __device__ __forceinline__ int num_tiles() const { return m_tiles * n_tiles; }

  // m-tile fastest: CTAs running at the same time share B tiles in L2.
  __device__ __forceinline__ TileJob job(int t) const {
    const int mt = t % m_tiles, nt = t / m_tiles;
    TileJob j;
    j.a_row = mt * kBM;
    j.b_row0 = nt * kBN;
    j.b_row1 = nt * kBN + 128;
    const size_t row_tile_bytes = (size_t)kgroups * kSFAtom;
    j.sfa = sfa + (size_t)mt * row_tile_bytes;
    j.sfb0 = sfb + (size_t)(2 * nt) * row_tile_bytes;
    j.sfb1 = (nt * kBN + 128 < N) ? sfb + (size_t)(2 * nt + 1) * row_tile_bytes : nullptr;
    j.expert = 0;
    j.m0 = mt * kBM;
    j.n0 = nt * kBN;
    return j;
  }

  // Columns [h*128, h*128+128) of the accumulator, 32 at a time.
  __device__ static constexpr uint32_t tmem_col(int h, int j) { return (uint32_t)(h * 128 + 32 * j); }

  // Epilogue of one warp (rows q*32.., columns h*128..): scale by ga*gb, round
  // to BF16, and write 32 x 16 boxes through the warp's shared staging box with
  // TMA stores (rows >= M and columns >= N are clipped by the tensor map). The
  // staging box uses the 32-byte swizzle, so the 32 row writes of a warp fall
  // on distinct shared-memory banks.
  __device__ __forceinline__ void store(const TileJob& job, int q, int h, int lane, const uint32_t (&acc)[4][32],
                                        uint8_t* stg, const CUtensorMap* tmC) const {
    const int row0 = job.m0 + q * 32;
    if (row0 >= M) return;
    const float alpha = __fmul_rn(*ga, *gb);
    const uint32_t sbase = smem_u32(stg);
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += kEpiCols) {
      const int n = job.n0 + h * 128 + c0;
      if (n >= N) break;
      if (lane == 0) bulk_wait_read_all();  // the previous box has left shared memory
      __syncwarp();
#pragma unroll
      for (int ch = 0; ch < kEpiCols / 8; ++ch) {
        const uint32_t* a = &acc[(c0 + ch * 8) / 32][(c0 + ch * 8) % 32];
        uint4 w;
        w.x = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(a[0]), alpha), __fmul_rn(__uint_as_float(a[1]), alpha));
        w.y = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(a[2]), alpha), __fmul_rn(__uint_as_float(a[3]), alpha));
        w.z = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(a[4]), alpha), __fmul_rn(__uint_as_float(a[5]), alpha));
        w.w = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(a[6]), alpha), __fmul_rn(__uint_as_float(a[7]), alpha));
        // 32-byte swizzle: 16-byte chunk index XOR bit 2 of the row
        st_shared_v4(sbase + lane * (kEpiCols * 2) + ((ch ^ ((lane >> 2) & 1)) << 4), w);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmC, stg, n, row0);
        bulk_commit_group();
      }
    }
  }
};

// ----------------------------------------------------------------------------
// Tensor maps. cuTensorMapEncodeTiled is a driver entry point; it is resolved
// once through the runtime so the library does not link libcuda directly.
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D byte tensor [rows][inner_bytes] with a 128-byte-swizzled box of
// box_rows x box_inner bytes; out-of-range elements read as zero.
CUresult encode_tensor_map_2d(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = get_encoder();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Row-major BF16 [rows][cols] output written in 32-row x kEpiCols-column boxes
// from a 32-byte-swizzled staging box. cols * 2 must be a multiple of 16.
CUresult encode_store_map_bf16(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
  EncodeTiledFn fn = get_encoder();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kEpiCols, 32};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <class Prob>
static cudaError_t prepare_kernel() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(nvf4_gemm_kernel<Prob>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)gemm_smem_bytes<Prob>());
  });
  return err;
}

constexpr uint64_t kGemmTimeoutNs = 2000000000ull;  // 2 s per wait: far beyond any legitimate stall

cudaError_t launch_gemm(const uint8_t* Aq, const uint8_t* As, const float* ga, const uint8_t* Bq,
                        const uint8_t* Bs, const float* gb, int64_t M, int64_t N, int64_t K, void* C,
                        int* status, int num_sms, cudaStream_t s, uint64_t timeout_ns, int skip_first_stage) {
  if (M == 0) return cudaSuccess;
  if (timeout_ns == 0) timeout_ns = kGemmTimeoutNs;
  CUtensorMap tmA, tmB;
  if (encode_tensor_map_2d(&tmA, Aq, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, kBK / 2, kBM) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&tmB, Bq, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, kBK / 2, 128) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  DenseProblem p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.m_tiles = (int)((M + kBM - 1) / kBM);
  p.n_tiles = (int)((N + kBN - 1) / kBN);
  p.kgroups = (int)(K / 64);
  p.sfa = As;
  p.sfb = Bs;
  p.ga = ga;
  p.gb = gb;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.sfa_lo = As;
  p.sfa_hi = As + (size_t)p.m_tiles * p.kgroups * kSFAtom;
  p.sfb_lo = Bs;
  p.sfb_hi = Bs + (size_t)((N + 127) / 128) * p.kgroups * kSFAtom;
  cudaError_t e = prepare_kernel<DenseProblem>();
  if (e != cudaSuccess) return e;
  CUtensorMap tmC;
  if (encode_store_map_bf16(&tmC, C, (uint64_t)N, (uint64_t)M) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  // Programmatic dependent launch: the CTAs' set-up (barriers, tensor
  // memory, descriptor prefetch) overlaps the tail of the kernel that wrote A
  // (the dynamic quantize); the kernel waits for it before reading A.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = gemm_smem_bytes<DenseProblem>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, nvf4_gemm_kernel<DenseProblem>, tmA, tmB, tmC, p, status, timeout_ns,
                            skip_first_stage);
}

}  // namespace nvfp4
