// NVFP4 quantize, four_over_six calibration and fake-quant kernels.
//
// The format is the two-level scaling of "How is Qwen3.8-Flash-Next-NVFP4's
// NVFP4 quantization done?" (section "Core: W4A4 two-level scaling"): an FP32
// global scale g per tensor (level 2) and an E4M3 block scale per 16
// contiguous elements (level 1), E2M1 element codes. four_over_six and the
// frozen-scale fake-quant follow Table 1 and "Quantization scale handling
// during QAD" of "Developing Nemotron 3.5 Lightning NVFP4 with QAD using
// NVIDIA Model Optimizer".
//
// Work decomposition (HBM-bound streaming): a warp handles a chunk of 256
// consecutive elements of the flattened [M x K] tensor; lane i loads 16 bytes
// (8 BF16) with one coalesced 128-bit load, a lane pair forms one 16-element
// block, the pair's maximum comes from one shuffle. Codes leave as one 32-bit
// store per lane (128 contiguous bytes per warp); four consecutive block
// scales (one 64-element group of a row) leave as one 32-bit store into the
// tiled scale layout.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kQThreads = 256;  // 8 warps
constexpr int kAmaxThreads = 256;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kUnroll = 2;  // chunks of 512 elements in flight per warp

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ----------------------------------------------------------------------------
// amax, pass 1: per-CTA maximum of |x| as a BF16 magnitude (bits & 0x7FFF).
// Magnitudes of finite BF16 values order like their bit patterns; anything
// >= 0x7F80 is Inf or NaN, so the maximum also flags non-finite input.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(kAmaxThreads, 8) amax_partial_kernel(const uint4* __restrict__ x,
                                                                    int64_t n_vec,
                                                                    uint32_t* __restrict__ partial) {
  uint32_t m2 = 0;  // two 16-bit magnitudes
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n_vec; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ld_stream(x + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m2 = __vmaxu2(m2, v[u].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].w & 0x7FFF7FFFu);
    }
  }
  for (; i < n_vec; i += stride) {
    const uint4 v = ld_stream(x + i);
    m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.w & 0x7FFF7FFFu);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
  __shared__ uint32_t red[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < kAmaxThreads / 32; ++w) r = max(r, red[w]);
    partial[blockIdx.x] = r;
  }
}

// Global scale for this call: reduce the pass-1 partials (dynamic) or read the
// static scale. Every CTA does this redundantly (a few hundred L2 reads), so
// no atomics and no zero-initialised scratch are needed. Returns g; sets
// *nonfinite when the amax is Inf/NaN.
__device__ __forceinline__ float resolve_global_scale(const uint32_t* partial, int n_partial,
                                                      const float* g_static, bool* nonfinite) {
  __shared__ float s_g;
  __shared__ int s_bad;
  if (threadIdx.x < 32) {
    float g;
    int bad = 0;
    if (g_static) {
      g = *g_static;
    } else {
      uint32_t m = 0;
      for (int base = 0; base < n_partial; base += 8 * 32) {  // 8 independent loads per lane
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + u * 32 + (int)threadIdx.x;
          v[u] = i < n_partial ? partial[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) m = max(m, v[u]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
      bad = m >= 0x7F80u;
      g = global_scale_from_amax(__uint_as_float(m << 16));
    }
    if (threadIdx.x == 0) {
      s_g = g;
      s_bad = bad;
    }
  }
  __syncthreads();
  *nonfinite = s_bad != 0;
  return s_g;
}

// Byte offset of scale (row, block column c) in the tiled layout; kgroups =
// K / 64 is the number of 4-scale tiles per 128-row tile row.
__device__ __forceinline__ int64_t scale_offset(int64_t row, int64_t c, int64_t kgroups) {
  return (((row >> 7) * kgroups + (c >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) +
         (c & 3);
}

// A warp's unit of work: 512 consecutive elements of one row ("chunk"), one
// 16-element block per lane. Chunks never straddle rows; a row of K elements
// has ceil(K/512) chunks and the last one may be partial. The row division is
// warp-uniform.
struct Chunk {
  int64_t row;
  int32_t col;        // this lane's first element within the row
  bool valid;         // col < K
  int64_t vec;        // 16-byte vector index of the block's first 8 elements
};

__device__ __forceinline__ Chunk chunk_at(int64_t ch, int32_t cpr, int64_t K, int lane) {
  Chunk c;
  const uint32_t chu = (uint32_t)ch;  // the launcher keeps chunk counts below 2^31
  const uint32_t r = chu / (uint32_t)cpr;
  c.row = r;
  c.col = (int32_t)(chu - r * (uint32_t)cpr) * 512 + lane * 16;
  c.valid = c.col < K;
  c.vec = (c.row * K + c.col) >> 3;
  return c;
}

__device__ __forceinline__ void load16(const uint4* x, int64_t vec, bool valid, float (&v)[16]) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (valid) {
    a = ld_stream(x + vec);
    b = ld_stream(x + vec + 1);
  }
  bf16x2_to_f32(a.x, v[0], v[1]);
  bf16x2_to_f32(a.y, v[2], v[3]);
  bf16x2_to_f32(a.z, v[4], v[5]);
  bf16x2_to_f32(a.w, v[6], v[7]);
  bf16x2_to_f32(b.x, v[8], v[9]);
  bf16x2_to_f32(b.y, v[10], v[11]);
  bf16x2_to_f32(b.z, v[12], v[13]);
  bf16x2_to_f32(b.w, v[14], v[15]);
}

// One 16-element block: scale code, packed codes (two 32-bit words, element 2j
// in the low nibble of byte j) and, when requested, the dequantized values
// and the block's squared error summed in element order.
struct Block {
  uint32_t sc;
  uint32_t q0, q1;
  float deq[16];
  float err;
};

template <bool kDeq, bool kErr>
__device__ __forceinline__ void quantize_block(const float (&v)[16], float bmax, float g, float mt, Block& b) {
  b.sc = block_scale_code(bmax, g, mt);
  const float d = __fmul_rn(g, e4m3_value(b.sc));
  const float r = __frcp_rn(d);
  float sv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) sv[i] = __fmul_rn(v[i], r);
  b.q0 = e2m1_pack8(sv);
  b.q1 = e2m1_pack8(sv + 8);
  if (kDeq || kErr) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      b.deq[i] = __fmul_rn(d, e2m1_value(((i < 8 ? b.q0 : b.q1) >> (4 * (i & 7))) & 0xFu));
  }
  if (kErr) {
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float df = __fsub_rn(v[i], b.deq[i]);
      acc = __fadd_rn(acc, __fmul_rn(df, df));
    }
    b.err = acc;
  } else {
    b.err = 0.0f;
  }
}

__device__ __forceinline__ float abs_max16(const float (&v)[16]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

// Gather the scale codes of the 4 blocks of a 64-element group onto the
// group's first lane (lanes 4c .. 4c+3 hold blocks 4c .. 4c+3).
__device__ __forceinline__ uint32_t gather_group_scales(uint32_t sc) {
  const uint32_t s1 = __shfl_down_sync(kFull, sc, 1);
  const uint32_t s2 = __shfl_down_sync(kFull, sc, 2);
  const uint32_t s3 = __shfl_down_sync(kFull, sc, 3);
  return sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
}

// Zero the scale bytes of the padding rows [M, ceil128(M)).
__device__ __forceinline__ void zero_pad_scale_rows(uint8_t* scales, int64_t M, int64_t kgroups) {
  const int64_t pad = ((M + 127) & ~int64_t(127)) - M;
  const int64_t total = pad * kgroups;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = M + i / kgroups, cg = i % kgroups;
    *reinterpret_cast<uint32_t*>(scales + scale_offset(row, cg * 4, kgroups)) = 0u;
  }
}

// ----------------------------------------------------------------------------
// Quantize (pass 2). kFos: four_over_six calibration.
// ----------------------------------------------------------------------------
template <bool kFos>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(
    const uint4* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ partial,
    int n_partial, const float* __restrict__ g_static, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ g_out, uint8_t* __restrict__ choice,
    int* status) {
  bool bad;
  const float g = resolve_global_scale(partial, n_partial, g_static, &bad);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (g_out) *g_out = g;
    if (bad) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
  }
  const int64_t kgroups = K >> 6;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int64_t n_chunks = M * cpr;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (kQThreads / 32);

  // kUnroll chunks per trip with all loads issued first (memory-level parallelism)
  for (int64_t ch0 = warp; ch0 < n_chunks; ch0 += kUnroll * nwarps) {
    float vv[kUnroll][16];
    Chunk cc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      cc[u] = chunk_at(ch0 + u * nwarps, cpr, K, lane);
      load16(x, cc[u].vec, cc[u].valid && ch0 + u * nwarps < n_chunks, vv[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (ch0 + u * nwarps >= n_chunks) break;  // warp-uniform
      const float bmax = abs_max16(vv[u]);
      Block b6;
      quantize_block<false, kFos>(vv[u], bmax, g, 6.0f, b6);
      uint32_t sc = b6.sc, q0 = b6.q0, q1 = b6.q1, pick4 = 0;
      if (kFos) {
        Block b4;
        quantize_block<false, true>(vv[u], bmax, g, 4.0f, b4);
        pick4 = b4.err < b6.err;  // tie keeps M = 6
        if (pick4) {
          sc = b4.sc;
          q0 = b4.q0;
          q1 = b4.q1;
        }
      }
      const uint32_t group = gather_group_scales(sc);
      if (cc[u].valid) {
        codes[cc[u].vec >> 1] = make_uint2(q0, q1);
        if ((lane & 3) == 0)
          *reinterpret_cast<uint32_t*>(scales + scale_offset(cc[u].row, cc[u].col >> 4, kgroups)) = group;
        if (kFos && choice) choice[cc[u].vec >> 1] = (uint8_t)pick4;
      }
    }
  }
  if (!kFos && choice) {  // max mode still fills the optional choice map with 0
    const int64_t nb = (M * K) >> 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb;
         i += (int64_t)gridDim.x * blockDim.x)
      choice[i] = 0;
  }
  zero_pad_scale_rows(scales, M, kgroups);
}

// ----------------------------------------------------------------------------
// Fake-quant: y = BF16(g * s * q). Modes: dynamic/static g with computed block
// scales (max or four_over_six), or frozen g* and s* (tiled layout).
// ----------------------------------------------------------------------------
template <bool kFos, bool kFrozen>
__global__ void __launch_bounds__(kQThreads) fake_quant_kernel(
    const uint4* __restrict__ x, int64_t M, int64_t K, const uint32_t* __restrict__ partial,
    int n_partial, const float* __restrict__ g_static, const uint8_t* __restrict__ scales_frozen,
    uint4* __restrict__ y, int* status) {
  bool bad;
  const float g = resolve_global_scale(partial, n_partial, g_static, &bad);
  if (blockIdx.x == 0 && threadIdx.x == 0 && bad) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
  const int64_t kgroups = K >> 6;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int64_t n_chunks = M * cpr;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (kQThreads / 32);

  for (int64_t ch0 = warp; ch0 < n_chunks; ch0 += kUnroll * nwarps) {
    float vv[kUnroll][16];
    Chunk cc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      cc[u] = chunk_at(ch0 + u * nwarps, cpr, K, lane);
      load16(x, cc[u].vec, cc[u].valid && ch0 + u * nwarps < n_chunks, vv[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (ch0 + u * nwarps >= n_chunks) break;  // warp-uniform
      float out[16];
      if (kFrozen) {
        const uint32_t sc = cc[u].valid ? scales_frozen[scale_offset(cc[u].row, cc[u].col >> 4, kgroups)] : 1u;
        const float d = __fmul_rn(g, e4m3_value(sc));
        const float r = __frcp_rn(d);
        float sv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[i] = __fmul_rn(vv[u][i], r);
        const uint32_t q0 = e2m1_pack8(sv), q1 = e2m1_pack8(sv + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) out[i] = __fmul_rn(d, e2m1_value(((i < 8 ? q0 : q1) >> (4 * (i & 7))) & 0xFu));
      } else {
        const float bmax = abs_max16(vv[u]);
        Block b6;
        quantize_block<true, kFos>(vv[u], bmax, g, 6.0f, b6);
        if (kFos) {
          Block b4;
          quantize_block<true, true>(vv[u], bmax, g, 4.0f, b4);
          const bool pick4 = b4.err < b6.err;
#pragma unroll
          for (int i = 0; i < 16; ++i) out[i] = pick4 ? b4.deq[i] : b6.deq[i];
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) out[i] = b6.deq[i];
        }
      }
      if (cc[u].valid) {
        uint4 w0, w1;
        w0.x = f32x2_to_bf16x2(out[0], out[1]);
        w0.y = f32x2_to_bf16x2(out[2], out[3]);
        w0.z = f32x2_to_bf16x2(out[4], out[5]);
        w0.w = f32x2_to_bf16x2(out[6], out[7]);
        w1.x = f32x2_to_bf16x2(out[8], out[9]);
        w1.y = f32x2_to_bf16x2(out[10], out[11]);
        w1.z = f32x2_to_bf16x2(out[12], out[13]);
        w1.w = f32x2_to_bf16x2(out[14], out[15]);
        y[cc[u].vec] = w0;
        y[cc[u].vec + 1] = w1;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Conversion primitives and the bounded-wait self test.
// ----------------------------------------------------------------------------
__global__ void convert_e2m1_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint8_t)e2m1_code(in[i]);
}

__global__ void convert_e4m3_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint8_t)e4m3_code(in[i]);
}

__device__ int g_never_set_flag = 0;

__global__ void selftest_timeout_kernel(uint64_t timeout_ns, int* status) {
  if (threadIdx.x != 0) return;
  volatile int* flag = &g_never_set_flag;
  const uint64_t t0 = globaltimer_ns();
  while (*flag == 0) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_status(status, NVFP4_ERR_TIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

// ----------------------------------------------------------------------------
// Host launchers.
// ----------------------------------------------------------------------------
static int grid_for(int64_t work_items, int per_block, int max_blocks) {
  int64_t b = (work_items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > max_blocks) b = max_blocks;
  return (int)b;
}

int amax_partial_count(int64_t n, int num_sms) {
  // about 4 vectors of 8 BF16 per thread per loop trip, 4 CTAs per SM at most
  return grid_for(n / 8, kAmaxThreads * 16, num_sms * 6 > kMaxPartials ? kMaxPartials : num_sms * 6);
}

cudaError_t launch_amax_partial(const void* x, int64_t n, uint32_t* partial, int n_partial,
                                cudaStream_t s) {
  amax_partial_kernel<<<n_partial, kAmaxThreads, 0, s>>>(static_cast<const uint4*>(x), n / 8, partial);
  return cudaGetLastError();
}

template <class Kern>
static int resident_blocks(Kern k) {
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, kQThreads, 0) != cudaSuccess || b < 1) b = 1;
  return b;
}

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, bool fos, const uint32_t* partial,
                            int n_partial, const float* g_static, uint8_t* codes, uint8_t* scales,
                            float* g_out, uint8_t* choice, int* status, int num_sms, cudaStream_t s) {
  const int64_t chunks = M * ((K + 511) / 512);
  if (chunks >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  static const int occ_max = resident_blocks(quantize_kernel<false>);
  static const int occ_fos = resident_blocks(quantize_kernel<true>);
  const int grid = grid_for(chunks, kQThreads / 32 * kUnroll, num_sms * (fos ? occ_fos : occ_max));
  if (fos)
    quantize_kernel<true><<<grid, kQThreads, 0, s>>>(static_cast<const uint4*>(x), M, K, partial, n_partial,
                                                      g_static, reinterpret_cast<uint2*>(codes), scales,
                                                      g_out, choice, status);
  else
    quantize_kernel<false><<<grid, kQThreads, 0, s>>>(static_cast<const uint4*>(x), M, K, partial, n_partial,
                                                       g_static, reinterpret_cast<uint2*>(codes), scales,
                                                       g_out, choice, status);
  return cudaGetLastError();
}

cudaError_t launch_fake_quant(const void* x, int64_t M, int64_t K, bool fos, const uint32_t* partial,
                              int n_partial, const float* g_static, const uint8_t* scales_frozen,
                              void* y, int* status, int num_sms, cudaStream_t s) {
  const int64_t chunks = M * ((K + 511) / 512);
  if (chunks >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  static const int occ = resident_blocks(fake_quant_kernel<true, false>);
  const int grid = grid_for(chunks, kQThreads / 32 * kUnroll, num_sms * occ);
  const uint4* xv = static_cast<const uint4*>(x);
  uint4* yv = static_cast<uint4*>(y);
  if (scales_frozen)
    fake_quant_kernel<false, true><<<grid, kQThreads, 0, s>>>(xv, M, K, partial, n_partial, g_static,
                                                              scales_frozen, yv, status);
  else if (fos)
    fake_quant_kernel<true, false><<<grid, kQThreads, 0, s>>>(xv, M, K, partial, n_partial, g_static,
                                                              nullptr, yv, status);
  else
    fake_quant_kernel<false, false><<<grid, kQThreads, 0, s>>>(xv, M, K, partial, n_partial, g_static,
                                                               nullptr, yv, status);
  return cudaGetLastError();
}

cudaError_t launch_convert(const float* in, int64_t n, uint8_t* out, bool e4m3, int num_sms,
                           cudaStream_t s) {
  const int grid = grid_for(n, 256, num_sms * 8);
  if (e4m3)
    convert_e4m3_kernel<<<grid, 256, 0, s>>>(in, n, out);
  else
    convert_e2m1_kernel<<<grid, 256, 0, s>>>(in, n, out);
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint64_t timeout_ns, int* status, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(timeout_ns, status);
  return cudaGetLastError();
}

}  // namespace nvfp4
