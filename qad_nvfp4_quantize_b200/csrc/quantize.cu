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
// Work decomposition: a warp's unit is a 512-element chunk of one row, one
// 16-element block per lane (block_math.cuh). Codes leave as one 8-byte store
// per lane, block scales as one byte per lane into the tiled scale layout,
// BF16 outputs (fake-quant, STE, dequantize) as one 32-byte store per lane
// when the output is 32-byte aligned.
// Dynamic calls run as a single cooperative launch (fused_dynamic_kernel);
// static-scale and frozen-scale calls stream once (stream_pass_kernel).
#include <type_traits>

#include "block_math.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kQThreads = 256;  // 8 warps
constexpr int kAmaxThreads = 256;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kUnroll = 2;  // chunks of 512 elements in flight per warp
constexpr uint64_t kFusedTimeoutNs = 2000000000ull;  // grid-barrier wait bound

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
  uint32_t m = mag_max_halves(m2);
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

// Buffer extents of an [M x K] tensor for the bounds-checking build: 16-byte
// vectors of BF16 values, 8-byte words of codes (16 codes), tiled scale bytes.
__device__ __forceinline__ int64_t n_vec16(int64_t M, int64_t K) { return (M * K) >> 3; }
__device__ __forceinline__ int64_t n_code_words(int64_t M, int64_t K) { return (M * K) >> 4; }
__device__ __forceinline__ int64_t n_scale_bytes(int64_t M, int64_t K) { return ((M + 127) >> 7) * (K >> 6) * 512; }

// Zero the scale bytes of the padding rows [M, ceil128(M)).
__device__ __forceinline__ void zero_pad_scale_rows(uint8_t* scales, int64_t M, int64_t kgroups, int* st) {
  const int64_t pad = ((M + 127) & ~int64_t(127)) - M;
  const int64_t total = pad * kgroups;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = M + i / kgroups, cg = i % kgroups;
    const int64_t off = scale_offset(row, cg * 4, kgroups);
    if (NVFP4_IN_BOUNDS(off + 3, n_scale_bytes(M, kgroups * 64), st))
      *reinterpret_cast<uint32_t*>(scales + off) = 0u;
  }
}

// ----------------------------------------------------------------------------
// Per-block operations. Each maps one lane's 16-element block (with the
// chunk it belongs to and the global scale) to the call's outputs.
// ----------------------------------------------------------------------------

// Quantize: codes, tiled block scales and (four_over_six) the choice map.
template <bool kFos>
struct QuantOp {
  static constexpr bool kBulkRefill = false;  // fused pass: phase 2 re-reads through registers
  uint2* codes;
  uint8_t* scales;
  uint8_t* choice;
  int64_t M, K;
  int* st;  // device status word (bounds-checking build)

  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    const float bmax = block_absmax(v);
    f32x2 xs[8];
    unpack_block(v, xs);
    Block b6;
    quantize_block_tab<false, kFos, false>(xs, bmax, b6);
    uint32_t sc = b6.sc, q0 = b6.q0, q1 = b6.q1, pick4 = 0;
    if (kFos) {
      Block b4;
      quantize_block_tab<false, true, true>(xs, bmax, b4);
      pick4 = b4.err < b6.err;  // tie keeps M = 6
      if (pick4) {
        sc = b4.sc;
        q0 = b4.q0;
        q1 = b4.q1;
      }
    }
    (void)lane;
    if (c.valid) {
      const int64_t off = block_scale_offset(c, K);
      if (NVFP4_IN_BOUNDS(c.vec >> 1, n_code_words(M, K), st)) codes[c.vec >> 1] = make_uint2(q0, q1);
      if (NVFP4_IN_BOUNDS(off, n_scale_bytes(M, K), st)) scales[off] = (uint8_t)sc;  // 4 lanes fill one 4-byte group
      if (kFos && choice && NVFP4_IN_BOUNDS(c.vec >> 1, n_code_words(M, K), st)) choice[c.vec >> 1] = (uint8_t)pick4;
    }
  }

  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }

  // Work independent of the values: zero padding-row scales; a max-mode call
  // that asked for a choice map gets zeros.
  __device__ __forceinline__ void finish() const {
    if (!kFos && choice) {
      const int64_t nb = (M * K) >> 4;
      for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb;
           i += (int64_t)gridDim.x * blockDim.x)
        choice[i] = 0;
    }
    zero_pad_scale_rows(scales, M, K >> 6, st);
  }
};

// Fake-quant with block scales computed from the values (max or four_over_six).
template <bool kFos>
struct FakeOp {
  static constexpr bool kBulkRefill = true;  // fused pass: phase 2 refills freed slots by bulk copies
  uint4* y;
  int64_t M, K;
  int* st;

  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    (void)lane;
    const float bmax = block_absmax(v);
    f32x2 xs[8];
    unpack_block(v, xs);
    Block b6;
    quantize_block_tab<true, kFos, false>(xs, bmax, b6);
    if (kFos) {
      Block b4;
      quantize_block_tab<true, true, true>(xs, bmax, b4);
      if (b4.err < b6.err) {
        store_bf16x16(y, c, b4.deq, n_vec16(M, K), st);
        return;
      }
    }
    store_bf16x16(y, c, b6.deq, n_vec16(M, K), st);
  }
  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }
  __device__ __forceinline__ void finish() const {}

  __device__ static __forceinline__ uint32_t to_bf16x2(f32x2 v) {
    float lo, hi;
    unpack2(v, lo, hi);
    return f32x2_to_bf16x2(lo, hi);
  }

  template <class C>
  __device__ static __forceinline__ void store_bf16x16(uint4* y, const C& c, const f32x2 (&out)[8], int64_t n_vec,
                                                       int* st) {
    (void)n_vec;
    (void)st;
    if (!c.valid || !NVFP4_IN_BOUNDS(c.vec + 1, n_vec, st)) return;
    const uint4 a = make_uint4(to_bf16x2(out[0]), to_bf16x2(out[1]), to_bf16x2(out[2]), to_bf16x2(out[3]));
    const uint4 b = make_uint4(to_bf16x2(out[4]), to_bf16x2(out[5]), to_bf16x2(out[6]), to_bf16x2(out[7]));
    // c.vec is even, so y + c.vec is 32-byte aligned when y is (the usual
    // case); a 16-byte aligned y takes two stores. One 32-byte store per
    // lane took the KV dequantize from 47.2 to 32.7 us.
    if ((reinterpret_cast<uintptr_t>(y) & 31u) == 0) {
      st_global_32b(y + c.vec, a, b);
    } else {
      y[c.vec] = a;
      y[c.vec + 1] = b;
    }
  }
};

// Fake-quant with frozen block scales s* (tiled layout) and frozen g*.
struct FrozenFakeOp {
  uint4* y;
  const uint8_t* scales_frozen;
  int64_t M, K;
  int* st;

  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    (void)lane;
    const int64_t off = block_scale_offset(c, K);
    const uint32_t sc = c.valid && NVFP4_IN_BOUNDS(off, n_scale_bytes(M, K), st) ? scales_frozen[off] : 1u;
    const float d = step_table().d[sc & 127u];
    const float r = step_table().r[sc & 127u];
    const f32x2 rr = pack2(r, r), dd = pack2(d, d);
    f32x2 sv[8], out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = mul2(bf16x2_unpack(v.w[i]), rr);
    e2m1_unpack4(e2m1_pack4(sv[0], sv[1], sv[2], sv[3]), out);
    e2m1_unpack4(e2m1_pack4(sv[4], sv[5], sv[6], sv[7]), out + 4);
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = mul2(dd, out[i]);
    FakeOp<false>::store_bf16x16(y, c, out, n_vec16(M, K), st);
  }
  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }
  __device__ __forceinline__ void finish() const {}
};

// QAD backward through the simulated quantization ("Developing Nemotron 3.5
// Lightning NVFP4 with QAD using NVIDIA Model Optimizer", Figure 2: the
// gradient returns to the FP weights through the fake-quant): a
// straight-through estimator clipped to the quantizer's range, grad_x =
// grad_y where |x * r| <= 6 for the block's forward r = RN(1/(g*s)), else 0.
__device__ __forceinline__ uint32_t ste_word(uint32_t gy, f32x2 xr) {
  float lo, hi;
  unpack2(xr, lo, hi);
  return gy & ((fabsf(lo) <= 6.0f ? 0x0000FFFFu : 0u) | (fabsf(hi) <= 6.0f ? 0xFFFF0000u : 0u));
}

template <class C>
__device__ __forceinline__ void ste_store(const uint4* gy, uint4* gx, const C& c, const f32x2 (&xs)[8],
                                          float r, int64_t n_vec, int* st) {
  (void)n_vec;
  (void)st;
  if (!c.valid || !NVFP4_IN_BOUNDS(c.vec + 1, n_vec, st)) return;
  const uint4 a = ld_stream(gy + c.vec), b = ld_stream(gy + c.vec + 1);
  const f32x2 rr = pack2(r, r);
  const uint4 lo = make_uint4(ste_word(a.x, mul2(xs[0], rr)), ste_word(a.y, mul2(xs[1], rr)),
                              ste_word(a.z, mul2(xs[2], rr)), ste_word(a.w, mul2(xs[3], rr)));
  const uint4 hi = make_uint4(ste_word(b.x, mul2(xs[4], rr)), ste_word(b.y, mul2(xs[5], rr)),
                              ste_word(b.z, mul2(xs[6], rr)), ste_word(b.w, mul2(xs[7], rr)));
  if ((reinterpret_cast<uintptr_t>(gx) & 31u) == 0) {  // as in FakeOp::store_bf16x16
    st_global_32b(gx + c.vec, lo, hi);
  } else {
    gx[c.vec] = lo;
    gx[c.vec + 1] = hi;
  }
}

// Backward with the forward's scales recomputed from x (max or four_over_six).
template <bool kFos>
struct SteOp {
  static constexpr bool kBulkRefill = true;
  const uint4* gy;
  uint4* gx;
  int64_t M, K;
  int* st;

  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }
  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    (void)lane;
    const float bmax = block_absmax(v);
    f32x2 xs[8];
    unpack_block(v, xs);
    uint32_t sc;
    if (kFos) {
      Block b6, b4;
      quantize_block_tab<false, true, false>(xs, bmax, b6);
      quantize_block_tab<false, true, true>(xs, bmax, b4);
      sc = b4.err < b6.err ? b4.sc : b6.sc;
    } else {
      sc = block_scale_code(bmax, g, 6.0f);
    }
    ste_store(gy, gx, c, xs, step_table().r[sc], n_vec16(M, K), st);
  }
  __device__ __forceinline__ void finish() const {}
};

// Backward with frozen block scales s* (tiled layout) and frozen g*.
struct FrozenSteOp {
  const uint4* gy;
  uint4* gx;
  const uint8_t* scales_frozen;
  int64_t M, K;
  int* st;

  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }
  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    (void)lane;
    const int64_t off = block_scale_offset(c, K);
    const uint32_t sc = c.valid && NVFP4_IN_BOUNDS(off, n_scale_bytes(M, K), st) ? scales_frozen[off] : 1u;
    f32x2 xs[8];
    unpack_block(v, xs);
    ste_store(gy, gx, c, xs, step_table().r[sc & 127u], n_vec16(M, K), st);
  }
  __device__ __forceinline__ void finish() const {}
};

// MSE calibration ("Developing Nemotron 3.5 Lightning NVFP4 with QAD using
// NVIDIA Model Optimizer", Table 1 "MSE"): every positive finite E4M3 code is
// a candidate block scale; the block keeps the lowest squared error, ties to
// the lowest code. Candidates run from code 126 down; the block's largest
// element alone costs (bmax - RN(6d))^2 once 6d < bmax (its code saturates at
// 6), which grows as d shrinks, so the search stops at the first candidate
// whose bound exceeds the best error (it cannot win or tie). d and 1/d per
// code are tabulated once per CTA.
struct MseOp {
  static constexpr bool kBulkRefill = false;
  uint2* codes;
  uint8_t* scales;
  uint8_t* choice;
  int64_t M, K;
  int* st;

  __device__ __forceinline__ void prepare(float g) const { build_step_table(g); }

  template <class C>
  __device__ __forceinline__ void operator()(const Raw16& v, const C& c, float g, int lane) const {
    (void)g;
    (void)lane;
    const StepTable& t = step_table();
    const float bmax = block_absmax(v);
    f32x2 xs[8];
    unpack_block(v, xs);
    Block b;
    encode_block<false, true>(xs, t.d[126], t.r[126], b);
    uint32_t best_sc = 126, q0 = b.q0, q1 = b.q1;
    float best = b.err;
    for (int code = 125; code >= 1; --code) {
      const float d = t.d[code];
      const float dm = __fmul_rn(d, 6.0f);
      if (dm < bmax) {
        const float df = __fsub_rn(bmax, dm);
        if (__fmul_rn(df, df) > best) break;
      }
      encode_block<false, true>(xs, d, t.r[code], b);
      if (b.err <= best) {  // ties move to the lower code
        best = b.err;
        best_sc = (uint32_t)code;
        q0 = b.q0;
        q1 = b.q1;
      }
    }
    if (c.valid) {
      const int64_t off = block_scale_offset(c, K);
      if (NVFP4_IN_BOUNDS(c.vec >> 1, n_code_words(M, K), st)) codes[c.vec >> 1] = make_uint2(q0, q1);
      if (NVFP4_IN_BOUNDS(off, n_scale_bytes(M, K), st)) scales[off] = (uint8_t)best_sc;
      if (choice && NVFP4_IN_BOUNDS(c.vec >> 1, n_code_words(M, K), st)) choice[c.vec >> 1] = 0;
    }
  }

  __device__ __forceinline__ void finish() const { zero_pad_scale_rows(scales, M, K >> 6, st); }
};

// ----------------------------------------------------------------------------
// Streaming pass with a known global scale (static g, or g reduced from the
// partials of a separate amax pass): grid-stride over 512-element chunks.
// ----------------------------------------------------------------------------
template <class Op, bool kNarrow>
__global__ void __launch_bounds__(kQThreads) stream_pass_kernel(const uint4* __restrict__ x, int64_t M, int64_t K,
                                                                 const uint32_t* __restrict__ partial, int n_partial,
                                                                 const float* __restrict__ g_static, Op op,
                                                                 float* __restrict__ g_out, int* status,
                                                                 uint64_t cpr_magic) {
  bool bad;
  const float g = resolve_global_scale(partial, n_partial, g_static, &bad);
  op.prepare(g);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (g_out) *g_out = g;
    if (bad) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
  }
  using Idx = typename std::conditional<kNarrow, uint32_t, int64_t>::type;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int32_t n_chunks = (int32_t)(M * cpr);  // < 2^31 (checked by the launcher)
  const int lane = threadIdx.x & 31;
  const int32_t warp = (int32_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
  const int32_t nwarps = (int32_t)gridDim.x * (kQThreads / 32);

  // kUnroll chunks per trip with all loads issued first (memory-level parallelism)
  for (int32_t ch0 = warp; ch0 < n_chunks; ch0 += kUnroll * nwarps) {
    Raw16 vv[kUnroll];
    ChunkT<Idx> cc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      cc[u] = chunk_at_t<Idx>(ch0 + u * nwarps, cpr, cpr_magic, K, lane);
      const bool live = cc[u].valid && ch0 + u * nwarps < n_chunks;
      load_raw16(x, cc[u].vec, live && NVFP4_IN_BOUNDS(cc[u].vec + 1, n_vec16(M, K), status), vv[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (ch0 + u * nwarps >= n_chunks) break;  // warp-uniform
      op(vv[u], cc[u], g, lane);
    }
  }
  op.finish();
}

// ----------------------------------------------------------------------------
// Fused dynamic pass: amax and quantization in one persistent launch.
//
// One CTA per SM (cooperative launch, so all CTAs are resident). CTA c owns a
// contiguous range of chunks. Phase 1 streams the range once, reducing the
// BF16 magnitude maximum and keeping the first kKeepChunks chunks (224 KB)
// in shared memory; chunk k of the range goes to slot k, owned by warp k % 32.
// The CTA maxima meet at a grid-wide barrier (a counter in the workspace that
// stays a multiple of the grid, so the workspace must be zero before its
// first use). Phase 2 then re-reads the range, in one of two ways chosen by
// the op (both read X from HBM about once in total):
//  * register re-reads (ops with little output: quantize, MSE): each warp
//    walks the range backwards, two chunks per trip; chunks that were not
//    kept -- read last in phase 1, so the most likely to still be in L2 --
//    come from global memory, the kept ones from shared memory;
//  * bulk refills (ops that write a BF16 tensor: fake-quant, STE): each warp
//    first processes its kept chunks, and every slot it frees is refilled at
//    once by one bulk copy (the TMA engine, completion on the slot's
//    mbarrier) of one of its not-kept chunks, newest first; kSlots chunks per
//    warp are then in flight while the warp computes and stores. Measured on
//    16384 x 4096: fake-quant 69.6 -> 63.5 us, STE 90.1 -> 81.9 us, while the
//    quantize ops were 2-4 us slower this way.
// ----------------------------------------------------------------------------
constexpr int kFusedThreads = 1024;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kSlots = 7;                              // kept / in-flight chunks per warp
constexpr int kKeepChunks = kSlots * 32;               // 1 KB of BF16 per chunk
constexpr int kFusedSmem = kKeepChunks * 1024 + kKeepChunks * 8;  // + one mbarrier per slot
constexpr int kFusedUnroll = 2;                        // register re-reads: chunks per trip
constexpr int kLoadUnroll = 4;                         // phase 1: chunk loads in flight per warp

// Grid-wide barrier on a 64-bit arrival counter that only grows: CTA arrival
// number `old` belongs to the barrier generation old / gridDim.x, which
// releases when the counter reaches the next multiple of gridDim.x. Every
// launch that uses a workspace has the same grid (one CTA per SM), so the
// counter stays a multiple of it between launches. Returns false if the wait
// ran out (the status is recorded by the caller).
__device__ __forceinline__ bool grid_barrier(unsigned long long* ctr, uint64_t timeout_ns) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();  // this CTA's partial maximum before its arrival
    const unsigned long long old = atomicAdd(ctr, 1ull);
    const unsigned long long target = (old / gridDim.x + 1) * gridDim.x;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      unsigned long long now;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(now) : "l"(ctr) : "memory");
      if ((long long)(now - target) >= 0) break;
      if (globaltimer_ns() - t0 > timeout_ns) {
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <class Op, bool kNarrow>
__global__ void __launch_bounds__(kFusedThreads, 1) fused_dynamic_kernel(const uint4* __restrict__ x, int64_t M,
                                                                           int64_t K, uint32_t* partial, uint32_t* bar,
                                                                           Op op, float* g_out, int* status,
                                                                           uint64_t timeout_ns, uint64_t cpr_magic) {
  extern __shared__ uint4 keep[];
  __shared__ uint32_t red[kFusedWarps];
  __shared__ float s_g;
  __shared__ int s_bad;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  using Idx = typename std::conditional<kNarrow, uint32_t, int64_t>::type;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int32_t n_chunks = (int32_t)(M * cpr);  // < 2^31 (checked by the launcher)
  const int32_t per = (int32_t)(((int64_t)n_chunks + gridDim.x - 1) / gridDim.x);
  const int32_t lo = (int32_t)min((int64_t)blockIdx.x * per, (int64_t)n_chunks);
  const int32_t hi = lo + per < n_chunks ? lo + per : n_chunks;
  const int32_t nkeep = hi - lo < kKeepChunks ? (hi - lo > 0 ? hi - lo : 0) : kKeepChunks;
  uint64_t* slot_bar = reinterpret_cast<uint64_t*>(keep + kKeepChunks * 64);
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kKeepChunks; ++i) mbar_init(&slot_bar[i], 1);
    s_abort = 0;
    fence_barrier_init();
  }

  // ---- phase 1: magnitude maximum, keep the first nkeep chunks
  uint32_t m2 = 0;
  for (int32_t base = lo + warp; base < hi; base += kLoadUnroll * kFusedWarps) {
    uint4 a[kLoadUnroll], b[kLoadUnroll];
#pragma unroll
    for (int u = 0; u < kLoadUnroll; ++u) {
      const int32_t ch = base + u * kFusedWarps;
      a[u] = b[u] = make_uint4(0, 0, 0, 0);
      if (ch < hi) {
        const ChunkT<Idx> c = chunk_at_t<Idx>(ch, cpr, cpr_magic, K, lane);
        if (c.valid && NVFP4_IN_BOUNDS(c.vec + 1, n_vec16(M, K), status)) {
          a[u] = ld_stream(x + c.vec);
          b[u] = ld_stream(x + c.vec + 1);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kLoadUnroll; ++u) {
      m2 = bmax2(m2, bmax2(bmax2(bmax2(a[u].x, a[u].y), bmax2(a[u].z, a[u].w)),
                           bmax2(bmax2(b[u].x, b[u].y), bmax2(b[u].z, b[u].w))));
      const int32_t k = base + u * kFusedWarps - lo;
      if (k < nkeep) {  // lane-contiguous halves: conflict-free 512-byte rows
        keep[k * 64 + lane] = a[u];
        keep[k * 64 + 32 + lane] = b[u];
      }
    }
  }
  uint32_t m = mag_max_halves(m2);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < kFusedWarps; ++w) r = max(r, red[w]);
    partial[blockIdx.x] = r;
  }

  // ---- grid-wide maximum -> global scale
  if (!grid_barrier(reinterpret_cast<unsigned long long*>(bar), timeout_ns) && threadIdx.x == 0) record_status(status, NVFP4_ERR_TIMEOUT);
  if (threadIdx.x < 32) {
    uint32_t mm = 0;
    for (int base = 0; base < (int)gridDim.x; base += 8 * 32) {
      uint32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * 32 + lane;
        v[u] = i < (int)gridDim.x ? __ldcg(partial + i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) mm = max(mm, v[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mm = max(mm, __shfl_xor_sync(kFull, mm, o));
    if (lane == 0) {
      s_g = global_scale_from_amax(__uint_as_float(mm << 16));
      s_bad = mm >= 0x7F80u;
    }
  }
  __syncthreads();
  const float g = s_g;
  op.prepare(g);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (g_out) *g_out = g;
    if (s_bad) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
  }

  grid_dependents_launch();  // a dependent GEMM may set up while phase 2 runs

  if constexpr (!Op::kBulkRefill) {
    // ---- phase 2, register re-reads: backwards, not-kept chunks from global
    // memory, then the kept ones
    for (int32_t top = hi - 1 - warp; top >= lo; top -= kFusedUnroll * kFusedWarps) {
      Raw16 vv[kFusedUnroll];
      ChunkT<Idx> cc[kFusedUnroll];
#pragma unroll
      for (int u = 0; u < kFusedUnroll; ++u) {
        const int32_t ch = top - u * kFusedWarps;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        cc[u] = chunk_at_t<Idx>(ch >= lo ? ch : lo, cpr, cpr_magic, K, lane);
        if (ch >= lo && cc[u].valid) {
          const int32_t k = ch - lo;
          if (k < nkeep) {
            a = keep[k * 64 + lane];
            b = keep[k * 64 + 32 + lane];
          } else if (NVFP4_IN_BOUNDS(cc[u].vec + 1, n_vec16(M, K), status)) {
            a = ld_stream(x + cc[u].vec);
            b = ld_stream(x + cc[u].vec + 1);
          }
        }
        vv[u].w[0] = a.x; vv[u].w[1] = a.y; vv[u].w[2] = a.z; vv[u].w[3] = a.w;
        vv[u].w[4] = b.x; vv[u].w[5] = b.y; vv[u].w[6] = b.z; vv[u].w[7] = b.w;
      }
#pragma unroll
      for (int u = 0; u < kFusedUnroll; ++u) {
        if (top - u * kFusedWarps < lo) break;  // warp-uniform
        op(vv[u], cc[u], g, lane);
      }
    }
  } else {
    // ---- phase 2: kept chunks first, then the not-kept ones through the freed
    // slots, each refilled by one bulk copy (1 KB, TMA engine) on the slot's
    // mbarrier as soon as its kept chunk has been quantized.
    const int32_t n = hi - lo;
    int32_t nx = n - 1 - warp;  // next not-kept chunk to fetch (relative to lo)
    uint32_t armed = 0, par = 0;  // per slot index t: a copy in flight; parity of its next completion
    const bool full_chunks = (K & 511) == 0;  // then chunk ch is the 1 KB at byte 1024 ch
    auto fetch_next = [&](int t) {
      if (nx < nkeep) return;
      const int32_t s = warp + t * kFusedWarps;
      Idx vec0;
      int64_t elems = 512;
      if (full_chunks) {
        vec0 = (Idx)(lo + nx) * (Idx)64;
      } else {
        const ChunkT<Idx> c0 = chunk_at_t<Idx>(lo + nx, cpr, cpr_magic, K, 0);
        vec0 = c0.vec;
        elems = K - c0.col < 512 ? K - c0.col : 512;
      }
      const uint32_t bytes = (uint32_t)elems * 2u;
      if (NVFP4_IN_BOUNDS(vec0 + (Idx)(elems / 8) - 1, n_vec16(M, K), status)) {
        __syncwarp();  // every lane has consumed the slot's previous contents
        if (lane == 0) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&slot_bar[s], bytes);
          bulk_load(&keep[s * 64], x + vec0, bytes, &slot_bar[s]);
        }
        armed |= 1u << t;
      }
      nx -= kFusedWarps;
    };
    {
      int t = 0;
      for (int32_t s = warp; s < nkeep; s += kFusedWarps, ++t) {
        const ChunkT<Idx> c = chunk_at_t<Idx>(lo + s, cpr, cpr_magic, K, lane);
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (c.valid) {
          a = keep[s * 64 + lane];
          b = keep[s * 64 + 32 + lane];
        }
        Raw16 v;
        v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
        v.w[4] = b.x; v.w[5] = b.y; v.w[6] = b.z; v.w[7] = b.w;
        op(v, c, g, lane);
        fetch_next(t);
      }
    }
    if (n > nkeep) {  // then nkeep == kKeepChunks: every warp owns kSlots slots
      int t = 0;
      bool ok = true;
      for (int32_t cur = n - 1 - warp; cur >= nkeep; cur -= kFusedWarps) {
        const int32_t s = warp + t * kFusedWarps;
        if ((armed >> t) & 1u) {
          if (!mbar_wait_warp(&slot_bar[s], (par >> t) & 1u, &s_abort, timeout_ns)) {
            ok = false;
            break;
          }
          par ^= 1u << t;
          armed &= ~(1u << t);
        }
        const ChunkT<Idx> c = chunk_at_t<Idx>(lo + cur, cpr, cpr_magic, K, lane);
        // the copy keeps global order (lane L's 32 bytes at 32 L); lanes 4-7 of
        // each group of 8 take their halves in the other order, so that each
        // 16-byte load instruction covers all 32 banks
        const uint8_t* sb = reinterpret_cast<const uint8_t*>(&keep[s * 64]) + lane * 32;
        const bool sw = (lane & 4) != 0;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (c.valid) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(sb + (sw ? 16 : 0));
          const uint4 u1 = *reinterpret_cast<const uint4*>(sb + (sw ? 0 : 16));
          a = sw ? u1 : u0;
          b = sw ? u0 : u1;
        }
        Raw16 v;
        v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
        v.w[4] = b.x; v.w[5] = b.y; v.w[6] = b.z; v.w[7] = b.w;
        op(v, c, g, lane);
        fetch_next(t);
        t = t + 1 == kSlots ? 0 : t + 1;
      }
      if (!ok) {
        if (lane == 0) record_status(status, NVFP4_ERR_TIMEOUT);
        // let the copies still in flight land (bounded) before the CTA exits
        for (int u = 0; u < kSlots; ++u) {
          if (!((armed >> u) & 1u)) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&slot_bar[warp + u * kFusedWarps], (par >> u) & 1u) &&
                 globaltimer_ns() - t0 < 1000000ull) {
          }
        }
      }
    }
  }
  op.finish();
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
  note_launch();
  amax_partial_kernel<<<n_partial, kAmaxThreads, 0, s>>>(static_cast<const uint4*>(x), n / 8, partial);
  return cudaGetLastError();
}

template <class Kern>
static int resident_blocks(Kern k, int threads, size_t smem) {
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, threads, smem) != cudaSuccess || b < 1) b = 0;
  return b;
}

template <class Op>
static cudaError_t launch_stream(const void* x, int64_t M, int64_t K, const uint32_t* partial, int n_partial,
                                 const float* g_static, const Op& op, float* g_out, int* status, int num_sms,
                                 cudaStream_t s) {
  const int64_t chunks = M * ((K + 511) / 512);
  if (chunks >= (int64_t(1) << 30)) return cudaErrorInvalidValue;  // 32-bit chunk loops
  static const int occ = resident_blocks(stream_pass_kernel<Op, false>, kQThreads, 0);
  const int grid = grid_for(chunks, kQThreads / 32 * kUnroll, num_sms * (occ > 0 ? occ : 1));
  note_launch();
  if (narrow_chunks(M, K))
    stream_pass_kernel<Op, true><<<grid, kQThreads, 0, s>>>(static_cast<const uint4*>(x), M, K, partial, n_partial,
                                                            g_static, op, g_out, status, chunk_magic_narrow(K));
  else
    stream_pass_kernel<Op, false><<<grid, kQThreads, 0, s>>>(static_cast<const uint4*>(x), M, K, partial, n_partial,
                                                             g_static, op, g_out, status, chunk_magic(K));
  return cudaGetLastError();
}

// Fused dynamic launch; returns cudaErrorNotSupported when a cooperative
// launch of one CTA per SM is not possible (the caller then runs two passes).
template <class Op>
static cudaError_t launch_fused(const void* x, int64_t M, int64_t K, uint32_t* ws, const Op& op, float* g_out,
                                int* status, int num_sms, cudaStream_t s) {
  const int64_t chunks = M * ((K + 511) / 512);
  if (chunks >= (int64_t(1) << 30)) return cudaErrorInvalidValue;  // 32-bit chunk loops
  const bool narrow = narrow_chunks(M, K);
  const void* kern = narrow ? (const void*)fused_dynamic_kernel<Op, true> : (const void*)fused_dynamic_kernel<Op, false>;
  static cudaError_t attr_n = cudaFuncSetAttribute(fused_dynamic_kernel<Op, true>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
  static cudaError_t attr_w = cudaFuncSetAttribute(fused_dynamic_kernel<Op, false>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
  static const int occ_n =
      attr_n == cudaSuccess ? resident_blocks(fused_dynamic_kernel<Op, true>, kFusedThreads, kFusedSmem) : 0;
  static const int occ_w =
      attr_w == cudaSuccess ? resident_blocks(fused_dynamic_kernel<Op, false>, kFusedThreads, kFusedSmem) : 0;
  if ((narrow ? occ_n : occ_w) < 1 || num_sms > kMaxPartials) return cudaErrorNotSupported;
  const uint4* xv = static_cast<const uint4*>(x);
  uint32_t* partial = ws;
  uint32_t* bar = ws + kMaxPartials;
  uint64_t timeout_ns = kFusedTimeoutNs;
  uint64_t magic = narrow ? chunk_magic_narrow(K) : chunk_magic(K);
  void* args[] = {(void*)&xv, (void*)&M, (void*)&K, (void*)&partial, (void*)&bar, (void*)&op, (void*)&g_out,
                  (void*)&status, (void*)&timeout_ns, (void*)&magic};
  note_launch();
  const cudaError_t e = cudaLaunchCooperativeKernel(kern, dim3(num_sms),
                                                    dim3(kFusedThreads), args, kFusedSmem, s);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return cudaErrorNotSupported;
  }
  return e;
}

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, int mode, const uint32_t* partial,
                            int n_partial, const float* g_static, uint8_t* codes, uint8_t* scales,
                            float* g_out, uint8_t* choice, int* status, int num_sms, cudaStream_t s) {
  uint2* c = reinterpret_cast<uint2*>(codes);
  if (mode == 2)
    return launch_stream(x, M, K, partial, n_partial, g_static, MseOp{c, scales, choice, M, K, status}, g_out, status,
                         num_sms, s);
  if (mode == 1)
    return launch_stream(x, M, K, partial, n_partial, g_static, QuantOp<true>{c, scales, choice, M, K, status}, g_out, status,
                         num_sms, s);
  return launch_stream(x, M, K, partial, n_partial, g_static, QuantOp<false>{c, scales, choice, M, K, status}, g_out, status,
                       num_sms, s);
}

cudaError_t launch_fake_quant(const void* x, int64_t M, int64_t K, bool fos, const uint32_t* partial,
                              int n_partial, const float* g_static, const uint8_t* scales_frozen,
                              void* y, int* status, int num_sms, cudaStream_t s) {
  uint4* yv = static_cast<uint4*>(y);
  if (scales_frozen)
    return launch_stream(x, M, K, partial, n_partial, g_static, FrozenFakeOp{yv, scales_frozen, M, K, status}, nullptr,
                         status, num_sms, s);
  if (fos)
    return launch_stream(x, M, K, partial, n_partial, g_static, FakeOp<true>{yv, M, K, status}, nullptr, status, num_sms, s);
  return launch_stream(x, M, K, partial, n_partial, g_static, FakeOp<false>{yv, M, K, status}, nullptr, status, num_sms, s);
}

cudaError_t launch_quantize_fused(const void* x, int64_t M, int64_t K, int mode, uint32_t* ws, uint8_t* codes,
                                  uint8_t* scales, float* g_out, uint8_t* choice, int* status, int num_sms,
                                  cudaStream_t s) {
  uint2* c = reinterpret_cast<uint2*>(codes);
  if (mode == 2) return launch_fused(x, M, K, ws, MseOp{c, scales, choice, M, K, status}, g_out, status, num_sms, s);
  if (mode == 1) return launch_fused(x, M, K, ws, QuantOp<true>{c, scales, choice, M, K, status}, g_out, status, num_sms, s);
  return launch_fused(x, M, K, ws, QuantOp<false>{c, scales, choice, M, K, status}, g_out, status, num_sms, s);
}

cudaError_t launch_fake_quant_fused(const void* x, int64_t M, int64_t K, bool fos, uint32_t* ws, void* y,
                                    int* status, int num_sms, cudaStream_t s) {
  uint4* yv = static_cast<uint4*>(y);
  if (fos) return launch_fused(x, M, K, ws, FakeOp<true>{yv, M, K, status}, nullptr, status, num_sms, s);
  return launch_fused(x, M, K, ws, FakeOp<false>{yv, M, K, status}, nullptr, status, num_sms, s);
}

cudaError_t launch_convert(const float* in, int64_t n, uint8_t* out, bool e4m3, int num_sms,
                           cudaStream_t s) {
  const int grid = grid_for(n, 256, num_sms * 8);
  note_launch();
  if (e4m3)
    convert_e4m3_kernel<<<grid, 256, 0, s>>>(in, n, out);
  else
    convert_e2m1_kernel<<<grid, 256, 0, s>>>(in, n, out);
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint64_t timeout_ns, int* status, cudaStream_t s) {
  note_launch();
  selftest_timeout_kernel<<<1, 32, 0, s>>>(timeout_ns, status);
  return cudaGetLastError();
}

cudaError_t launch_fake_quant_bwd(const void* x, const void* gy, int64_t M, int64_t K, bool fos,
                                  const uint32_t* partial, int n_partial, const float* g_static,
                                  const uint8_t* scales_frozen, void* gx, int* status, int num_sms, cudaStream_t s) {
  const uint4* gyv = static_cast<const uint4*>(gy);
  uint4* gxv = static_cast<uint4*>(gx);
  if (scales_frozen)
    return launch_stream(x, M, K, partial, n_partial, g_static, FrozenSteOp{gyv, gxv, scales_frozen, M, K, status}, nullptr,
                         status, num_sms, s);
  if (fos)
    return launch_stream(x, M, K, partial, n_partial, g_static, SteOp<true>{gyv, gxv, M, K, status}, nullptr, status,
                         num_sms, s);
  return launch_stream(x, M, K, partial, n_partial, g_static, SteOp<false>{gyv, gxv, M, K, status}, nullptr, status, num_sms,
                       s);
}

cudaError_t launch_fake_quant_bwd_fused(const void* x, const void* gy, int64_t M, int64_t K, bool fos, uint32_t* ws,
                                        void* gx, int* status, int num_sms, cudaStream_t s) {
  const uint4* gyv = static_cast<const uint4*>(gy);
  uint4* gxv = static_cast<uint4*>(gx);
  if (fos) return launch_fused(x, M, K, ws, SteOp<true>{gyv, gxv, M, K, status}, nullptr, status, num_sms, s);
  return launch_fused(x, M, K, ws, SteOp<false>{gyv, gxv, M, K, status}, nullptr, status, num_sms, s);
}

// ----------------------------------------------------------------------------
// Dequantize: y = BF16(g * s * q) from stored codes and tiled scales -- the
// read side of an NVFP4 KV cache ("Developing Nemotron 3.5 Lightning NVFP4
// with QAD using NVIDIA Model Optimizer", Table 1 "four_over_six + NVFP4 KV":
// K and V stored in NVFP4, QK^T kept in BF16). Same products as fake-quant
// (d = g*s, then d*q, FP32), so dequantize(quantize(x)) == fake_quant(x).
// ----------------------------------------------------------------------------
template <bool kNarrow>
__global__ void __launch_bounds__(kQThreads) dequantize_kernel(const uint2* __restrict__ codes,
                                                                const uint8_t* __restrict__ scales,
                                                                const float* __restrict__ g_ptr, int64_t M,
                                                                int64_t K, uint64_t cpr_magic, uint4* __restrict__ y,
                                                                int* status) {
  using Idx = typename std::conditional<kNarrow, uint32_t, int64_t>::type;
  const float g = *g_ptr;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int32_t n_chunks = (int32_t)(M * cpr);  // < 2^31 (checked by the launcher)
  const int lane = threadIdx.x & 31;
  const int32_t warp = (int32_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
  const int32_t nwarps = (int32_t)gridDim.x * (kQThreads / 32);
  for (int32_t ch0 = warp; ch0 < n_chunks; ch0 += kUnroll * nwarps) {
    ChunkT<Idx> cc[kUnroll];
    uint2 q[kUnroll];
    uint32_t sc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int32_t ch = ch0 + u * nwarps;
      cc[u] = chunk_at_t<Idx>(ch < n_chunks ? ch : 0, cpr, cpr_magic, K, lane);
      const bool ok = ch < n_chunks && cc[u].valid;
      const int64_t off = block_scale_offset(cc[u], K);
      q[u] = ok && NVFP4_IN_BOUNDS(cc[u].vec >> 1, n_code_words(M, K), status) ? codes[cc[u].vec >> 1]
                                                                                : make_uint2(0, 0);
      sc[u] = ok && NVFP4_IN_BOUNDS(off, n_scale_bytes(M, K), status) ? scales[off] : 1u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (ch0 + u * nwarps >= n_chunks) break;  // warp-uniform
      const float d = __fmul_rn(g, scale_value(sc[u]));
      const f32x2 dd = pack2(d, d);
      f32x2 v[8];
      e2m1_unpack4(q[u].x, v);
      e2m1_unpack4(q[u].y, v + 4);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = mul2(dd, v[i]);
      FakeOp<false>::store_bf16x16(y, cc[u], v, n_vec16(M, K), status);
    }
  }
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t M, int64_t K,
                              void* y, int* status, int num_sms, cudaStream_t s) {
  const int64_t chunks = M * ((K + 511) / 512);
  if (chunks == 0) return cudaSuccess;
  if (chunks >= (int64_t(1) << 30)) return cudaErrorInvalidValue;  // 32-bit chunk loops
  static const int occ = resident_blocks(dequantize_kernel<false>, kQThreads, 0);
  const int grid = grid_for(chunks, kQThreads / 32 * kUnroll, num_sms * (occ > 0 ? occ : 1));
  note_launch();
  if (narrow_chunks(M, K))
    dequantize_kernel<true><<<grid, kQThreads, 0, s>>>(reinterpret_cast<const uint2*>(codes), scales, g, M, K,
                                                       chunk_magic_narrow(K), static_cast<uint4*>(y), status);
  else
    dequantize_kernel<false><<<grid, kQThreads, 0, s>>>(reinterpret_cast<const uint2*>(codes), scales, g, M, K,
                                                        chunk_magic(K), static_cast<uint4*>(y), status);
  return cudaGetLastError();
}

}  // namespace nvfp4
