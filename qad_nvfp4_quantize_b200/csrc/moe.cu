// Routed-expert (MoE) layer in NVFP4 W4A4.
//
// The routed experts are the tensors the pages quantize first: 99.2% of the
// quantized tensors in "2. PTQ" of "Model-Optimizer in practice: recovering
// Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD" (fused gate/up and down
// projections), and the only ones in "How is Qwen3.8-Flash-Next-NVFP4's NVFP4
// quantization done?" (top-k routing, dynamic activation quantization,
// section "the A4 side: dynamic activations").
//
// Pipeline (all on the caller's stream, no host synchronisation):
//   1 route      stable counting sort of the T*topk (token, slot) pairs by
//                expert; expert segments padded to 128 rows; per-m-tile
//                expert table; per-expert amax slots zeroed.
//   2 token pass per token: row amax -> per-expert amax (atomicMax over the
//                experts it is routed to); zero the output row.
//   3 gather+quantize  each padded row gets its token's x quantized with its
//                expert's dynamic global scale (pad rows: zero codes/scales).
//   4 gate_up    grouped tcgen05 GEMM; a tile holds 128 gate and the matching
//                128 up columns; epilogue h = SiLU(gate)*up -> BF16, plus the
//                per-expert amax of h.
//   5 quantize h per expert, dynamic global scale.
//   6 down       grouped tcgen05 GEMM; epilogue scales by the routing weight
//                and adds into out[token] in FP32 (vector atomics).
#include <mutex>

#include <type_traits>

#include "block_math.cuh"
#include "gemm_kernel.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr unsigned kFullMask = 0xFFFFFFFFu;

int64_t align256(int64_t v) { return (v + 255) & ~int64_t(255); }

int64_t scale_bytes_(int64_t rows, int64_t K) { return ((rows + 127) / 128) * (K / 64) * 512; }

}  // namespace

constexpr int kRouteCtasMax = 128;  // routing CTAs (each owns a contiguous pair range)

// Workspace layout (all regions 256-byte aligned).
struct MoeLayout {
  int64_t R, P;
  int64_t counts, offsets, cursor, row_pair, tile_expert, tile_count, amax_x, amax_h, cta_count, cta_base;
  int64_t xq_codes, xq_scales, xq_g, h, hq_codes, hq_scales, hq_g, total;
};

int64_t moe_rows_capacity(int64_t T, int topk, int E) {
  const int64_t P = T * topk;
  return ((P + (int64_t)E * 127 + 127) / 128) * 128;
}

static MoeLayout moe_layout(int64_t T, int64_t H, int64_t I, int E, int topk) {
  MoeLayout L;
  L.P = T * topk;
  L.R = moe_rows_capacity(T, topk, E);
  int64_t o = 0;
  auto take = [&o](int64_t bytes) {
    const int64_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.counts = take(4 * (int64_t)E);
  L.offsets = take(4 * ((int64_t)E + 1));
  L.cursor = take(4 * (int64_t)E);
  L.row_pair = take(4 * L.R);
  L.tile_expert = take(4 * (L.R / 128));
  L.tile_count = take(4);
  L.amax_x = take(4 * (int64_t)E);
  L.amax_h = take(4 * (int64_t)E);
  L.cta_count = take(4 * (int64_t)kRouteCtasMax * E);
  L.cta_base = take(4 * (int64_t)kRouteCtasMax * E);
  L.xq_codes = take(L.R * H / 2);
  L.xq_scales = take(scale_bytes_(L.R, H));
  L.xq_g = take(4 * (int64_t)E);
  L.h = take(L.R * I * 2);
  L.hq_codes = take(L.R * I / 2);
  L.hq_scales = take(scale_bytes_(L.R, I));
  L.hq_g = take(4 * (int64_t)E);
  L.total = o;
  return L;
}

// ----------------------------------------------------------------------------
// 1. Routing: a stable counting sort of the P = T*topk pairs by expert, in
// three launches. G routing CTAs each own the contiguous pair range
// [c*P/G, (c+1)*P/G).
//   count  per-CTA expert histograms -> cta_count[c][e]
//   scan   one CTA: per expert, exclusive prefix over CTAs -> cta_base[c][e],
//          totals -> counts, 128-padded segment offsets, m-tile -> expert
//          table, pad rows of row_pair = -1, per-expert amax slots zeroed
//   place  each CTA ranks its pairs again: per-warp histograms give each
//          warp its base inside every expert segment, and within a warp pairs
//          are ranked with __match_any_sync, so the order inside an expert is
//          increasing pair index (stable).
// ----------------------------------------------------------------------------
constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

__device__ __forceinline__ void route_range(int64_t P, int G, int c, int64_t& lo, int64_t& hi) {
  lo = P * c / G;
  hi = P * (c + 1) / G;
}

__global__ void __launch_bounds__(kRouteThreads) moe_route_count_kernel(const int32_t* __restrict__ topk_ids,
                                                                         int64_t P, int E,
                                                                         int32_t* __restrict__ cta_count,
                                                                         int* status) {
  extern __shared__ int32_t hist[];  // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  int64_t lo, hi;
  route_range(P, gridDim.x, blockIdx.x, lo, hi);
  bool bad = false;
  for (int64_t p = lo + threadIdx.x; p < hi; p += blockDim.x) {
    const int e = topk_ids[p];
    if (e < 0 || e >= E) {
      bad = true;
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  if (bad) record_status(status, NVFP4_ERR_INVALID_ARG);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cta_count[(int64_t)blockIdx.x * E + e] = hist[e];
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads, 1) moe_route_scan_kernel(
    const int32_t* __restrict__ cta_count, int G, int E, int32_t* __restrict__ cta_base,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ row_pair,
    int32_t* __restrict__ tile_expert, int32_t* __restrict__ tile_count, uint32_t* __restrict__ amax_x,
    uint32_t* __restrict__ amax_h) {
  __shared__ int32_t seg[kScanThreads + 1];   // padded segment sizes, then offsets
  __shared__ int32_t wsum[kScanThreads / 32];
  const int e = threadIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t total = 0;
  if (e < E) {
    for (int c0 = 0; c0 < G; c0 += 8) {  // eight independent loads in flight
      int32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c0 + u < G ? cta_count[(int64_t)(c0 + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (c0 + u < G) cta_base[(int64_t)(c0 + u) * E + e] = total;
        total += v[u];
      }
    }
    counts[e] = total;
    amax_x[e] = 0u;
    amax_h[e] = 0u;
  }
  const int32_t padded = e < E ? (total + 127) & ~127 : 0;
  // exclusive scan of padded sizes over experts (thread e = expert e)
  int32_t incl = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += v;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int32_t excl = incl - padded + (warp > 0 ? wsum[warp - 1] : 0);
  if (e < E) {
    offsets[e] = excl;
    for (int32_t t = excl / 128; t < (excl + padded) / 128; ++t) tile_expert[t] = e;
    for (int32_t r = excl + total; r < excl + padded; ++r) row_pair[r] = -1;  // pad rows
  }
  if (e == E - 1) {
    offsets[E] = excl + padded;
    *tile_count = (excl + padded) / 128;
  }
}

__global__ void __launch_bounds__(kRouteThreads) moe_route_place_kernel(const int32_t* __restrict__ topk_ids,
                                                                         int64_t P, int E,
                                                                         const int32_t* __restrict__ cta_base,
                                                                         const int32_t* __restrict__ offsets,
                                                                         int32_t* __restrict__ row_pair) {
  extern __shared__ int32_t wcount[];  // [kRouteWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kRouteWarps * E; i += blockDim.x) wcount[i] = 0;
  __syncthreads();
  int64_t lo, hi;
  route_range(P, gridDim.x, blockIdx.x, lo, hi);
  const int64_t wlo = lo + (hi - lo) * warp / kRouteWarps, whi = lo + (hi - lo) * (warp + 1) / kRouteWarps;
  for (int64_t p = wlo + lane; p < whi; p += 32) {
    const int e = topk_ids[p];
    if (e >= 0 && e < E) atomicAdd(&wcount[warp * E + e], 1);
  }
  __syncthreads();
  // per expert: segment offset + this CTA's base + exclusive prefix over warps
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = offsets[e] + cta_base[(int64_t)blockIdx.x * E + e];
    for (int w = 0; w < kRouteWarps; ++w) {
      const int32_t c = wcount[w * E + e];
      wcount[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t base = wlo; base < whi; base += 32) {
    const int64_t p = base + lane;
    int e = p < whi ? topk_ids[p] : -1;
    if (e >= E) e = -1;
    const unsigned same = __match_any_sync(kFullMask, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    const int leader = __ffs(same) - 1;
    if (e >= 0) row_pair[wcount[warp * E + e] + rank] = (int32_t)p;
    __syncwarp();
    if (e >= 0 && lane == leader) wcount[warp * E + e] += __popc(same);
    __syncwarp();
  }
}

// ----------------------------------------------------------------------------
// 2. Token pass: row amax of x[t] -> atomicMax into the amax of every expert
// the token is routed to; zero out[t]. One warp per token.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) moe_token_pass_kernel(const uint4* __restrict__ x, int64_t T, int64_t H,
                                                              const int32_t* __restrict__ topk_ids, int topk,
                                                              int E, uint32_t* __restrict__ amax_x,
                                                              float4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nw) {
    const uint4* row = x + t * (H / 8);
    uint32_t m2 = 0;
    for (int64_t i = lane; i < H / 8; i += 32) {
      const uint4 v = row[i];
      m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v.w & 0x7FFF7FFFu);
    }
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));
    if (lane < topk) {
      const int e = topk_ids[t * topk + lane];
      if (e >= 0 && e < E) atomicMax(&amax_x[e], m);
    }
    float4* orow = out + t * (H / 4);
    for (int64_t i = lane; i < H / 4; i += 32) orow[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ----------------------------------------------------------------------------
// 3 / 5. Row-gathered quantization with a per-expert dynamic global scale.
// A warp's unit is a 512-element chunk of one padded row, one 16-element
// block per lane (block_math.cuh). Each trip takes kRowUnroll chunks: first
// their row lookups, then all their (gathered) loads, then the arithmetic, so
// several chunks' loads are in flight together. Source row of padded row p:
// kGather ? x[row_pair[p] / topk] : src[p]; pad rows get zero codes and
// scales. amax_bits[e] is the BF16 magnitude (kGather) or the FP32 bits (h)
// of expert e's amax; every CTA turns them into global scales in shared
// memory once.
// ----------------------------------------------------------------------------
constexpr int kRowThreads = 256;
constexpr int kRowUnroll = 4;

template <bool kGather, bool kNarrow>
__global__ void __launch_bounds__(kRowThreads) moe_quantize_rows_kernel(
    const uint4* __restrict__ src, int64_t K, int topk, const int32_t* __restrict__ row_pair,
    const int32_t* __restrict__ tile_expert, const int32_t* __restrict__ tile_count,
    const uint32_t* __restrict__ amax_bits, int E, uint2* __restrict__ codes, uint8_t* __restrict__ scales,
    float* __restrict__ g_out, int* status, uint64_t cpr_magic) {
  extern __shared__ float g_s[];  // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const uint32_t a = amax_bits[e];
    const float amax = kGather ? __uint_as_float(a << 16) : __uint_as_float(a);
    const float g = global_scale_from_amax(amax);
    g_s[e] = g;
    if (blockIdx.x == 0) {
      g_out[e] = g;
      if (kGather ? a >= 0x7F80u : !(amax <= 3.0e38f)) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
    }
  }
  __syncthreads();
  using Idx = typename std::conditional<kNarrow, uint32_t, int64_t>::type;
  const int lane = threadIdx.x & 31;
  const int32_t rows = (*tile_count) * 128;
  const int32_t cpr = (int32_t)((K + 511) >> 9);
  const int32_t n_chunks = rows * cpr;  // < 2^30 (the launcher bounds the padded rows)
  const int32_t warp = (int32_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
  const int32_t nwarps = (int32_t)gridDim.x * (kRowThreads / 32);
  for (int32_t ch0 = warp; ch0 < n_chunks; ch0 += kRowUnroll * nwarps) {
    ChunkT<Idx> cc[kRowUnroll];
    int32_t pr[kRowUnroll], ex[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int32_t ch = ch0 + u * nwarps;
      cc[u] = chunk_at_t<Idx>(ch < n_chunks ? ch : 0, cpr, cpr_magic, K, lane);
      pr[u] = ch < n_chunks ? row_pair[cc[u].row] : -1;
      ex[u] = ch < n_chunks ? tile_expert[cc[u].row >> 7] : 0;
    }
    Raw16 vv[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const Idx srow = kGather ? (Idx)(pr[u] >= 0 ? pr[u] / topk : 0) : cc[u].row;
      load_raw16(src, (srow * (Idx)K + (Idx)cc[u].col) >> 3, pr[u] >= 0 && cc[u].valid, vv[u]);
    }
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      if (ch0 + u * nwarps >= n_chunks) break;  // warp-uniform
      Block b;
      if (pr[u] >= 0) {
        quantize_block<false, false>(vv[u], block_absmax(vv[u]), g_s[ex[u]], 6.0f, b);
      } else {
        b.sc = b.q0 = b.q1 = 0u;  // pad row: zero codes and scales, no arithmetic
      }
      if (cc[u].valid) {
        codes[cc[u].vec >> 1] = make_uint2(b.q0, b.q1);
        scales[block_scale_offset(cc[u], K)] = (uint8_t)b.sc;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// 4. gate_up grouped GEMM problem. Tiles are n-fastest: the I/128 column tiles
// of one m-tile run on neighbouring CTAs (A read once), and the m-tiles of an
// expert are adjacent (its weight tiles are re-read from L2).
// ----------------------------------------------------------------------------
struct GateUpProblem {
  static constexpr int kPipeStages = 4;
  static constexpr uint32_t kEpiWarpBytes = 0;  // direct stores
  int K;             // H
  int I;
  int n_tiles;       // I / 128
  int kgroups;       // H / 64
  int64_t sf_expert_bytes;
  const int32_t* tile_count;
  const int32_t* tile_expert;
  const uint8_t* sfa;      // xq scales
  const uint8_t* sfb;      // w13 scales
  const float* ga;         // xq_g [E]
  const float* gb;         // w13_g [E]
  __nv_bfloat16* h;        // [R][I]
  uint32_t* amax_h;

  __device__ __forceinline__ int num_tiles() const { return (*tile_count) * n_tiles; }

  __device__ __forceinline__ TileJob job(int t) const {
    const int mt = t / n_tiles, nt = t - mt * n_tiles;
    const int e = tile_expert[mt];
    const size_t rt = (size_t)kgroups * kSFAtom;
    TileJob j;
    j.a_row = mt * 128;
    j.b_row0 = e * 2 * I + nt * 128;
    j.b_row1 = e * 2 * I + I + nt * 128;
    j.sfa = sfa + (size_t)mt * rt;
    const uint8_t* sfe = sfb + (size_t)e * sf_expert_bytes;
    j.sfb0 = sfe + (size_t)nt * rt;
    j.sfb1 = sfe + (size_t)(I / 128 + nt) * rt;
    j.expert = e;
    j.m0 = mt * 128;
    j.n0 = nt * 128;
    return j;
  }

  // gate columns [h*64, h*64+64) and the matching up columns 128 later
  __device__ static constexpr uint32_t tmem_col(int h, int j) {
    return (uint32_t)(j < 2 ? h * 64 + 32 * j : 128 + h * 64 + 32 * (j - 2));
  }

  __device__ __forceinline__ void store(const TileJob& job, int q, int hh, int lane,
                                        const uint32_t (&acc)[4][32], uint8_t*, const CUtensorMap*) const {
    const int row = job.m0 + q * 32 + lane;
    const float alpha = __fmul_rn(ga[job.expert], gb[job.expert]);
    __nv_bfloat16* hrow = h + (size_t)row * I + job.n0 + hh * 64;
    uint32_t mx = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
        uint32_t packed[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float hv[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float z = __fmul_rn(__uint_as_float(acc[j][c + 2 * u + k]), alpha);
            const float up = __fmul_rn(__uint_as_float(acc[j + 2][c + 2 * u + k]), alpha);
            // hardware exp2-based exp and approximate division: relative error
            // ~1e-6, far below the BF16 rounding of h that follows
            const float silu = __fdividef(z, __fadd_rn(1.0f, __expf(-z)));
            hv[k] = __fmul_rn(silu, up);
          }
          packed[u] = f32x2_to_bf16x2(hv[0], hv[1]);
          mx = __vmaxu2(mx, packed[u] & 0x7FFF7FFFu);
        }
        *reinterpret_cast<uint4*>(hrow + 32 * j + c) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    }
    uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));
    if (lane == 0) atomicMax(&amax_h[job.expert], m << 16);  // FP32 bits of the BF16 amax
  }
};

// ----------------------------------------------------------------------------
// 6. down grouped GEMM problem: out[token] += w * (g_h * g_w2) * acc.
// The rows of a tile belong to different tokens, so the sum over a token's
// experts is a reduction into out. Each epilogue lane stages 32 FP32 values
// of its row (128 bytes, rows 144 bytes apart so the 32 lanes' writes fall on
// distinct banks) and adds them into out with one bulk reduction
// (cp.reduce.async.bulk .add.f32: element-wise atomic adds done by the memory
// system), 1024 per tile instead of 8192 vector atomics.
// ----------------------------------------------------------------------------
constexpr uint32_t kDownRowStride = 144;  // staged row pitch (128 bytes of data)

struct DownProblem {
  static constexpr int kPipeStages = 3;    // K = I is short: 3 stages cover 1.5 tiles
  static constexpr uint32_t kEpiWarpBytes = 32 * kDownRowStride;
  int K;             // I
  int H;
  int n_tiles;       // ceil(H / 256)
  int kgroups;       // I / 64
  int topk;
  int64_t sf_expert_bytes;
  const int32_t* tile_count;
  const int32_t* tile_expert;
  const int32_t* row_pair;
  const float* topk_w;
  const uint8_t* sfa;      // hq scales
  const uint8_t* sfb;      // w2 scales
  const float* ga;         // hq_g [E]
  const float* gb;         // w2_g [E]
  float* out;

  __device__ __forceinline__ int num_tiles() const { return (*tile_count) * n_tiles; }

  __device__ __forceinline__ TileJob job(int t) const {
    const int mt = t / n_tiles, nt = t - mt * n_tiles;
    const int e = tile_expert[mt];
    const size_t rt = (size_t)kgroups * kSFAtom;
    TileJob j;
    j.a_row = mt * 128;
    j.b_row0 = e * H + nt * 256;
    j.b_row1 = e * H + nt * 256 + 128;
    j.sfa = sfa + (size_t)mt * rt;
    const uint8_t* sfe = sfb + (size_t)e * sf_expert_bytes;
    j.sfb0 = sfe + (size_t)(2 * nt) * rt;
    j.sfb1 = (nt * 256 + 128 < H) ? sfe + (size_t)(2 * nt + 1) * rt : nullptr;
    j.expert = e;
    j.m0 = mt * 128;
    j.n0 = nt * 256;
    return j;
  }

  __device__ static constexpr uint32_t tmem_col(int h, int j) { return (uint32_t)(h * 128 + 32 * j); }

  __device__ __forceinline__ void store(const TileJob& job, int q, int hh, int lane,
                                        const uint32_t (&acc)[4][32], uint8_t* stg, const CUtensorMap*) const {
    const int row = job.m0 + q * 32 + lane;
    const int32_t pair = row_pair[row];
    const float alpha = __fmul_rn(ga[job.expert], gb[job.expert]);
    const float w = pair >= 0 ? topk_w[pair] : 0.0f;
    float* orow = out + (size_t)(pair >= 0 ? pair / topk : 0) * H;
    const uint32_t srow = smem_u32(stg) + lane * kDownRowStride;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = job.n0 + hh * 128 + 32 * j;
      if (n >= H) break;
      bulk_wait_read_all();  // this lane's previous row segment has left shared memory
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        uint4 v;
        v.x = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 0]), alpha), w));
        v.y = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 1]), alpha), w));
        v.z = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 2]), alpha), w));
        v.w = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 3]), alpha), w));
        st_shared_v4(srow + c * 4, v);
      }
      fence_proxy_async_smem();
      if (pair >= 0) {
        bulk_reduce_add_f32(orow + n, srow, 128);
        bulk_commit_group();
      }
    }
  }
};

template <class Prob>
static cudaError_t prepare_moe_kernel() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(nvf4_gemm_kernel<Prob>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)gemm_smem_bytes<Prob>());
  });
  return err;
}

constexpr uint64_t kMoeTimeoutNs = 2000000000ull;

cudaError_t launch_moe(const MoeArgs& a, int* status, int num_sms, cudaStream_t s) {
  const MoeLayout L = moe_layout(a.T, a.H, a.I, a.E, a.topk);
  uint8_t* ws = a.ws;
  auto I32 = [ws](int64_t off) { return reinterpret_cast<int32_t*>(ws + off); };
  auto U32 = [ws](int64_t off) { return reinterpret_cast<uint32_t*>(ws + off); };
  auto F32 = [ws](int64_t off) { return reinterpret_cast<float*>(ws + off); };
  const int64_t P = L.P, R = L.R;
  if (R * ((a.H + 511) / 512) >= (int64_t(1) << 30) || R * ((a.I + 511) / 512) >= (int64_t(1) << 30))
    return cudaErrorInvalidValue;  // 32-bit chunk loops of the row quantizer
  cudaError_t e;

  // 1. route: count, scan, place
  {
    int64_t G64 = (P + 511) / 512;
    const int G = (int)(G64 < 1 ? 1 : (G64 > kRouteCtasMax ? kRouteCtasMax : G64));
    note_launch();
    moe_route_count_kernel<<<G, kRouteThreads, (size_t)a.E * sizeof(int32_t), s>>>(a.topk_ids, P, a.E,
                                                                                    I32(L.cta_count), status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    note_launch();
    moe_route_scan_kernel<<<1, kScanThreads, 0, s>>>(I32(L.cta_count), G, a.E, I32(L.cta_base), I32(L.counts),
                                                      I32(L.offsets), I32(L.row_pair), I32(L.tile_expert),
                                                      I32(L.tile_count), U32(L.amax_x), U32(L.amax_h));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    note_launch();
    moe_route_place_kernel<<<G, kRouteThreads, (size_t)kRouteWarps * a.E * sizeof(int32_t), s>>>(
        a.topk_ids, P, a.E, I32(L.cta_base), I32(L.offsets), I32(L.row_pair));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // 2. token pass
  {
    int64_t blocks = (a.T + 7) / 8;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    note_launch();
    moe_token_pass_kernel<<<(int)blocks, 256, 0, s>>>(static_cast<const uint4*>(a.x), a.T, a.H, a.topk_ids,
                                                       a.topk, a.E, U32(L.amax_x), reinterpret_cast<float4*>(a.out));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  const int qgrid = num_sms * 4;
  const size_t qsmem = (size_t)a.E * sizeof(float);
  // 3. gather + quantize x per expert
  note_launch();
  if (narrow_chunks(R, a.H) && narrow_chunks(a.T, a.H))
    moe_quantize_rows_kernel<true, true><<<qgrid, kRowThreads, qsmem, s>>>(
        static_cast<const uint4*>(a.x), a.H, a.topk, I32(L.row_pair), I32(L.tile_expert), I32(L.tile_count),
        U32(L.amax_x), a.E, reinterpret_cast<uint2*>(ws + L.xq_codes), ws + L.xq_scales, F32(L.xq_g), status,
        chunk_magic_narrow(a.H));
  else
    moe_quantize_rows_kernel<true, false><<<qgrid, kRowThreads, qsmem, s>>>(
        static_cast<const uint4*>(a.x), a.H, a.topk, I32(L.row_pair), I32(L.tile_expert), I32(L.tile_count),
        U32(L.amax_x), a.E, reinterpret_cast<uint2*>(ws + L.xq_codes), ws + L.xq_scales, F32(L.xq_g), status,
        chunk_magic(a.H));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // 4. gate_up grouped GEMM
  {
    CUtensorMap tmA, tmB;
    if (encode_tensor_map_2d(&tmA, ws + L.xq_codes, a.H / 2, R, a.H / 2, kBK / 2, kBM) != CUDA_SUCCESS ||
        encode_tensor_map_2d(&tmB, a.w13_q, a.H / 2, (uint64_t)a.E * 2 * a.I, a.H / 2, kBK / 2, 128) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    GateUpProblem p;
    p.K = (int)a.H;
    p.I = (int)a.I;
    p.n_tiles = (int)(a.I / 128);
    p.kgroups = (int)(a.H / 64);
    p.sf_expert_bytes = scale_bytes_(2 * a.I, a.H);
    p.tile_count = I32(L.tile_count);
    p.tile_expert = I32(L.tile_expert);
    p.sfa = ws + L.xq_scales;
    p.sfb = a.w13_s;
    p.ga = F32(L.xq_g);
    p.gb = a.w13_g;
    p.h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
    p.amax_h = U32(L.amax_h);
    if ((e = prepare_moe_kernel<GateUpProblem>()) != cudaSuccess) return e;
    int64_t max_tiles = (R / 128) * p.n_tiles;
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    note_launch();
    nvf4_gemm_kernel<GateUpProblem><<<grid, kGemmThreads, gemm_smem_bytes<GateUpProblem>(), s>>>(
        tmA, tmB, tmA /* output map unused: direct stores */, p, status, kMoeTimeoutNs, 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // 5. quantize h per expert
  note_launch();
  if (narrow_chunks(R, a.I))
    moe_quantize_rows_kernel<false, true><<<qgrid, kRowThreads, qsmem, s>>>(
        reinterpret_cast<const uint4*>(ws + L.h), a.I, a.topk, I32(L.row_pair), I32(L.tile_expert),
        I32(L.tile_count), U32(L.amax_h), a.E, reinterpret_cast<uint2*>(ws + L.hq_codes), ws + L.hq_scales,
        F32(L.hq_g), status, chunk_magic_narrow(a.I));
  else
    moe_quantize_rows_kernel<false, false><<<qgrid, kRowThreads, qsmem, s>>>(
        reinterpret_cast<const uint4*>(ws + L.h), a.I, a.topk, I32(L.row_pair), I32(L.tile_expert),
        I32(L.tile_count), U32(L.amax_h), a.E, reinterpret_cast<uint2*>(ws + L.hq_codes), ws + L.hq_scales,
        F32(L.hq_g), status, chunk_magic(a.I));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // 6. down grouped GEMM + weighted FP32 combine
  {
    CUtensorMap tmA, tmB;
    if (encode_tensor_map_2d(&tmA, ws + L.hq_codes, a.I / 2, R, a.I / 2, kBK / 2, kBM) != CUDA_SUCCESS ||
        encode_tensor_map_2d(&tmB, a.w2_q, a.I / 2, (uint64_t)a.E * a.H, a.I / 2, kBK / 2, 128) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    DownProblem p;
    p.K = (int)a.I;
    p.H = (int)a.H;
    p.n_tiles = (int)((a.H + 255) / 256);
    p.kgroups = (int)(a.I / 64);
    p.topk = a.topk;
    p.sf_expert_bytes = scale_bytes_(a.H, a.I);
    p.tile_count = I32(L.tile_count);
    p.tile_expert = I32(L.tile_expert);
    p.row_pair = I32(L.row_pair);
    p.topk_w = a.topk_w;
    p.sfa = ws + L.hq_scales;
    p.sfb = a.w2_s;
    p.ga = F32(L.hq_g);
    p.gb = a.w2_g;
    p.out = a.out;
    if ((e = prepare_moe_kernel<DownProblem>()) != cudaSuccess) return e;
    int64_t max_tiles = (R / 128) * p.n_tiles;
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    note_launch();
    nvf4_gemm_kernel<DownProblem><<<grid, kGemmThreads, gemm_smem_bytes<DownProblem>(), s>>>(
        tmA, tmB, tmA /* output map unused: bulk reductions */, p, status, kMoeTimeoutNs, 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nvfp4

// ----------------------------------------------------------------------------
// C ABI of the MoE layer.
// ----------------------------------------------------------------------------
extern "C" {

size_t nvfp4_moe_workspace_bytes(int64_t T, int64_t H, int64_t I, int E, int topk) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0) return 0;
  return (size_t)nvfp4::moe_layout(T, H, I, E, topk).total;
}

nvfp4_status nvfp4_moe_grouped_gemm(const void* x, int64_t T, int64_t H, const int32_t* topk_ids,
                                    const float* topk_w, int topk, int E, int64_t I, const uint8_t* w13_q,
                                    const uint8_t* w13_s, const float* w13_g, const uint8_t* w2_q,
                                    const uint8_t* w2_s, const float* w2_g, float* out, void* workspace,
                                    size_t workspace_bytes, nvfp4_stream_t stream) {
  if (T < 0 || H <= 0 || I <= 0 || H % 256 || I % 128 || topk < 1 || E < 1 || E > 1024 || topk > E ||
      T * topk >= (1ll << 31) || (int64_t)E * 2 * I >= (1ll << 31) || (int64_t)E * H >= (1ll << 31))
    return NVFP4_ERR_INVALID_ARG;
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!w13_q || !w13_s || !w13_g || !w2_q || !w2_s || !w2_g || !al(w13_q) || !al(w13_s) || !al(w2_q) || !al(w2_s))
    return NVFP4_ERR_INVALID_ARG;
  if (T > 0 && (!x || !topk_ids || !topk_w || !out || !al(x) || !al(out))) return NVFP4_ERR_INVALID_ARG;
  if (!workspace || !al(workspace) || workspace_bytes < nvfp4_moe_workspace_bytes(T, H, I, E, topk))
    return NVFP4_ERR_WORKSPACE;
  int num_sms = 0;
  int* status = nullptr;
  const int st = nvfp4::current_device_context(&num_sms, &status);
  if (st != NVFP4_OK) return (nvfp4_status)st;
  if (T == 0) return NVFP4_OK;
  nvfp4::MoeArgs a;
  a.x = x;
  a.T = T;
  a.H = H;
  a.I = I;
  a.topk_ids = topk_ids;
  a.topk_w = topk_w;
  a.topk = topk;
  a.E = E;
  a.w13_q = w13_q;
  a.w13_s = w13_s;
  a.w13_g = w13_g;
  a.w2_q = w2_q;
  a.w2_s = w2_s;
  a.w2_g = w2_g;
  a.out = out;
  a.ws = static_cast<uint8_t*>(workspace);
  return nvfp4::launch_moe(a, status, num_sms, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? NVFP4_OK
             : NVFP4_ERR_CUDA;
}

nvfp4_status nvfp4_moe_workspace_layout(int64_t T, int64_t H, int64_t I, int E, int topk,
                                        nvfp4_moe_layout* out) {
  if (!out || T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0) return NVFP4_ERR_INVALID_ARG;
  const nvfp4::MoeLayout L = nvfp4::moe_layout(T, H, I, E, topk);
  out->rows_capacity = L.R;
  out->counts = L.counts;
  out->offsets = L.offsets;
  out->row_pair = L.row_pair;
  out->xq_codes = L.xq_codes;
  out->xq_scales = L.xq_scales;
  out->xq_g = L.xq_g;
  out->h = L.h;
  out->hq_codes = L.hq_codes;
  out->hq_scales = L.hq_scales;
  out->hq_g = L.hq_g;
  out->total_bytes = L.total;
  return NVFP4_OK;
}

}  // extern "C"
