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
//   1 front A    per token: row amax -> per-CTA amax of every expert it is
//                routed to; per-CTA pair counts per expert; zero out[t].
//   2 front B    (programmatic dependent of A) expert totals, 128-padded
//                segment offsets, per-expert global scales, a stable sort of
//                the (token, slot) pairs by expert, and each token's x row
//                quantized once per routed expert into that expert's rows.
//   3 gate_up    grouped tcgen05 GEMM; a tile holds 128 gate and the matching
//                128 up columns; epilogue h = SiLU(gate)*up -> BF16, plus the
//                per-expert amax of h (pad rows: h = 0, not in the amax).
//   4 quantize h per expert, dynamic global scale.
//   5 down       grouped tcgen05 GEMM; epilogue scales by the routing weight
//                and adds into out[token] in FP32 (bulk reduce-adds).
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

constexpr int kFrontCtasMax = 256;      // front-end CTAs (each owns a contiguous token range)
constexpr int kFrontThreads = 512;
constexpr int kFrontWarps = kFrontThreads / 32;
constexpr int kFrontBatchPairs = 4096;  // (token, slot) pairs placed and quantized per batch

// Workspace layout (all regions 256-byte aligned).
struct MoeLayout {
  int64_t R, P, Ep;
  int64_t counts, offsets, row_pair, tile_expert, tile_count, amax_h, cta_count, cta_amax;
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
  L.Ep = ((int64_t)E + 3) & ~int64_t(3);  // per-CTA table rows padded to 16 bytes
  int64_t o = 0;
  auto take = [&o](int64_t bytes) {
    const int64_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.counts = take(4 * (int64_t)E);
  L.offsets = take(4 * ((int64_t)E + 1));
  L.row_pair = take(4 * L.R);
  L.tile_expert = take(4 * (L.R / 128));
  L.tile_count = take(4);
  L.amax_h = take(4 * (int64_t)E);
  L.cta_count = take(4 * (int64_t)kFrontCtasMax * L.Ep);
  L.cta_amax = take(4 * (int64_t)kFrontCtasMax * L.Ep);
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
// 1. Front pass A. G CTAs; CTA c owns tokens [T*c/G, T*(c+1)/G). Per token:
// the magnitude maximum of x[t] (BF16 bits & 0x7FFF; Inf and NaN order
// above every finite value) goes into a shared-memory maximum for every
// expert the token is routed to, the token's (token, slot) pairs are counted
// per expert, and its output row is zeroed (the down projection adds into
// it). The two tables leave as row c of cta_amax and cta_count (rows of Ep
// entries, the padding zero). Routing ids outside [0, E) are reported and
// skipped.
// ----------------------------------------------------------------------------
constexpr int kCountThreads = 1024;
constexpr int kCountWarps = kCountThreads / 32;

__global__ void __launch_bounds__(kCountThreads) moe_front_count_kernel(
    const uint4* __restrict__ x, int64_t T, int64_t H, const int32_t* __restrict__ topk_ids, int topk, int E,
    int Ep, int32_t* __restrict__ cta_count, uint32_t* __restrict__ cta_amax, float4* __restrict__ out,
    int* status) {
  extern __shared__ uint32_t front_a[];
  uint32_t* hist = front_a;        // [Ep]
  uint32_t* amax = front_a + Ep;   // [Ep]
  for (int e = threadIdx.x; e < Ep; e += blockDim.x) {
    hist[e] = 0u;
    amax[e] = 0u;
  }
  __syncthreads();
  grid_dependents_launch();  // front pass B may start its set-up
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
  const int64_t hv = H / 8;   // 16-byte vectors per row
  bool bad = false;
  // two tokens per warp per trip, all their loads issued first
  for (int64_t ta = t0 + warp; ta < t1; ta += 2 * kCountWarps) {
    const int64_t tb = ta + kCountWarps;
    const uint4* row_a = x + ta * hv;
    const uint4* row_b = x + (tb < t1 ? tb : ta) * hv;
    uint32_t ma2 = 0, mb2 = 0;
    for (int64_t i0 = lane; i0 < hv; i0 += 32 * 8) {
      uint4 va[8], vb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool in = i0 + 32 * u < hv;
        va[u] = in && NVFP4_IN_BOUNDS(ta * hv + i0 + 32 * u, T * hv, status) ? ld_stream(row_a + i0 + 32 * u)
                                                                                : make_uint4(0, 0, 0, 0);
        vb[u] = in && tb < t1 && NVFP4_IN_BOUNDS(tb * hv + i0 + 32 * u, T * hv, status)
                    ? ld_stream(row_b + i0 + 32 * u)
                    : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        ma2 = __vmaxu2(ma2, va[u].x & 0x7FFF7FFFu);
        ma2 = __vmaxu2(ma2, va[u].y & 0x7FFF7FFFu);
        ma2 = __vmaxu2(ma2, va[u].z & 0x7FFF7FFFu);
        ma2 = __vmaxu2(ma2, va[u].w & 0x7FFF7FFFu);
        mb2 = __vmaxu2(mb2, vb[u].x & 0x7FFF7FFFu);
        mb2 = __vmaxu2(mb2, vb[u].y & 0x7FFF7FFFu);
        mb2 = __vmaxu2(mb2, vb[u].z & 0x7FFF7FFFu);
        mb2 = __vmaxu2(mb2, vb[u].w & 0x7FFF7FFFu);
      }
    }
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      const int64_t t = side ? tb : ta;
      if (t >= t1) break;  // warp-uniform
      const uint32_t m2 = side ? mb2 : ma2;
      uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));
      for (int j = lane; j < topk; j += 32) {
        const int e = topk_ids[t * topk + j];
        if (e >= 0 && e < E) {
          atomicAdd(&hist[e], 1u);
          atomicMax(&amax[e], m);
        } else {
          bad = true;
        }
      }
      float4* orow = out + t * (H / 4);
      if (NVFP4_IN_BOUNDS(t, T, status))
        for (int64_t i = lane; i < H / 4; i += 32) orow[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  if (bad) record_status(status, NVFP4_ERR_INVALID_ARG);
  __syncthreads();
  for (int e = threadIdx.x; e < Ep; e += blockDim.x) {
    if (!NVFP4_IN_BOUNDS((int64_t)blockIdx.x * Ep + e, (int64_t)kFrontCtasMax * Ep, status)) continue;
    cta_count[(int64_t)blockIdx.x * Ep + e] = (int32_t)hist[e];
    cta_amax[(int64_t)blockIdx.x * Ep + e] = amax[e];
  }
}

// Exclusive scan over `n` <= 2 * kFrontThreads values held two per thread
// (v0 at index 2*tid, v1 at 2*tid+1); returns the exclusive prefix of v0.
// Every thread of the CTA calls it.
__device__ __forceinline__ int32_t block_excl_scan2(int32_t v0, int32_t v1, int32_t* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t pair = v0 + v1;
  int32_t incl = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(kFullMask, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < kFrontWarps ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(kFullMask, w, o);
      if (lane >= o) w += v;
    }
    if (lane < kFrontWarps) wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int32_t r = incl - pair + (warp > 0 ? wsum[warp - 1] : 0);
  __syncthreads();  // wsum may be reused
  return r;
}

// ----------------------------------------------------------------------------
// 2. Front pass B, a programmatic dependent of pass A on the same G CTAs and
// token ranges. Every CTA reduces the per-CTA tables over all CTAs (16-byte
// loads, S row slices per group of four experts): expert totals -> segments
// padded to 128 rows (exclusive scan over experts), each expert's global
// scale g = amax/2688 over the rows routed to it, and this CTA's base inside
// each segment (the pairs of the CTAs before it). CTA 0 publishes counts,
// offsets, the tile count and the global scales, and zeroes the amax slots
// of h; the m-tile -> expert entries and pad-row markers of expert e are
// written by CTA e % G. Then, batch by batch, the CTA ranks its pairs per
// expert in pair order (per-warp counts, a prefix over warps, and
// __match_any_sync inside each group of 32 pairs: a stable sort), records the
// pair of every row, and quantizes each token's row once per routed expert
// straight into that expert's rows: a row's 16-element blocks are loaded and
// their maxima taken once, the block scales and codes follow each expert's g.
// Pad rows of the gathered activations are left as they are: the gate/up
// epilogue writes zero for them and keeps them out of the amax of h.
// ----------------------------------------------------------------------------
struct FrontB {
  const uint4* x;
  int64_t T, H;
  int64_t R;               // padded row capacity of the gathered activations
  const int32_t* topk_ids;
  int topk, E, Ep;
  const int32_t* cta_count;
  const uint32_t* cta_amax;
  int32_t *counts, *offsets, *row_pair, *tile_expert, *tile_count;
  float* xq_g;
  uint32_t* amax_h;
  uint2* xq_codes;
  uint8_t* xq_scales;
  int* status;
};

template <class Idx>
__global__ void __launch_bounds__(kFrontThreads, 1) moe_front_place_quantize_kernel(const FrontB a) {
  extern __shared__ int32_t front_b[];
  const int E = a.E, Ep = a.Ep, topk = a.topk;
  const int G = gridDim.x, c = blockIdx.x;
  int32_t* base = front_b;                                  // [Ep]  running row of each expert
  float* g_s = reinterpret_cast<float*>(base + Ep);        // [Ep]
  int32_t* wcnt = base + 2 * Ep;                            // [kFrontWarps][Ep]
  int32_t* pos_s = wcnt + kFrontWarps * Ep;                 // [kFrontBatchPairs]
  int32_t* exp_s = pos_s + kFrontBatchPairs;                // [kFrontBatchPairs]
  __shared__ int32_t wsum[kFrontWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  grid_dependency_wait();  // pass A's tables are complete and visible

  // ---- column reduction of the per-CTA tables: groups of four experts x S row slices
  {
    const int groups = Ep / 4;
    // three [S][Ep] partial tables in the space of wcnt, pos_s and exp_s
    const int cap = (kFrontWarps * Ep + 2 * kFrontBatchPairs) / (3 * Ep);
    int S = kFrontThreads / groups;
    S = S > cap ? cap : S;
    S = S > G ? G : S;
    S = S < 1 ? 1 : S;
    int32_t* tot = wcnt;                    // [S][Ep]
    int32_t* below = wcnt + S * Ep;         // [S][Ep]
    uint32_t* mx = reinterpret_cast<uint32_t*>(wcnt + 2 * S * Ep);  // [S][Ep]
    for (int item = threadIdx.x; item < groups * S; item += blockDim.x) {
      const int g4 = item % groups, sl = item / groups;
      const int r0 = G * sl / S, r1 = G * (sl + 1) / S;
      int4 t4 = make_int4(0, 0, 0, 0), b4 = make_int4(0, 0, 0, 0);
      uint4 m4 = make_uint4(0, 0, 0, 0);
      const int4* cc = reinterpret_cast<const int4*>(a.cta_count) + g4;
      const uint4* ca = reinterpret_cast<const uint4*>(a.cta_amax) + g4;
#pragma unroll 8
      for (int r = r0; r < r1; ++r) {
        const int4 v = __ldcg(cc + (int64_t)r * groups);
        const uint4 w = __ldcg(ca + (int64_t)r * groups);
        t4.x += v.x; t4.y += v.y; t4.z += v.z; t4.w += v.w;
        if (r < c) {
          b4.x += v.x; b4.y += v.y; b4.z += v.z; b4.w += v.w;
        }
        m4.x = max(m4.x, w.x); m4.y = max(m4.y, w.y); m4.z = max(m4.z, w.z); m4.w = max(m4.w, w.w);
      }
      int32_t* tp = tot + sl * Ep + 4 * g4;
      int32_t* bp = below + sl * Ep + 4 * g4;
      uint32_t* mp = mx + sl * Ep + 4 * g4;
      tp[0] = t4.x; tp[1] = t4.y; tp[2] = t4.z; tp[3] = t4.w;
      bp[0] = b4.x; bp[1] = b4.y; bp[2] = b4.z; bp[3] = b4.w;
      mp[0] = m4.x; mp[1] = m4.y; mp[2] = m4.z; mp[3] = m4.w;
    }
    __syncthreads();
    // thread i owns experts 2i and 2i+1
    int32_t tv[2] = {0, 0}, bv[2] = {0, 0};
    uint32_t mv[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = 2 * threadIdx.x + k;
      if (e < E)
        for (int sl = 0; sl < S; ++sl) {
          tv[k] += tot[sl * Ep + e];
          bv[k] += below[sl * Ep + e];
          mv[k] = max(mv[k], mx[sl * Ep + e]);
        }
    }
    const int32_t p0 = (tv[0] + 127) & ~127, p1 = (tv[1] + 127) & ~127;
    const int32_t ex0 = block_excl_scan2(p0, p1, wsum);    // ends with __syncthreads: tables may be reused
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = 2 * threadIdx.x + k;
      if (e >= E) continue;
      const int32_t off = k == 0 ? ex0 : ex0 + p0;
      const int32_t padded = k == 0 ? p0 : p1;
      base[e] = off + bv[k];
      const float gv = global_scale_from_amax(__uint_as_float(mv[k] << 16));
      g_s[e] = gv;
      if (c == 0) {
        a.counts[e] = tv[k];
        a.offsets[e] = off;
        a.xq_g[e] = gv;
        a.amax_h[e] = 0u;
        if (mv[k] >= 0x7F80u) record_status(a.status, NVFP4_ERR_NONFINITE_INPUT);
        if (e == E - 1) {
          a.offsets[E] = off + padded;
          *a.tile_count = (off + padded) / 128;
        }
      }
      if (e % G == c) {
        for (int32_t t = off / 128; t < (off + padded) / 128; ++t)
          if (NVFP4_IN_BOUNDS(t, a.R / 128, a.status)) a.tile_expert[t] = e;
        for (int32_t r = off + tv[k]; r < off + padded; ++r)
          if (NVFP4_IN_BOUNDS(r, a.R, a.status)) a.row_pair[r] = -1;  // pad rows
      }
    }
    __syncthreads();
  }

  // ---- placement and quantization, batch by batch
  const int64_t t0 = a.T * c / G, t1 = a.T * (c + 1) / G;
  const int64_t tok_per_batch = kFrontBatchPairs / topk > 0 ? kFrontBatchPairs / topk : 1;
  const int32_t cpr = (int32_t)((a.H + 511) >> 9);
  const int64_t hv = a.H / 8;
  const int64_t kgroups = a.H / 64;
  for (int64_t tb0 = t0; tb0 < t1; tb0 += tok_per_batch) {
    const int64_t tb1 = tb0 + tok_per_batch < t1 ? tb0 + tok_per_batch : t1;
    const int64_t pb0 = tb0 * topk, np = (tb1 - tb0) * topk;
    for (int i = threadIdx.x; i < kFrontWarps * Ep; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int64_t wlo = pb0 + np * warp / kFrontWarps, whi = pb0 + np * (warp + 1) / kFrontWarps;
    for (int64_t p = wlo + lane; p < whi; p += 32) {
      const int e = a.topk_ids[p];
      if (e >= 0 && e < E) atomicAdd(&wcnt[warp * Ep + e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int32_t run = base[e];
      for (int w = 0; w < kFrontWarps; ++w) {
        const int32_t n = wcnt[w * Ep + e];
        wcnt[w * Ep + e] = run;
        run += n;
      }
      base[e] = run;
    }
    __syncthreads();
    for (int64_t q0 = wlo; q0 < whi; q0 += 32) {
      const int64_t p = q0 + lane;
      int e = p < whi ? a.topk_ids[p] : -1;
      if (e >= E) e = -1;
      const unsigned same = __match_any_sync(kFullMask, e);
      const int rank = __popc(same & ((1u << lane) - 1u));
      const int leader = __ffs(same) - 1;
      int32_t row = -1;
      if (e >= 0) {
        row = wcnt[warp * Ep + e] + rank;
        if (NVFP4_IN_BOUNDS(row, a.R, a.status)) a.row_pair[row] = (int32_t)p;
      }
      if (p < whi) {
        pos_s[p - pb0] = row;
        exp_s[p - pb0] = e;
      }
      __syncwarp();
      if (e >= 0 && lane == leader) wcnt[warp * Ep + e] += __popc(same);
      __syncwarp();
    }
    __syncthreads();
    // one warp per token: its blocks loaded once, quantized once per routed expert
    for (int64_t t = tb0 + warp; t < tb1; t += kFrontWarps) {
      const int32_t* pp = pos_s + (t - tb0) * topk;
      const int32_t* pe = exp_s + (t - tb0) * topk;
      for (int32_t ch0 = 0; ch0 < cpr; ch0 += 4) {
        Raw16 raw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int32_t col = (ch0 + u) * 512 + lane * 16;
          load_raw16(a.x, (Idx)t * (Idx)hv + (Idx)(col >> 3),
                     ch0 + u < cpr && col < a.H && NVFP4_IN_BOUNDS(t * hv + (col >> 3) + 1, a.T * hv, a.status),
                     raw[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (ch0 + u >= cpr) break;  // warp-uniform
          const int32_t col = (ch0 + u) * 512 + lane * 16;
          const bool valid = col < a.H;
          const float bmax = block_absmax(raw[u]);
          f32x2 xs[8];
          unpack_block(raw[u], xs);
          for (int j = 0; j < topk; ++j) {
            const int e = pe[j];
            if (e < 0) continue;  // warp-uniform
            const Idx row = (Idx)pp[j];
            Block b;
            quantize_block<false, false>(xs, bmax, g_s[e], 6.0f, b);
            if (valid) {
              const Idx cw = (row * (Idx)a.H + (Idx)col) >> 4;
              const Idx so = (((row >> 7) * (Idx)kgroups + (Idx)(col >> 6)) << 9) + ((row & 31) << 4) +
                             (((row >> 5) & 3) << 2) + (Idx)((col >> 4) & 3);
              if (NVFP4_IN_BOUNDS(cw, a.R * a.H / 16, a.status)) a.xq_codes[cw] = make_uint2(b.q0, b.q1);
              if (NVFP4_IN_BOUNDS(so, a.R / 128 * kgroups * 512, a.status)) a.xq_scales[so] = (uint8_t)b.sc;
            }
          }
        }
      }
    }
    __syncthreads();  // pos_s / exp_s / wcnt are rewritten by the next batch
  }
}

// ----------------------------------------------------------------------------
// 4. Quantization of h with a per-expert dynamic global scale. A warp's unit
// is a 512-element chunk of one padded row, one 16-element block per lane
// (block_math.cuh). Each trip takes kRowUnroll chunks: first their row
// lookups, then all their loads, then the arithmetic, so several chunks'
// loads are in flight together. Pad rows get zero codes and scales.
// amax_bits[e] holds the FP32 bits of expert e's amax of h (written by the
// gate/up epilogue); every CTA turns them into global scales in shared memory
// once.
// ----------------------------------------------------------------------------
constexpr int kRowThreads = 256;
constexpr int kRowUnroll = 4;

template <bool kNarrow>
__global__ void __launch_bounds__(kRowThreads, 4) moe_quantize_h_kernel(
    const uint4* __restrict__ src, int64_t K, int64_t R, const int32_t* __restrict__ row_pair,
    const int32_t* __restrict__ tile_expert, const int32_t* __restrict__ tile_count,
    const uint32_t* __restrict__ amax_bits, int E, uint2* __restrict__ codes, uint8_t* __restrict__ scales,
    float* __restrict__ g_out, int* status, uint64_t cpr_magic) {
  extern __shared__ float g_s[];  // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float amax = __uint_as_float(amax_bits[e]);
    const float g = global_scale_from_amax(amax);
    g_s[e] = g;
    if (blockIdx.x == 0) {
      g_out[e] = g;
      if (!(amax <= 3.0e38f)) record_status(status, NVFP4_ERR_NONFINITE_INPUT);
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
      const bool in = ch < n_chunks && NVFP4_IN_BOUNDS(cc[u].row, R, status);
      pr[u] = in ? row_pair[cc[u].row] : -1;
      ex[u] = in ? tile_expert[cc[u].row >> 7] : 0;
    }
    Raw16 vv[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u)
      load_raw16(src, cc[u].vec, pr[u] >= 0 && cc[u].valid && NVFP4_IN_BOUNDS(cc[u].vec + 1, R * K / 8, status),
                 vv[u]);
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
        const int64_t so = block_scale_offset(cc[u], K);
        if (NVFP4_IN_BOUNDS(cc[u].vec >> 1, R * K / 16, status)) codes[cc[u].vec >> 1] = make_uint2(b.q0, b.q1);
        if (NVFP4_IN_BOUNDS(so, R / 128 * (K / 64) * 512, status)) scales[so] = (uint8_t)b.sc;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// 3. gate_up grouped GEMM problem. Tiles are n-fastest: the I/128 column tiles
// of one m-tile run on neighbouring CTAs (A read once), and the m-tiles of an
// expert are adjacent (its weight tiles are re-read from L2).
// ----------------------------------------------------------------------------
struct GateUpProblem {
  static constexpr int kPipeStages = 4;
  static constexpr uint32_t kEpiWarpBytes = kEpiBytes;  // 32 x 16 BF16 staging box per warp
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
  const int32_t* row_pair; // -1 marks a pad row
  int64_t R;               // padded row capacity
  int* st;
  const uint8_t *sfa_lo, *sfa_hi, *sfb_lo, *sfb_hi;  // scale buffers (bounds-checking build)

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

  // Epilogue of one warp (rows q*32.., gate columns hh*64..): h =
  // SiLU(gate)*up in BF16, written through the warp's shared staging box
  // (32 rows x 16 columns, 32-byte swizzle) with TMA stores, so each tile's h
  // leaves as whole 32-byte row pieces; plus the per-expert amax of h.
  __device__ __forceinline__ void store(const TileJob& job, int q, int hh, int lane,
                                        const uint32_t (&acc)[4][32], uint8_t* stg, const CUtensorMap* tmH) const {
    const int row0 = job.m0 + q * 32;
    const float alpha = __fmul_rn(ga[job.expert], gb[job.expert]);
    // pad rows: their gathered activations were never written, so their
    // accumulators are meaningless; h gets zeros and stays out of the amax
    const uint32_t live =
        NVFP4_IN_BOUNDS(row0 + lane, R, st) && row_pair[row0 + lane] >= 0 ? 0xFFFFFFFFu : 0u;
    const uint32_t sbase = smem_u32(stg);
    uint32_t mx = 0;
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += kEpiCols) {
      if (lane == 0) bulk_wait_read_all();  // the previous box has left shared memory
      __syncwarp();
#pragma unroll
      for (int ch = 0; ch < kEpiCols / 8; ++ch) {
        const int j = (c0 + ch * 8) / 32, c = (c0 + ch * 8) % 32;
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
          packed[u] = f32x2_to_bf16x2(hv[0], hv[1]) & live;
          mx = __vmaxu2(mx, packed[u] & 0x7FFF7FFFu);
        }
        // 32-byte swizzle: 16-byte chunk index XOR bit 2 of the row
        st_shared_v4(sbase + lane * (kEpiCols * 2) + ((ch ^ ((lane >> 2) & 1)) << 4),
                     make_uint4(packed[0], packed[1], packed[2], packed[3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmH, stg, job.n0 + hh * 64 + c0, row0);
        bulk_commit_group();
      }
    }
    uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFullMask, m, o));
    if (lane == 0) atomicMax(&amax_h[job.expert], m << 16);  // FP32 bits of the BF16 amax
  }
};

// ----------------------------------------------------------------------------
// 5. down grouped GEMM problem: out[token] += w * (g_h * g_w2) * acc.
// The rows of a tile belong to different tokens, so the sum over a token's
// experts is a reduction into out, done by bulk reductions
// (cp.reduce.async.bulk .add.f32: element-wise adds performed by the memory
// system). The two epilogue warps of a tensor-memory lane quarter (same 32
// rows, column halves 0-127 and 128-255) stage whole 256-column row segments
// (1 KB of FP32) 16 rows at a time, alternating between two regions of 16
// rows, and the first warp's lanes 0..15 add each staged row into out with
// one 1 KB bulk reduction: 128 reductions of 1 KB per tile. (Each bulk
// operation has a fixed cost in the copy engine; with 128-byte pieces, 1024
// per tile, that cost bound the kernel. With 1 KB pieces the kernel is still
// bound per SM: on half the SMs it takes 1.9x as long.)
// ----------------------------------------------------------------------------
constexpr uint32_t kDownRowStride = 1040;       // staged row pitch: 1 KB of data + 16 B (conflict-free v4 stores)
constexpr uint32_t kDownGroupRows = 16;         // rows staged per bulk-reduction round
constexpr uint32_t kDownRegion = kDownGroupRows * kDownRowStride;  // one staging region

struct DownProblem {
  // One pipeline stage: the shared memory goes to two staging regions per
  // lane quarter, so a round never waits for the tile's other round
  // (measured: 153.0 -> 149.6 us against two stages and one region).
  static constexpr int kPipeStages = 1;
  static constexpr uint32_t kEpiWarpBytes = kDownRegion;  // a lane quarter's two regions span two warp slots
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
  int64_t R, P;            // padded row capacity, (token, slot) pairs
  int* st;
  const uint8_t *sfa_lo, *sfa_hi, *sfb_lo, *sfb_hi;  // scale buffers (bounds-checking build)

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

  // Epilogue warps 2..9: q = warp & 3 is the lane quarter, hh the column
  // half; warp slot (warp - 2) = hh*4 + ((q - 2) & 3). The quarter's region
  // is the two consecutive slots starting at slot 2*((q - 2) & 3), and named
  // barrier 1 + ((q - 2) & 3) pairs its two warps (64 threads).
  __device__ __forceinline__ void store(const TileJob& job, int q, int hh, int lane,
                                        const uint32_t (&acc)[4][32], uint8_t* stg, const CUtensorMap*) const {
    const int qi = (q - 2) & 3;
    uint8_t* epi_base = stg - (uint32_t)(hh * 4 + qi) * kEpiWarpBytes;
    const uint32_t region0 = smem_u32(epi_base + (uint32_t)qi * 2u * kDownRegion);
    const int row = job.m0 + q * 32 + lane;
    int32_t pair = NVFP4_IN_BOUNDS(row, R, st) ? row_pair[row] : -1;
    if (pair >= 0 && !NVFP4_IN_BOUNDS(pair, P, st)) pair = -1;
    const float alpha = __fmul_rn(ga[job.expert], gb[job.expert]);
    const float w = pair >= 0 ? topk_w[pair] : 0.0f;
    const int bar_id = 1 + qi;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      // round g uses region g; it is free once the previous tile's round-g
      // reductions have read it (one group per issuing lane and round, so at
      // most the latest group may still be pending)
      const uint32_t region = region0 + (uint32_t)g * kDownRegion;
      if (hh == 0 && lane < (int)kDownGroupRows) bulk_wait_read_but_one();
      named_barrier_sync(bar_id, 64);
      if ((lane >> 4) == g) {
        const uint32_t srow = region + (uint32_t)(lane & 15) * kDownRowStride + (uint32_t)hh * 512u;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            uint4 v;
            v.x = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 0]), alpha), w));
            v.y = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 1]), alpha), w));
            v.z = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 2]), alpha), w));
            v.w = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(acc[j][c + 3]), alpha), w));
            st_shared_v4(srow + (uint32_t)(32 * j + c) * 4u, v);
          }
        fence_proxy_async_smem();
      }
      named_barrier_sync(bar_id, 64);
      // lanes 0..15 of the first warp add staged rows 16g + lane into out
      const int32_t p = __shfl_sync(0xFFFFFFFFu, pair, (16 * g + lane) & 31);
      if (hh == 0 && lane < (int)kDownGroupRows) {
        if (p >= 0)
          bulk_reduce_add_f32(out + (size_t)(p / topk) * H + job.n0, region + (uint32_t)lane * kDownRowStride, 1024);
        bulk_commit_group();  // also when empty: one group per round
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
  const int64_t R = L.R;
  if (R * ((a.H + 511) / 512) >= (int64_t(1) << 30) || R * ((a.I + 511) / 512) >= (int64_t(1) << 30))
    return cudaErrorInvalidValue;  // 32-bit chunk loops of the row quantizer
  cudaError_t e;

  // 1-2. front end: per-CTA counts and amax, then placement and quantization
  {
    int G = num_sms < kFrontCtasMax ? num_sms : kFrontCtasMax;
    if (G < 1) G = 1;
    const int Ep = (int)L.Ep;
    note_launch();
    moe_front_count_kernel<<<G, kCountThreads, (size_t)2 * Ep * sizeof(uint32_t), s>>>(
        static_cast<const uint4*>(a.x), a.T, a.H, a.topk_ids, a.topk, a.E, Ep, I32(L.cta_count), U32(L.cta_amax),
        reinterpret_cast<float4*>(a.out), status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    FrontB fb;
    fb.x = static_cast<const uint4*>(a.x);
    fb.T = a.T;
    fb.H = a.H;
    fb.R = R;
    fb.topk_ids = a.topk_ids;
    fb.topk = a.topk;
    fb.E = a.E;
    fb.Ep = Ep;
    fb.cta_count = I32(L.cta_count);
    fb.cta_amax = U32(L.cta_amax);
    fb.counts = I32(L.counts);
    fb.offsets = I32(L.offsets);
    fb.row_pair = I32(L.row_pair);
    fb.tile_expert = I32(L.tile_expert);
    fb.tile_count = I32(L.tile_count);
    fb.xq_g = F32(L.xq_g);
    fb.amax_h = U32(L.amax_h);
    fb.xq_codes = reinterpret_cast<uint2*>(ws + L.xq_codes);
    fb.xq_scales = ws + L.xq_scales;
    fb.status = status;
    const size_t smem = (size_t)(2 + kFrontWarps) * Ep * sizeof(int32_t) + 2 * kFrontBatchPairs * sizeof(int32_t);
    const bool narrow = narrow_chunks(R, a.H) && narrow_chunks(a.T, a.H);
    const void* kern = narrow ? (const void*)moe_front_place_quantize_kernel<uint32_t>
                              : (const void*)moe_front_place_quantize_kernel<int64_t>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
      const int big = (int)((2 + kFrontWarps) * 1024 * sizeof(int32_t) + 2 * kFrontBatchPairs * sizeof(int32_t));
      attr_err = cudaFuncSetAttribute(moe_front_place_quantize_kernel<uint32_t>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, big);
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(moe_front_place_quantize_kernel<int64_t>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    });
    if (attr_err != cudaSuccess) return attr_err;
    // programmatic dependent of pass A: its CTAs start while pass A runs and
    // wait (griddepcontrol.wait) for pass A's tables before reading them
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kFrontThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {(void*)&fb};
    note_launch();
    if ((e = cudaLaunchKernelExC(&cfg, kern, args)) != cudaSuccess) return e;
  }

  // quantize h: one wave of resident CTAs (a grid beyond what fits leaves a
  // partial second wave behind the first)
  const size_t qsmem = (size_t)a.E * sizeof(float);
  auto q_occupancy = [qsmem](auto kern) {
    int occ = 0;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kRowThreads, qsmem) == cudaSuccess && occ > 0
               ? occ
               : 1;
  };
  const int qgrid = num_sms * (narrow_chunks(R, a.I) ? q_occupancy(moe_quantize_h_kernel<true>)
                                                     : q_occupancy(moe_quantize_h_kernel<false>));

  // 3. gate_up grouped GEMM
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
    p.row_pair = I32(L.row_pair);
    p.R = R;
    p.st = status;
    p.sfa_lo = ws + L.xq_scales;
    p.sfa_hi = p.sfa_lo + scale_bytes_(R, a.H);
    p.sfb_lo = a.w13_s;
    p.sfb_hi = a.w13_s + (size_t)a.E * p.sf_expert_bytes;
    if ((e = prepare_moe_kernel<GateUpProblem>()) != cudaSuccess) return e;
    CUtensorMap tmH;
    if (encode_store_map_bf16(&tmH, ws + L.h, (uint64_t)a.I, (uint64_t)R) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    int64_t max_tiles = (R / 128) * p.n_tiles;
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    note_launch();
    nvf4_gemm_kernel<GateUpProblem><<<grid, kGemmThreads, gemm_smem_bytes<GateUpProblem>(), s>>>(
        tmA, tmB, tmH, p, status, kMoeTimeoutNs, 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // 4. quantize h per expert
  note_launch();
  if (narrow_chunks(R, a.I))
    moe_quantize_h_kernel<true><<<qgrid, kRowThreads, qsmem, s>>>(
        reinterpret_cast<const uint4*>(ws + L.h), a.I, R, I32(L.row_pair), I32(L.tile_expert), I32(L.tile_count),
        U32(L.amax_h), a.E, reinterpret_cast<uint2*>(ws + L.hq_codes), ws + L.hq_scales, F32(L.hq_g), status,
        chunk_magic_narrow(a.I));
  else
    moe_quantize_h_kernel<false><<<qgrid, kRowThreads, qsmem, s>>>(
        reinterpret_cast<const uint4*>(ws + L.h), a.I, R, I32(L.row_pair), I32(L.tile_expert), I32(L.tile_count),
        U32(L.amax_h), a.E, reinterpret_cast<uint2*>(ws + L.hq_codes), ws + L.hq_scales, F32(L.hq_g), status,
        chunk_magic(a.I));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // 5. down grouped GEMM + weighted FP32 combine
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
    p.R = R;
    p.P = a.T * a.topk;
    p.st = status;
    p.sfa_lo = ws + L.hq_scales;
    p.sfa_hi = p.sfa_lo + scale_bytes_(R, a.I);
    p.sfb_lo = a.w2_s;
    p.sfb_hi = a.w2_s + (size_t)a.E * p.sf_expert_bytes;
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
