// Top-k logit KL distillation loss ("Model-Optimizer in practice: recovering
// Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD", section "QAD":
// --logit_kl_topk 4096 restricts the KD loss to the teacher's top-4096
// vocabulary entries, so no dense [seq x vocab] FP32 tensor is formed).
//
// Per row: the set is the k entries with the largest teacher logits (ties to
// the lower index); teacher and student distributions are softmax over the
// set; loss = KL(p_t || p_s) = sum p_t (t - s) - lse_t + lse_s with
// p_t = exp(t - lse_t); d loss / d s = p_s - p_t on the set.
//
// One CTA of 512 threads per row (persistent over rows, two CTAs per SM).
// The set is found by a two-digit radix select on order-preserving 16-bit
// keys of the BF16 teacher logits (high byte, then low byte among the
// high-byte bin that holds the k-th largest), which gives the threshold key
// T, the count above it, and
// how many entries equal to T the set takes (the lowest indices). A third
// pass walks the row in index order, ranks the entries equal to T with a
// block scan, and accumulates the two log-sum-exps and sum p_t (t - s)
// online (rescaled when the running maximum grows). The histograms are
// per warp (shared-memory atomics; logits concentrate in few bins, so warps
// must not share counters).
//
// Fast path (taken when it can be): a 1/16 sample of the row gives a key T0
// just below the k-th largest; one pass compacts the entries with key >= T0
// (each warp its own contiguous segment, so the candidates stay in index
// order) into shared memory; the exact select, the tie ranking and the
// accumulation then run on the candidates only, and the student logits are
// read at the candidates alone. The compaction tests two logits per
// instruction against T0's value (packed BF16 compare) and works on keys
// only for the few entries that pass; each candidate's student logit is
// fetched by an asynchronous 4-byte copy into shared memory issued as the
// candidate is found, so the gathers overlap the rest of the pass; the set
// and the gradient are written from those shared-memory candidates. If the
// sample undershoots (fewer than k candidates) or a segment overflows its
// capacity, the row takes the full three-pass path.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

constexpr int kKdThreads = 512;  // two CTAs per SM: one row's selection overlaps another's streaming
constexpr int kKdWarps = kKdThreads / 32;
constexpr int kKdUnroll = 4;  // 16-byte loads in flight per thread in the histogram passes

// BF16 bits -> key whose unsigned order is the value order (-0 maps to +0).
__device__ __forceinline__ uint32_t kd_key(uint32_t b) {
  b &= 0xFFFFu;
  if (b == 0x8000u) b = 0u;
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
// Inverse of kd_key (for -0 it gives +0, the same value).
__device__ __forceinline__ float kd_value(uint32_t key) {
  const uint32_t b = (key & 0x8000u) ? (key ^ 0x8000u) : (~key & 0xFFFFu);
  return __uint_as_float(b << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per half of two BF16 pairs: 0xFFFF where a >= b or either is NaN, else 0.
__device__ __forceinline__ uint32_t bf16x2_geu_mask(uint32_t a, uint32_t b) {
  return __hgeu2_mask(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
}

// 4-byte asynchronous copy global -> shared (completion: cp_async_wait_all).
__device__ __forceinline__ void cp_async_4(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

constexpr int kSampleStride = 16;   // the sample reads every 16th 16-byte vector of a row
constexpr int kCandPerWarp = 512;   // candidate capacity of one warp's row segment

struct KdShared {
  uint32_t whist[kKdWarps][256];  // per-warp histograms (no cross-warp contention)
  uint32_t hist[256];
  uint32_t scan[kKdWarps];
  uint32_t bin, above;      // find_bin result
  uint32_t eq_base, sel_base;
  uint32_t wcount[kKdWarps];  // candidates per warp segment
  uint32_t wtmp[kKdWarps];
  uint32_t fsel[kKdWarps], feq[kKdWarps];  // fast path: per-warp output base and tie rank base
  uint32_t fT, fneed;                      // fast path: threshold key and ties taken
  int overflow;
  float red[kKdWarps][5];
  uint16_t ckey[kKdWarps][kCandPerWarp];  // candidate keys, index order within a warp's segment
  uint32_t cstu[kKdWarps][kCandPerWarp];  // aligned student word holding the candidate's logit
  int32_t cidx[kKdWarps][kCandPerWarp];   // their vocabulary indices
};

// Histogram add into this warp's own histogram (lanes of one warp that hit
// the same bin are serialised by the shared-memory atomic unit; no other
// warp touches these counters).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// hist[b] = sum over warps of whist[w][b].
__device__ __forceinline__ void reduce_hist(KdShared& sh) {
  if (threadIdx.x < 256) {
    uint32_t c = 0;
#pragma unroll 8
    for (int w = 0; w < kKdWarps; ++w) c += sh.whist[w][threadIdx.x];
    sh.hist[threadIdx.x] = c;
  }
  __syncthreads();
}

// Bin b where the count of entries in bins >= b first reaches `need` (need >=
// 1 and at most the histogram total); also the count strictly above b. Called
// by all threads; reads sh.hist, writes sh.bin / sh.above.
__device__ __forceinline__ void find_bin(KdShared& sh, uint32_t need) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint32_t suf = 0, own = 0;
  if (t < 256) {
    own = sh.hist[t];
    suf = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
      if (lane + o < 32) suf += v;
    }
    if (lane == 0) sh.scan[warp] = suf;  // warp total
  }
  __syncthreads();
  if (t < 256) {
    for (int w = warp + 1; w < 8; ++w) suf += sh.scan[w];
    if (suf >= need && suf - own < need) {
      sh.bin = (uint32_t)t;
      sh.above = suf - own;
    }
  }
  __syncthreads();
}

// Block-wide exclusive scan of v (all threads); returns the exclusive prefix
// and writes the block total to *total.
__device__ __forceinline__ uint32_t block_scan(KdShared& sh, uint32_t v, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sh.scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kKdWarps ? sh.scan[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < kKdWarps) sh.scan[lane] = w;
  }
  __syncthreads();
  const uint32_t excl = incl - v + (warp > 0 ? sh.scan[warp - 1] : 0u);
  *total = sh.scan[kKdWarps - 1];
  __syncthreads();  // sh.scan is reused by the next scan
  return excl;
}

// Online log-sum-exp state with the teacher-weighted sum of (t - s).
struct KdAcc {
  float mt, zt, a, ms, zs;
  __device__ __forceinline__ void init() {
    mt = ms = -INFINITY;
    zt = a = zs = 0.0f;
  }
  __device__ __forceinline__ void add(float t, float s) {
    if (t > mt) {
      const float c = mt == -INFINITY ? 0.0f : expf(mt - t);
      zt = zt * c + 1.0f;
      a = a * c + (t - s);
      mt = t;
    } else {
      const float w = expf(t - mt);
      zt += w;
      a += w * (t - s);
    }
    if (s > ms) {
      zs = zs * (ms == -INFINITY ? 0.0f : expf(ms - s)) + 1.0f;
      ms = s;
    } else {
      zs += expf(s - ms);
    }
  }
  __device__ __forceinline__ void merge(const KdAcc& o) {
    if (o.mt != -INFINITY) {
      const float m = fmaxf(mt, o.mt);
      const float c1 = mt == -INFINITY ? 0.0f : expf(mt - m), c2 = expf(o.mt - m);
      zt = zt * c1 + o.zt * c2;
      a = a * c1 + o.a * c2;
      mt = m;
    }
    if (o.ms != -INFINITY) {
      const float m = fmaxf(ms, o.ms);
      zs = zs * (ms == -INFINITY ? 0.0f : expf(ms - m)) + o.zs * expf(o.ms - m);
      ms = m;
    }
  }
};

// Exclusive prefix of sh.wtmp over warps for warp w (sum of warps below w).
__device__ __forceinline__ uint32_t warp_prefix(const KdShared& sh, int w) {
  uint32_t p = 0;
  for (int i = 0; i < w; ++i) p += sh.wtmp[i];
  return p;
}

// Fast path of one row (see the file comment). Returns false, with nothing
// written, when the row must take the full path. All threads call it.
__device__ bool kd_fast_row(KdShared& sh, const uint4* trow, const uint16_t* srow16, int64_t nvec, int k,
                            KdAcc& acc, int32_t* idx_row, int* status) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;

  // ---- A: sample every kSampleStride-th vector; key of its ks-th largest
  const int64_t nsv = (nvec + kSampleStride - 1) / kSampleStride;    // sampled vectors
  const int64_t nse = nsv * 8;                                         // sampled elements
  const int64_t ks64 = (int64_t)k / kSampleStride + (int64_t)k / (4 * kSampleStride) + 32;
  uint32_t T0 = 0u;  // all entries are candidates unless the sample is large enough
  if (ks64 < nse) {
    const uint32_t ks = (uint32_t)ks64;
    for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
    __syncthreads();
    for (int64_t m = t; m < nsv; m += kKdThreads) {
      const uint4 v = trow[m * kSampleStride];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hist_add(sh.whist[warp], kd_key(w[e]) >> 8, true);
        hist_add(sh.whist[warp], kd_key(w[e] >> 16) >> 8, true);
      }
    }
    __syncthreads();
    reduce_hist(sh);
    find_bin(sh, ks);
    const uint32_t b1 = sh.bin, above1 = sh.above;
    for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
    __syncthreads();
    for (int64_t m = t; m < nsv; m += kKdThreads) {
      const uint4 v = trow[m * kSampleStride];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t k0 = kd_key(w[e]), k1 = kd_key(w[e] >> 16);
        hist_add(sh.whist[warp], k0 & 0xFFu, (k0 >> 8) == b1);
        hist_add(sh.whist[warp], k1 & 0xFFu, (k1 >> 8) == b1);
      }
    }
    __syncthreads();
    reduce_hist(sh);
    find_bin(sh, ks - above1);
    T0 = (b1 << 8) | sh.bin;
  }

  // ---- B: each warp compacts the entries >= T0 of its contiguous segment
  const int64_t lo = nvec * warp / kKdWarps, hi = nvec * (warp + 1) / kKdWarps;
  // T0 as a BF16 value in both halves; key 0 (every entry a candidate) maps
  // to a NaN pattern, which the unordered compare passes everywhere.
  const uint32_t tvb = (T0 & 0x8000u) ? (T0 ^ 0x8000u) : (~T0 & 0xFFFFu);
  const uint32_t thr2 = tvb | (tvb << 16);
  const uint32_t cstu_base = (uint32_t)__cvta_generic_to_shared(&sh.cstu[warp][0]);
  uint32_t cnt = 0;   // slots used (warp-uniform)
  uint32_t real = 0;  // candidates with key >= T0 (the value test also passes NaN)
  for (int64_t base = lo; base < hi; base += 4 * 32) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = base + u * 32 + lane;
      v[u] = j < hi ? trow[j] : make_uint4(0, 0, 0, 0);
    }
    // One bit per passing element at bit 8e (e = element within the vector).
    uint64_t q[4];
    uint32_t n[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = base + u * 32 + lane;
      const uint32_t lo4 = __byte_perm(bf16x2_geu_mask(v[u].x, thr2), bf16x2_geu_mask(v[u].y, thr2), 0x6420) & 0x01010101u;
      const uint32_t hi4 = __byte_perm(bf16x2_geu_mask(v[u].z, thr2), bf16x2_geu_mask(v[u].w, thr2), 0x6420) & 0x01010101u;
      q[u] = j < hi ? ((uint64_t)lo4 | ((uint64_t)hi4 << 32)) : 0ull;
      n[u] = (uint32_t)__popcll(q[u]);
    }
    // Slots: one warp scan of the four counts, two per 32-bit word.
    uint32_t p01 = n[0] | (n[1] << 16), p23 = n[2] | (n[3] << 16);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, p01, o), y = __shfl_up_sync(0xFFFFFFFFu, p23, o);
      if (lane >= o) {
        p01 += x;
        p23 += y;
      }
    }
    const uint32_t t01 = __shfl_sync(0xFFFFFFFFu, p01, 31), t23 = __shfl_sync(0xFFFFFFFFu, p23, 31);
    const uint32_t incl[4] = {p01 & 0xFFFFu, p01 >> 16, p23 & 0xFFFFu, p23 >> 16};
    const uint32_t tot[4] = {t01 & 0xFFFFu, t01 >> 16, t23 & 0xFFFFu, t23 >> 16};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = base + u * 32 + lane;
      uint64_t bits = q[u];
      uint32_t pos = cnt + incl[u] - n[u];
      while (bits) {  // ascending element order
        const int e = (__ffsll((long long)bits) - 1) >> 3;
        bits &= bits - 1;
        const int wi = e >> 1;
        const uint32_t wv = wi == 0 ? v[u].x : wi == 1 ? v[u].y : wi == 2 ? v[u].z : v[u].w;
        const uint32_t key = kd_key((e & 1) ? (wv >> 16) : wv);
        real += key >= T0;
        if (pos < (uint32_t)kCandPerWarp) {
          const int64_t idx = 8 * j + e;
          sh.ckey[warp][pos] = (uint16_t)key;
          sh.cidx[warp][pos] = (int32_t)idx;
          cp_async_4(cstu_base + 4u * pos, srow16 + (idx & ~int64_t(1)));
        }
        ++pos;
      }
      cnt += tot[u];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) real += __shfl_xor_sync(0xFFFFFFFFu, real, o);
  if (lane == 0) {
    sh.wcount[warp] = cnt;
    sh.wtmp[warp] = real;
  }
  __syncthreads();
  uint32_t total = 0;
  bool over = false;
  for (int w = 0; w < kKdWarps; ++w) {
    total += sh.wtmp[w];
    over |= sh.wcount[w] > (uint32_t)kCandPerWarp;
  }
  __syncthreads();  // sh.wtmp is reused below
  if (over || total < (uint32_t)k) {
    cp_async_wait_all();  // no copy may land in a later row's slots
    __syncthreads();
    return false;
  }

  // ---- C: exact select among the candidates
  const uint32_t mine = sh.wcount[warp];
  for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
  __syncthreads();
  for (uint32_t i = lane; i < mine; i += 32) hist_add(sh.whist[warp], (uint32_t)sh.ckey[warp][i] >> 8, true);
  __syncthreads();
  reduce_hist(sh);
  find_bin(sh, (uint32_t)k);
  const uint32_t b1 = sh.bin, above1 = sh.above;
  for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
  __syncthreads();
  for (uint32_t i = lane; i < mine; i += 32) {
    const uint32_t key = sh.ckey[warp][i];
    hist_add(sh.whist[warp], key & 0xFFu, (key >> 8) == b1);
  }
  __syncthreads();
  reduce_hist(sh);
  find_bin(sh, (uint32_t)k - above1);
  const uint32_t T = (b1 << 8) | sh.bin;
  const uint32_t need_eq = (uint32_t)k - (above1 + sh.above);

  // ---- D: rank ties in index order, accumulate, place the set
  cp_async_wait_all();  // this lane's student copies; then the warp's
  __syncwarp();
  uint32_t n_eq = 0;
  for (uint32_t i0 = 0; i0 < mine; i0 += 32) {
    const uint32_t i = i0 + lane;
    n_eq += __popc(__ballot_sync(0xFFFFFFFFu, i < mine && sh.ckey[warp][i] == T));
  }
  if (lane == 0) sh.wtmp[warp] = n_eq;
  __syncthreads();
  uint32_t eq_rank = warp_prefix(sh, warp), n_sel = 0;
  __syncthreads();
  for (uint32_t i0 = 0; i0 < mine; i0 += 32) {
    const uint32_t i = i0 + lane;
    const uint32_t key = i < mine ? sh.ckey[warp][i] : 0u;
    const unsigned eqm = __ballot_sync(0xFFFFFFFFu, i < mine && key == T);
    const bool eq = (eqm >> lane) & 1u;
    const bool sel = i < mine && (key > T || (eq && eq_rank + __popc(eqm & lt_mask) < need_eq));
    eq_rank += __popc(eqm);
    n_sel += __popc(__ballot_sync(0xFFFFFFFFu, sel));
    if (sel) {
      const uint32_t sw = sh.cstu[warp][i];
      acc.add(kd_value(key), __uint_as_float((sh.cidx[warp][i] & 1) ? (sw & 0xFFFF0000u) : (sw << 16)));
    }
  }
  if (idx_row) {
    if (lane == 0) sh.wtmp[warp] = n_sel;
    __syncthreads();
    uint32_t pos = warp_prefix(sh, warp);
    __syncthreads();
    if (lane == 0) sh.wtmp[warp] = n_eq;
    __syncthreads();
    eq_rank = warp_prefix(sh, warp);
    if (lane == 0) {  // kept for the gradient pass (kd_fast_grad)
      sh.fsel[warp] = pos;
      sh.feq[warp] = eq_rank;
      if (warp == 0) {
        sh.fT = T;
        sh.fneed = need_eq;
      }
    }
    for (uint32_t i0 = 0; i0 < mine; i0 += 32) {
      const uint32_t i = i0 + lane;
      const uint32_t key = i < mine ? sh.ckey[warp][i] : 0u;
      const unsigned eqm = __ballot_sync(0xFFFFFFFFu, i < mine && key == T);
      const bool eq = (eqm >> lane) & 1u;
      const bool sel = i < mine && (key > T || (eq && eq_rank + __popc(eqm & lt_mask) < need_eq));
      eq_rank += __popc(eqm);
      const unsigned selm = __ballot_sync(0xFFFFFFFFu, sel);
      if (sel && NVFP4_IN_BOUNDS(pos + __popc(selm & lt_mask), k, status))
        idx_row[pos + __popc(selm & lt_mask)] = sh.cidx[warp][i];
      pos += __popc(selm);
    }
  }
  __syncthreads();
  return true;
}

// Gradient p_s - p_t of a row the fast path served, written at the same
// output positions as its idx, from the candidates still in shared memory.
__device__ void kd_fast_grad(const KdShared& sh, float lse_t, float lse_s, float* grad_row, int k, int* status) {
  (void)k;
  (void)status;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  const uint32_t mine = sh.wcount[warp], T = sh.fT, need_eq = sh.fneed;
  uint32_t pos = sh.fsel[warp], eq_rank = sh.feq[warp];
  for (uint32_t i0 = 0; i0 < mine; i0 += 32) {
    const uint32_t i = i0 + lane;
    const uint32_t key = i < mine ? sh.ckey[warp][i] : 0u;
    const unsigned eqm = __ballot_sync(0xFFFFFFFFu, i < mine && key == T);
    const bool eq = (eqm >> lane) & 1u;
    const bool sel = i < mine && (key > T || (eq && eq_rank + __popc(eqm & lt_mask) < need_eq));
    eq_rank += __popc(eqm);
    const unsigned selm = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel && NVFP4_IN_BOUNDS(pos + __popc(selm & lt_mask), k, status)) {
      const uint32_t sw = sh.cstu[warp][i];
      const float sv = __uint_as_float((sh.cidx[warp][i] & 1) ? (sw & 0xFFFF0000u) : (sw << 16));
      grad_row[pos + __popc(selm & lt_mask)] = expf(sv - lse_s) - expf(kd_value(key) - lse_t);
    }
    pos += __popc(selm);
  }
}

__global__ void __launch_bounds__(kKdThreads, 2) topk_kl_kernel(const uint4* __restrict__ teacher,
                                                                 const uint4* __restrict__ student, int64_t rows,
                                                                 int64_t V, int k, float* __restrict__ loss,
                                                                 int32_t* __restrict__ idx_out,
                                                                 float* __restrict__ grad_out, int* status) {
  extern __shared__ __align__(16) uint8_t kd_smem[];
  KdShared& sh = *reinterpret_cast<KdShared*>(kd_smem);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t nvec = V / 8;
  const int64_t trips = (nvec + kKdThreads - 1) / kKdThreads;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint4* trow = teacher + row * nvec;
    const uint4* srow = student + row * nvec;
    KdAcc acc;
    acc.init();
    const bool fast = kd_fast_row(sh, trow, reinterpret_cast<const uint16_t*>(srow), nvec, k, acc,
                                  idx_out ? idx_out + row * k : nullptr, status);
    if (!fast) {
    // ---- pass 1: histogram of the key's high byte
    for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
    __syncthreads();
    for (int64_t it = 0; it < trips; it += kKdUnroll) {
      uint4 v[kKdUnroll];
#pragma unroll
      for (int u = 0; u < kKdUnroll; ++u) {
        const int64_t j = (it + u) * kKdThreads + t;
        v[u] = j < nvec ? trow[j] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kKdUnroll; ++u) {
        const bool act = (it + u) * kKdThreads + t < nvec;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hist_add(sh.whist[warp], kd_key(w[e]) >> 8, act);
          hist_add(sh.whist[warp], kd_key(w[e] >> 16) >> 8, act);
        }
      }
    }
    __syncthreads();
    reduce_hist(sh);
    find_bin(sh, (uint32_t)k);
    const uint32_t b1 = sh.bin, above1 = sh.above;
    __syncthreads();

    // ---- pass 2: histogram of the low byte inside bin b1
    for (int i = t; i < kKdWarps * 256; i += kKdThreads) (&sh.whist[0][0])[i] = 0u;
    __syncthreads();
    for (int64_t it = 0; it < trips; it += kKdUnroll) {
      uint4 v[kKdUnroll];
#pragma unroll
      for (int u = 0; u < kKdUnroll; ++u) {
        const int64_t j = (it + u) * kKdThreads + t;
        v[u] = j < nvec ? trow[j] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kKdUnroll; ++u) {
        const bool act = (it + u) * kKdThreads + t < nvec;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t k0 = kd_key(w[e]), k1 = kd_key(w[e] >> 16);
          hist_add(sh.whist[warp], k0 & 0xFFu, act && (k0 >> 8) == b1);
          hist_add(sh.whist[warp], k1 & 0xFFu, act && (k1 >> 8) == b1);
        }
      }
    }
    __syncthreads();
    reduce_hist(sh);
    find_bin(sh, (uint32_t)k - above1);
    const uint32_t T = (b1 << 8) | sh.bin;
    const uint32_t need_eq = (uint32_t)k - (above1 + sh.above);  // entries equal to T taken
    if (t == 0) {
      sh.eq_base = 0u;
      sh.sel_base = 0u;
    }
    __syncthreads();

    // ---- pass 3: select in index order, accumulate
    uint4 v_next = t < nvec ? trow[t] : make_uint4(0, 0, 0, 0);
    uint4 s_next = t < nvec ? srow[t] : make_uint4(0, 0, 0, 0);
    for (int64_t it = 0; it < trips; ++it) {
      const int64_t j = it * kKdThreads + t;
      const bool act = j < nvec;
      const uint4 v = v_next, sv = s_next;
      {  // next tile's loads overlap this tile's scans
        const int64_t jn = j + kKdThreads;
        v_next = jn < nvec ? trow[jn] : make_uint4(0, 0, 0, 0);
        s_next = jn < nvec ? srow[jn] : make_uint4(0, 0, 0, 0);
      }
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t keys[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        keys[2 * e] = act ? kd_key(w[e]) : 0u;
        keys[2 * e + 1] = act ? kd_key(w[e] >> 16) : 0u;
      }
      uint32_t n_eq = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) n_eq += keys[e] == T && act;
      uint32_t tot_eq = 0, eq_rank0 = sh.eq_base;
      if (__syncthreads_or(n_eq != 0)) eq_rank0 += block_scan(sh, n_eq, &tot_eq);
      uint32_t selmask = 0, r = eq_rank0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const bool eq = act && keys[e] == T;
        const bool sel = act && (keys[e] > T || (eq && r < need_eq));
        r += eq;
        selmask |= (uint32_t)sel << e;
      }
      uint32_t tot_sel = 0, pos = 0;
      if (idx_out) pos = sh.sel_base + block_scan(sh, (uint32_t)__popc(selmask), &tot_sel);
      if (selmask) {
        const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (!((selmask >> e) & 1u)) continue;
          const float tv = (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
          const float svv = (e & 1) ? bf16_hi(sw[e >> 1]) : bf16_lo(sw[e >> 1]);
          acc.add(tv, svv);
          if (idx_out) {
            if (NVFP4_IN_BOUNDS(pos, k, status)) idx_out[row * k + pos] = (int32_t)(8 * j + e);
            ++pos;
          }
        }
      }
      __syncthreads();  // everyone has read eq_base / sel_base
      if (t == 0) {
        sh.eq_base += tot_eq;
        if (idx_out) sh.sel_base += tot_sel;
      }
      __syncthreads();
    }

    }  // full path

    // ---- block reduction of the accumulators
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      KdAcc other;
      other.mt = __shfl_xor_sync(0xFFFFFFFFu, acc.mt, o);
      other.zt = __shfl_xor_sync(0xFFFFFFFFu, acc.zt, o);
      other.a = __shfl_xor_sync(0xFFFFFFFFu, acc.a, o);
      other.ms = __shfl_xor_sync(0xFFFFFFFFu, acc.ms, o);
      other.zs = __shfl_xor_sync(0xFFFFFFFFu, acc.zs, o);
      acc.merge(other);
    }
    if (lane == 0) {
      sh.red[warp][0] = acc.mt;
      sh.red[warp][1] = acc.zt;
      sh.red[warp][2] = acc.a;
      sh.red[warp][3] = acc.ms;
      sh.red[warp][4] = acc.zs;
    }
    __syncthreads();
    if (t == 0) {
      KdAcc tot;
      tot.init();
      for (int w2 = 0; w2 < kKdWarps; ++w2) {
        KdAcc o;
        o.mt = sh.red[w2][0];
        o.zt = sh.red[w2][1];
        o.a = sh.red[w2][2];
        o.ms = sh.red[w2][3];
        o.zs = sh.red[w2][4];
        tot.merge(o);
      }
      const float lse_t = tot.mt + logf(tot.zt), lse_s = tot.ms + logf(tot.zs);
      loss[row] = tot.a / tot.zt - lse_t + lse_s;
      sh.red[0][0] = lse_t;
      sh.red[0][1] = lse_s;
    }
    __syncthreads();

    // ---- optional pass 4: gradient p_s - p_t at the selected entries
    if (grad_out && idx_out && fast) {
      kd_fast_grad(sh, sh.red[0][0], sh.red[0][1], grad_out + row * k, k, status);
    } else if (grad_out && idx_out) {
      const float lse_t = sh.red[0][0], lse_s = sh.red[0][1];
      const uint16_t* t16 = reinterpret_cast<const uint16_t*>(trow);
      const uint16_t* s16 = reinterpret_cast<const uint16_t*>(srow);
      for (int i = t; i < k; i += kKdThreads) {
        int32_t v = idx_out[row * k + i];
        if (!NVFP4_IN_BOUNDS(v, V, status)) v = 0;
        const float tv = __uint_as_float((uint32_t)t16[v] << 16), svv = __uint_as_float((uint32_t)s16[v] << 16);
        grad_out[row * k + i] = expf(svv - lse_s) - expf(tv - lse_t);
      }
    }
    __syncthreads();
  }
}

cudaError_t launch_topk_kl(const void* teacher, const void* student, int64_t rows, int64_t V, int k, float* loss,
                           int32_t* idx, float* grad, int* status, int num_sms, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  static const cudaError_t attr = cudaFuncSetAttribute(topk_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)sizeof(KdShared));
  if (attr != cudaSuccess) return attr;
  const int64_t slots = 2 * (int64_t)num_sms;
  const int grid = (int)(rows < slots ? rows : slots);
  note_launch();
  topk_kl_kernel<<<grid, kKdThreads, sizeof(KdShared), s>>>(static_cast<const uint4*>(teacher), static_cast<const uint4*>(student),
                                             rows, V, k, loss, idx, grad, status);
  return cudaGetLastError();
}

}  // namespace nvfp4
