// Per-block NVFP4 arithmetic shared by the quantize, fake-quant and MoE
// row-quantize kernels: one lane owns one 16-element block of BF16 values.
//
// The format is the two-level scaling of "How is Qwen3.8-Flash-Next-NVFP4's
// NVFP4 quantization done?" (section "Core: W4A4 two-level scaling"): block
// scale s = E4M3(bmax / (M*g)) floored at 2^-9, element codes
// E2M1(x * RN(1/(g*s))); four_over_six (M = 4 or 6 by the block's squared
// error) follows Table 1 of "Developing Nemotron 3.5 Lightning NVFP4 with QAD
// using NVIDIA Model Optimizer".
#pragma once

#include "common.cuh"

namespace nvfp4 {

// One 32-byte store (two consecutive 16-byte vectors); p must be 32-byte
// aligned. A warp then writes whole 32-byte sectors in one instruction.
__device__ __forceinline__ void st_global_32b(uint4* p, uint4 a, uint4 b) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Lane-wise magnitude maximum of two BF16 pairs: |result| = max(|a|, |b|) per
// half (the sign bits hold the XOR of the inputs' signs and are masked off by
// every user); NaN in either input gives NaN.
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t m;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
  return m;
}

// Larger of the two 16-bit magnitudes (bits & 0x7FFF) of a BF16 pair.
__device__ __forceinline__ uint32_t mag_max_halves(uint32_t m2) {
  return max(m2 & 0x7FFFu, (m2 >> 16) & 0x7FFFu);
}

// Byte offset of scale (row, block column c) in the tiled layout; kgroups =
// K / 64 is the number of 4-scale tiles per 128-row tile row.
__device__ __forceinline__ int64_t scale_offset(int64_t row, int64_t c, int64_t kgroups) {
  return (((row >> 7) * kgroups + (c >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) +
         (c & 3);
}

// Two FP32 values in one 64-bit register (element 2j in the low half), for
// the packed sm_100 f32x2 instructions; each half is an IEEE FP32 operation.
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// BF16 pair (one 32-bit word) -> FP32 pair, exact.
__device__ __forceinline__ f32x2 bf16x2_unpack(uint32_t w) {
  return pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// Four FP32 pairs -> one word of eight E2M1 codes (element 2j in the low
// nibble of byte j). cvt.e2m1x2 puts its first source in the high nibble.
__device__ __forceinline__ uint32_t e2m1_pack4(f32x2 v0, f32x2 v1, f32x2 v2, f32x2 v3) {
  uint32_t out;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t.reg .f32 a0, a1, a2, a3, a4, a5, a6, a7;\n\t"
      "mov.b64 {a0, a1}, %1;\n\tmov.b64 {a2, a3}, %2;\n\tmov.b64 {a4, a5}, %3;\n\tmov.b64 {a6, a7}, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, a1, a0;\n\tcvt.rn.satfinite.e2m1x2.f32 q1, a3, a2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, a5, a4;\n\tcvt.rn.satfinite.e2m1x2.f32 q3, a7, a6;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(out)
      : "l"(v0), "l"(v1), "l"(v2), "l"(v3));
  return out;
}

// Byte of two E2M1 codes (low bits of `byte`) -> their values as an FP32 pair
// (exact, through the hardware E2M1 -> f16x2 conversion; low nibble -> low
// half). The byte is narrowed with cvt.u8 on purpose: unpacking a 32-bit word
// into four 8-bit registers with one vector mov did not yield bytes 2 and 3.
__device__ __forceinline__ f32x2 e2m1_byte_value(uint32_t byte) {
  float lo, hi;
  asm("{\n\t.reg .b8 t;\n\t.reg .b32 h;\n\t.reg .b16 a, b;\n\t"
      "cvt.u8.u32 t, %2;\n\tcvt.rn.f16x2.e2m1x2 h, t;\n\t"
      "mov.b32 {a, b}, h;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(byte));
  return pack2(lo, hi);
}

// One word of eight E2M1 codes -> their values as four FP32 pairs.
__device__ __forceinline__ void e2m1_unpack4(uint32_t w, f32x2* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = e2m1_byte_value(w >> (8 * j));
}

// Value of an E4M3 scale code (exact, through the hardware E4M3 -> f16x2
// conversion; the code sits in both bytes so either half holds it).
__device__ __forceinline__ float scale_value(uint32_t code) {
  float v;
  asm("{\n\t.reg .b16 t, a, b;\n\t.reg .b32 h;\n\tcvt.u16.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 h, t;\n\tmov.b32 {a, b}, h;\n\tcvt.f32.f16 %0, a;\n\t}"
      : "=f"(v)
      : "r"(code * 0x101u));
  return v;
}

// A lane's 16-element block as 8 raw BF16 words.
struct Raw16 {
  uint32_t w[8];
};

__device__ __forceinline__ void load_raw16(const uint4* x, int64_t vec, bool valid, Raw16& r) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (valid) {
    a = ld_stream(x + vec);
    b = ld_stream(x + vec + 1);
  }
  r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
  r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
}

// max |x| of the block as an FP32 value.
__device__ __forceinline__ float block_absmax(const Raw16& r) {
  uint32_t m = bmax2(bmax2(bmax2(r.w[0], r.w[1]), bmax2(r.w[2], r.w[3])),
                     bmax2(bmax2(r.w[4], r.w[5]), bmax2(r.w[6], r.w[7])));
  m = bmax2(m, __byte_perm(m, 0, 0x1032));  // both halves now hold the maximum
  return __uint_as_float((m & 0x7FFFu) << 16);
}

// One 16-element block: scale code, packed codes (two 32-bit words, element
// 2j in the low nibble of byte j) and, when requested, the dequantized values
// (pairs) and the block's squared error summed in element order.
struct Block {
  uint32_t sc;
  uint32_t q0, q1;
  f32x2 deq[8];
  float err;
};

// The block's 16 values as FP32 pairs (exact).
__device__ __forceinline__ void unpack_block(const Raw16& raw, f32x2 (&xs)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) xs[i] = bf16x2_unpack(raw.w[i]);
}

// Codes of a block under step d = g*s and its reciprocal r = RN(1/d), and on
// request the dequantized values and the squared error (sequential FP32 sum).
template <bool kDeq, bool kErr>
__device__ __forceinline__ void encode_block(const f32x2 (&xs)[8], float d, float r, Block& b) {
  const f32x2 rr = pack2(r, r);
  f32x2 sv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sv[i] = mul2(xs[i], rr);
  b.q0 = e2m1_pack4(sv[0], sv[1], sv[2], sv[3]);
  b.q1 = e2m1_pack4(sv[4], sv[5], sv[6], sv[7]);
  if (kDeq || kErr) {
    f32x2 v[8];
    e2m1_unpack4(b.q0, v);
    e2m1_unpack4(b.q1, v + 4);
    if (kErr) {
      // Scalar products here: with a packed multiply feeding the packed
      // subtraction below, the compiler was seen to fuse the two into one
      // fused multiply-add (one rounding of x - d*q where the method rounds
      // d*q first), which flips near-tie four_over_six choices.
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float lo, hi;
        unpack2(v[i], lo, hi);
        b.deq[i] = pack2(__fmul_rn(d, lo), __fmul_rn(d, hi));
      }
    } else {
      const f32x2 dd = pack2(d, d);
#pragma unroll
      for (int i = 0; i < 8; ++i) b.deq[i] = mul2(dd, v[i]);
    }
  }
  if (kErr) {
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const f32x2 df = sub2(xs[i], b.deq[i]);
      float lo, hi;
      unpack2(mul2(df, df), lo, hi);
      acc = __fadd_rn(acc, lo);  // element order: 2i, then 2i+1
      acc = __fadd_rn(acc, hi);
    }
    b.err = acc;
  } else {
    b.err = 0.0f;
  }
}

// Block scale for target magnitude mt (6 or 4), then the codes under it.
template <bool kDeq, bool kErr>
__device__ __forceinline__ void quantize_block(const f32x2 (&xs)[8], float bmax, float g, float mt, Block& b) {
  b.sc = block_scale_code(bmax, g, mt);
  const float d = __fmul_rn(g, scale_value(b.sc));
  encode_block<kDeq, kErr>(xs, d, __frcp_rn(d), b);
}

// Per-CTA table, built once the global scale g is known: the block step
// d = RN(g * s) and RN(1/d) for every E4M3 scale code 0..127 (code 0: d = 0,
// code 127 is NaN), and the scale-code divisors RN(6g), RN(4g). Lookups give
// exactly the values quantize_block computes.
struct StepTable {
  float d[128];
  float r[128];
  float div6, div4;
};

__device__ __forceinline__ StepTable& step_table() {
  __shared__ StepTable t;
  return t;
}

// Called by every thread of the CTA; ends with __syncthreads().
__device__ __forceinline__ void build_step_table(float g) {
  StepTable& t = step_table();
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    const float d = __fmul_rn(g, scale_value((uint32_t)c));
    t.d[c] = d;
    t.r[c] = __frcp_rn(d);
  }
  if (threadIdx.x == 0) {
    t.div6 = __fmul_rn(6.0f, g);
    t.div4 = __fmul_rn(4.0f, g);
  }
  __syncthreads();
}

// quantize_block with the CTA's step table (same results; kFour selects M = 4).
template <bool kDeq, bool kErr, bool kFour>
__device__ __forceinline__ void quantize_block_tab(const f32x2 (&xs)[8], float bmax, Block& b) {
  const StepTable& t = step_table();
  const uint32_t c = e4m3_code(__fdiv_rn(bmax, kFour ? t.div4 : t.div6));
  b.sc = c > 1u ? c : 1u;
  encode_block<kDeq, kErr>(xs, t.d[b.sc], t.r[b.sc], b);
}

template <bool kDeq, bool kErr>
__device__ __forceinline__ void quantize_block(const Raw16& raw, float bmax, float g, float mt, Block& b) {
  f32x2 xs[8];
  unpack_block(raw, xs);
  quantize_block<kDeq, kErr>(xs, bmax, g, mt, b);
}

// A warp's unit of work: 512 consecutive elements of one row ("chunk"), one
// 16-element block per lane. Chunks never straddle rows; a row of K elements
// has ceil(K/512) chunks and the last one may be partial. The row division is
// warp-uniform. Index type I: uint32_t ("narrow") when every element index,
// scale-byte offset and chunk-row division of the tensor fits 32-bit
// arithmetic (narrow_chunks on the host decides), else int64_t.
template <class I>
struct ChunkT {
  I row;
  int32_t col;        // this lane's first element within the row
  bool valid;         // col < K
  I vec;              // 16-byte vector index of the block's first 8 elements
};
using Chunk = ChunkT<int64_t>;

__device__ __forceinline__ Chunk chunk_at(int64_t ch, int32_t cpr, uint64_t cpr_magic, int64_t K, int lane) {
  Chunk c;
  // ch / cpr by multiplication with cpr_magic = ceil(2^64 / cpr) (exact for
  // ch * cpr < 2^64; division by an invariant integer, Granlund & Montgomery 1994)
  const uint64_t r = cpr == 1 ? (uint64_t)ch : __umul64hi((uint64_t)ch, cpr_magic);
  c.row = (int64_t)r;
  c.col = (int32_t)((uint64_t)ch - r * (uint64_t)cpr) * 512 + lane * 16;
  c.valid = c.col < K;
  c.vec = (c.row * K + c.col) >> 3;
  return c;
}

// Narrow form: cpr_magic = ceil(2^32 / cpr), exact for ch * cpr < 2^32.
__device__ __forceinline__ ChunkT<uint32_t> chunk_at_narrow(uint32_t ch, uint32_t cpr, uint32_t cpr_magic,
                                                            uint32_t K, int lane) {
  ChunkT<uint32_t> c;
  const uint32_t r = cpr == 1u ? ch : __umulhi(ch, cpr_magic);
  c.row = r;
  c.col = (int32_t)((ch - r * cpr) * 512u + (uint32_t)lane * 16u);
  c.valid = c.col < (int32_t)K;
  c.vec = (r * K + (uint32_t)c.col) >> 3;
  return c;
}

// Chunk `ch` in the index width I (cpr_magic: the 64-bit or 32-bit divisor
// magic to match).
template <class I>
__device__ __forceinline__ ChunkT<I> chunk_at_t(int64_t ch, int32_t cpr, uint64_t cpr_magic, int64_t K, int lane) {
  if constexpr (sizeof(I) == 4)
    return chunk_at_narrow((uint32_t)ch, (uint32_t)cpr, (uint32_t)cpr_magic, (uint32_t)K, lane);
  else
    return chunk_at(ch, cpr, cpr_magic, K, lane);
}

// Byte offset of the lane's block scale in the tiled layout.
__device__ __forceinline__ int64_t block_scale_offset(const ChunkT<int64_t>& c, int64_t K) {
  return scale_offset(c.row, c.col >> 4, K >> 6);
}
__device__ __forceinline__ uint32_t block_scale_offset(const ChunkT<uint32_t>& c, int64_t K) {
  const uint32_t row = c.row, cb = (uint32_t)c.col >> 4, kgroups = (uint32_t)(K >> 6);
  return (((row >> 7) * kgroups + (cb >> 2)) << 9) + ((row & 31u) << 4) + (((row >> 5) & 3u) << 2) + (cb & 3u);
}

}  // namespace nvfp4
