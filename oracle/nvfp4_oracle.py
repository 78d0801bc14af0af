"""Plain CPU oracle for NVFP4 W4A4 quantization, fake-quant, the block-scaled
W4A4 GEMM and the routed-expert (MoE) pipeline.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it. It shares no code,
table or constant generator with the CUDA library.

Pages cited (titles as printed on each page):

* [QF-NVFP4]   "How is Qwen3.8-Flash-Next-NVFP4's NVFP4 quantization done?
               W4A4 two-level scaling and why only routed experts are quantized"
               -- sections "Core: W4A4 two-level scaling" (level 1 block scale,
               level 2 global scale, "why 4.5 bit", "the A4 side: dynamic
               activations") and "Evidence chain" (scale audit).
* [NEMO-QAD]   "Developing Nemotron 3.5 Lightning NVFP4 with QAD using NVIDIA
               Model Optimizer" -- Table 1 (PTQ recipes: max / MSE /
               four_over_six) and "Quantization scale handling during QAD"
               (dynamic vs frozen scales, Figure 2).
* [QWEN36-QAD] "Model-Optimizer in practice: recovering Qwen3.6-35B-A3B W4A4
               NVFP4 accuracy with quantization-aware distillation" --
               "Why W4A4 rather than W4A16", "2. PTQ" (routed experts,
               fused gate/up/down projections) and "QAD" (top-k logit KD).

Readings taken where the pages are silent:

R1  E2M1 and E4M3 conversions round to nearest, ties to the even code, and
    saturate (E2M1 to +-6, E4M3 to 448). The sign of an E2M1 code is the sign
    bit of the scaled value, so -0.0 and small negatives give code 0x8.
R2  The global scale is g = amax / (6 * 448) = amax / 2688 in FP32, so the
    block holding the tensor's amax gets block scale exactly 448 -- the
    maximum the [QF-NVFP4] scale audit reports. amax == 0 gives g = 1.
R3  Block scale s = E4M3(bmax / (M * g)), M = 6, with FP32 product and
    quotient, floored at the smallest positive E4M3 value 2^-9 so that every
    stored scale is positive, as the [QF-NVFP4] audit requires.
R4  Elements are scaled by the FP32 reciprocal r = 1 / (g * s), computed once
    per block: v = x * r, code = E2M1(v).
R5  Two codes per byte, element 2j in the low nibble of byte j.
R6  four_over_six: candidates M = 6 and M = 4 (same g); err_M is the block's
    squared error in the original value domain, FP32, summed over the 16
    elements in index order; M = 4 wins only if err_4 < err_6 (tie -> 6).
R7  Fake-quant output is BF16(g * s * q) with FP32 products, round to nearest
    even. Frozen mode takes g*, s* as given (codes still saturate at +-6).
R8  The GEMM reference is C = ga * gb * sum_k (sa qa)(sb qb) in FP64 over the
    exactly dequantized operands; S = sum_k |a_k b_k| sets the tolerance.
R9  MoE: routing is input; pairs are stably sorted by expert; each expert's
    rows are quantized with that expert's own dynamic g; h = SiLU(gate) * up
    (gate = first I columns of gate_up) rounded to BF16; h is quantized per
    expert; the weighted combine is a plain sum.
R11 QAD backward through the simulated quantization ([NEMO-QAD] Figure 2:
    "gradient back to the FP weights through the loss"; the estimator is not
    named): a straight-through estimator clipped to the quantizer's range --
    dL/dx = dL/dy where |x * r| <= 6 for the block's r = RN(1/(g*s)) (FP32
    product), else 0. Rounding is passed straight through; saturation is not.
    The scales are those of the forward: recomputed (dynamic) or frozen.
R12 Top-k logit KL ([QWEN36-QAD] "QAD": --logit_kl_topk 4096 restricts the KD loss
    to the teacher's top-4096 vocabulary entries; the loss compares teacher
    and student logits element-wise over the vocabulary): per row, the k
    entries with the largest teacher logits (ties to the lower index) form
    the set; teacher and student distributions are softmax over that set
    (temperature 1, the pages give none); loss = KL(teacher || student) =
    sum p_t (log p_t - log p_s); its gradient w.r.t. the student logits on
    the set is p_s - p_t (0 elsewhere).
R10 MSE calibration ([NEMO-QAD] Table 1 "MSE"; "Quantization scale handling
    during QAD": MSE reaches its scales by a search that minimises the
    quantization error): for each block, every positive finite E4M3 code
    (1..126, i.e. 2^-9 .. 448) is a candidate scale under the same g; the
    block keeps the candidate with the lowest FP32 squared error computed as
    in R6; ties keep the lowest code.
"""
from __future__ import annotations

import numpy as np

BLOCK = 16                 # elements per block scale [QF-NVFP4, level 1]
E2M1_MAX = 6.0             # largest E2M1 magnitude
E4M3_MAX = 448.0           # largest finite E4M3 value
E4M3_MAX_CODE = 126        # its code (0x7F is NaN)
GLOBAL_DIVISOR = np.float32(6.0 * 448.0)   # R2: 2688


# ----------------------------------------------------------------------------
# Element formats. [QF-NVFP4 "Core: W4A4 two-level scaling", level 1]:
# elements are E2M1 (num_bits [2,1]); block scales are E4M3 (scale_bits [4,3]).
# ----------------------------------------------------------------------------

def e2m1_decode_table() -> np.ndarray:
    """Value of each 4-bit E2M1 code 0..15, from the bit layout.

    Bit 3 is the sign, bits 2..1 the exponent (bias 1), bit 0 the mantissa.
    Exponent field 0 is subnormal: value = m * 2^-1.
    """
    out = np.zeros(16, dtype=np.float64)
    for code in range(16):
        sign = -1.0 if code & 0x8 else 1.0
        e = (code >> 1) & 0x3
        m = code & 0x1
        if e == 0:
            mag = m * 0.5
        else:
            mag = (1.0 + m / 2.0) * 2.0 ** (e - 1)
        out[code] = sign * mag
    return out


def e4m3_decode_table() -> np.ndarray:
    """Value of each non-negative E4M3 code 0..126 (0x7F is NaN, excluded).

    4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal:
    value = m * 2^-9.
    """
    out = np.zeros(127, dtype=np.float64)
    for code in range(127):
        e = code >> 3
        m = code & 0x7
        if e == 0:
            out[code] = m * 2.0 ** -9
        else:
            out[code] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_E2M1_MAG = e2m1_decode_table()[:8]           # 0, .5, 1, 1.5, 2, 3, 4, 6
_E4M3_VAL = e4m3_decode_table()               # increasing with the code


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """E2M1 code of each FP32 value: nearest magnitude, tie -> even code,
    |v| >= 6 saturates to 6, sign bit copied from v (R1)."""
    v = np.asarray(v, dtype=np.float32)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    chunk = 1 << 20
    for lo in range(0, flat.size, chunk):
        part = flat[lo:lo + chunk]
        mag = np.abs(part).astype(np.float64)
        dist = np.abs(mag[:, None] - _E2M1_MAG[None, :])      # exact in FP64
        best = dist.min(axis=1)
        idx = np.argmin(dist, axis=1)                          # lowest index on a tie
        # a tie is between two neighbours; move to the even one
        nxt = np.minimum(idx + 1, 7)
        tie_up = (idx % 2 == 1) & (idx < 7) & (dist[np.arange(idx.size), nxt] == best)
        idx = np.where(tie_up, idx + 1, idx)
        idx = np.where(mag >= E2M1_MAX, 7, idx)                # saturation (also +-inf)
        sign = np.signbit(part).astype(np.uint8) << 3
        out[lo:lo + chunk] = idx.astype(np.uint8) | sign
    return out.reshape(v.shape)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return e2m1_decode_table()[np.asarray(codes, dtype=np.int64)]


def e4m3_encode(t: np.ndarray) -> np.ndarray:
    """E4M3 code of each non-negative FP32 value: nearest, tie -> even code,
    values >= 448 saturate to 448 (R1, satfinite)."""
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("block scale arguments must be non-negative numbers")
    hi = np.searchsorted(_E4M3_VAL, t, side="left")            # VAL[hi-1] < t <= VAL[hi]
    hi_c = np.minimum(hi, 126)
    lo_c = np.maximum(hi - 1, 0)
    d_lo = t - _E4M3_VAL[lo_c]
    d_hi = _E4M3_VAL[hi_c] - t
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi_c % 2 == 0))
    code = np.where(pick_hi, hi_c, lo_c)
    code = np.where(t >= E4M3_MAX, 126, code)
    code = np.where(t == 0, 0, code)
    return code.astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    if np.any(c > 126):
        raise ValueError("E4M3 code 0x7F (NaN) or a negative code is not a valid block scale")
    return _E4M3_VAL[c]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round FP32 values to BF16 (nearest, ties to even); returns FP32 holding
    the BF16 value. Finite inputs only."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32)


def bf16_round_f64(x: np.ndarray) -> np.ndarray:
    """Round FP64 values straight to the nearest BF16 (ties to even), no
    intermediate FP32 rounding. Returns FP64 holding the BF16 value."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                 # 8 significant bits for BF16
    r = np.round(scaled)                    # numpy rounds half to even
    return np.ldexp(r, e - 8)


# ----------------------------------------------------------------------------
# Level 2: global scale. [QF-NVFP4 "Core: W4A4 two-level scaling", level 2;
# "Evidence chain": every scale finite and positive, largest 448.0]
# ----------------------------------------------------------------------------

def global_scale(x: np.ndarray) -> tuple[np.float32, np.float32]:
    """(g, amax) of a tensor: amax = max |x| (exact), g = amax / 2688 in FP32
    (R2); amax == 0 gives g = 1. Non-finite input raises."""
    x = np.asarray(x, dtype=np.float32)
    if x.size == 0:
        return np.float32(1.0), np.float32(0.0)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    amax = np.float32(np.max(np.abs(x)))
    if amax == 0:
        return np.float32(1.0), amax
    g = np.float32(amax / GLOBAL_DIVISOR)
    return g, amax


# ----------------------------------------------------------------------------
# Level 1: block scale and element codes, max and four_over_six calibration.
# ----------------------------------------------------------------------------

def block_scale_codes(bmax: np.ndarray, g: np.float32, m_target: float) -> np.ndarray:
    """E4M3 code of s = E4M3(bmax / (M * g)), floored at 2^-9 (R3)."""
    denom = np.float32(m_target) * np.float32(g)               # FP32 product
    t = np.asarray(bmax, dtype=np.float32) / denom             # FP32 quotient
    code = e4m3_encode(t)
    return np.maximum(code, 1).astype(np.uint8)                # code 1 == 2^-9


def _encode_blocks(blocks: np.ndarray, g: np.float32, s_codes: np.ndarray):
    """Codes and FP32 squared error of blocks [..., 16] under block scales."""
    s = e4m3_decode(s_codes).astype(np.float32)
    d = np.float32(g) * s                                      # R4: d = g * s
    r = np.float32(1.0) / d                                    # FP32 reciprocal
    v = blocks * r[..., None]                                  # FP32 products
    q = e2m1_encode(v)
    deq = d[..., None] * e2m1_decode(q).astype(np.float32)     # FP32 products
    diff = blocks - deq
    sq = diff * diff
    err = np.zeros(blocks.shape[:-1], dtype=np.float32)
    for i in range(BLOCK):                                     # R6: index order
        err = err + sq[..., i]
    return q, err


def quantize(x: np.ndarray, mode: str = "max", g: np.float32 | None = None):
    """NVFP4-quantize a row-major [rows, K] tensor along its last dimension.

    Returns a dict with
      codes  uint8 [rows, K]       4-bit codes, one per element (unpacked)
      scales uint8 [rows, K/16]    E4M3 block-scale codes
      g      float32               global scale used
      choice uint8 [rows, K/16]    0 -> M=6 target, 1 -> M=4 (four_over_six)
      err    float32 [rows, K/16]  squared error of the kept candidate

    mode "max": every block targets M=6 ([NEMO-QAD] Table 1 "max";
    [QF-NVFP4] dynamic activations use the same rule).
    mode "four_over_six": per block keep the M=6 or M=4 scale, whichever
    gives the lower block error ([NEMO-QAD] Table 1, four_over_six).
    mode "mse": per block keep, of all 126 positive finite E4M3 scales, the
    one with the lowest block error (R10; [NEMO-QAD] Table 1, MSE).
    g: a static global scale; None computes it from the tensor (dynamic).
    """
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2 or x.shape[1] % BLOCK:
        raise ValueError("x must be [rows, K] with K a multiple of 16")
    rows, K = x.shape
    if g is None:
        g, _ = global_scale(x)
    g = np.float32(g)
    blocks = x.reshape(rows, K // BLOCK, BLOCK)
    bmax = np.max(np.abs(blocks), axis=2) if K else np.zeros((rows, 0), np.float32)
    s6 = block_scale_codes(bmax, g, 6.0)
    q6, e6 = _encode_blocks(blocks, g, s6)
    if mode == "max":
        return dict(codes=q6.reshape(rows, K), scales=s6, g=g,
                    choice=np.zeros_like(s6), err=e6)
    if mode == "mse":
        best_s = np.ones(s6.shape, np.uint8)
        best_q, best_e = _encode_blocks(blocks, g, best_s)
        for c in range(2, E4M3_MAX_CODE + 1):                   # R10: increasing code
            sc = np.full(s6.shape, c, np.uint8)
            q, e = _encode_blocks(blocks, g, sc)
            better = e < best_e                                  # ties keep the lower code
            best_q = np.where(better[..., None], q, best_q)
            best_s = np.where(better, sc, best_s).astype(np.uint8)
            best_e = np.where(better, e, best_e)
        return dict(codes=best_q.reshape(rows, K), scales=best_s, g=g,
                    choice=np.zeros_like(s6), err=best_e)
    if mode != "four_over_six":
        raise ValueError(f"unknown mode {mode!r}")
    s4 = block_scale_codes(bmax, g, 4.0)
    q4, e4 = _encode_blocks(blocks, g, s4)
    pick4 = e4 < e6                                            # tie keeps M=6
    codes = np.where(pick4[..., None], q4, q6)
    scales = np.where(pick4, s4, s6).astype(np.uint8)
    err = np.where(pick4, e4, e6)
    return dict(codes=codes.reshape(rows, K), scales=scales, g=g,
                choice=pick4.astype(np.uint8), err=err)


def dequantize(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    """FP32 value g*s*q of every element: d = g*s, then d*q, both FP32 (R7)."""
    rows, K = codes.shape
    d = np.float32(g) * e4m3_decode(scales).astype(np.float32)
    q = e2m1_decode(codes).astype(np.float32).reshape(rows, K // BLOCK, BLOCK)
    return (d[..., None] * q).reshape(rows, K)


def fake_quant(x: np.ndarray, mode: str = "max", g_frozen=None, scales_frozen=None) -> np.ndarray:
    """Quantize-dequantize forward of QAD's simulated quantization, BF16 out.

    Dynamic ([NEMO-QAD] "Quantization scale handling during QAD", top lane):
    g and s are recomputed from x. Frozen (bottom lane): g*, s* are taken as
    given and only the codes follow x; they saturate at +-6 (R7).
    Returns FP32 arrays holding BF16 values.
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    if (g_frozen is None) != (scales_frozen is None):
        raise ValueError("frozen mode needs both g and the block scales")
    if g_frozen is None:
        qz = quantize(x, mode)
        codes, scales, g = qz["codes"], qz["scales"], qz["g"]
    else:
        g = np.float32(g_frozen)
        scales = np.asarray(scales_frozen, dtype=np.uint8).reshape(rows, K // BLOCK)
        q, _ = _encode_blocks(x.reshape(rows, K // BLOCK, BLOCK), g, scales)
        codes = q.reshape(rows, K)
    return bf16_round(dequantize(codes, scales, g))


def fake_quant_backward(x: np.ndarray, grad_y: np.ndarray, mode: str = "max", g_frozen=None,
                        scales_frozen=None) -> np.ndarray:
    """Gradient of the QAD fake-quant w.r.t. x (R11): grad_y where the
    element is inside its block's quantizer range |x * RN(1/(g*s))| <= 6, else
    0. Scales as in ``fake_quant`` (dynamic: from x with ``mode``; frozen:
    given). Returns FP32 arrays holding the (BF16) gradient values."""
    x = np.asarray(x, dtype=np.float32)
    gy = np.asarray(grad_y, dtype=np.float32)
    rows, K = x.shape
    if (g_frozen is None) != (scales_frozen is None):
        raise ValueError("frozen mode needs both g and the block scales")
    if g_frozen is None:
        qz = quantize(x, mode)
        scales, g = qz["scales"], qz["g"]
    else:
        g = np.float32(g_frozen)
        scales = np.asarray(scales_frozen, dtype=np.uint8).reshape(rows, K // BLOCK)
    d = np.float32(g) * e4m3_decode(scales).astype(np.float32)          # R4
    r = np.float32(1.0) / d
    v = x.reshape(rows, K // BLOCK, BLOCK) * r[..., None]               # FP32 products
    inside = (np.abs(v) <= np.float32(E2M1_MAX)).reshape(rows, K)
    return np.where(inside, gy, np.float32(0.0)).astype(np.float32)


def topk_kl(teacher: np.ndarray, student: np.ndarray, k: int):
    """Top-k logit KL distillation loss per row (R12), in FP64.

    teacher, student: [rows, V] logits (BF16 values). Returns a dict with
      loss  float64 [rows]      KL(p_t || p_s) over the teacher's top-k set
      idx   int64 [rows, k]     the set, ascending vocabulary index
      grad  float64 [rows, k]   d loss / d student logit at idx
      lse_t, lse_s float64 [rows]  log-sum-exp of each side over the set
    """
    t = np.asarray(teacher, dtype=np.float64)
    s = np.asarray(student, dtype=np.float64)
    rows, V = t.shape
    if not 1 <= k <= V:
        raise ValueError("need 1 <= k <= V")
    out = dict(loss=np.empty(rows), idx=np.empty((rows, k), np.int64), grad=np.empty((rows, k)),
               lse_t=np.empty(rows), lse_s=np.empty(rows))
    for r in range(rows):
        order = np.argsort(-t[r], kind="stable")   # descending; equal logits keep index order
        idx = np.sort(order[:k])
        tt, ss = t[r, idx], s[r, idx]
        mt, ms = tt.max(), ss.max()
        lse_t = mt + np.log(np.sum(np.exp(tt - mt)))
        lse_s = ms + np.log(np.sum(np.exp(ss - ms)))
        lpt, lps = tt - lse_t, ss - lse_s
        pt = np.exp(lpt)
        out["loss"][r] = np.sum(pt * (lpt - lps))
        out["idx"][r] = idx
        out["grad"][r] = np.exp(lps) - pt
        out["lse_t"][r], out["lse_s"][r] = lse_t, lse_s
    return out


# ----------------------------------------------------------------------------
# Storage: packed codes and the tiled block-scale layout.
# ----------------------------------------------------------------------------

def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, K] 4-bit codes -> [rows, K/2] bytes; element 2j in the low
    nibble of byte j (R5). [QF-NVFP4 "Evidence chain": codes stored as U8]"""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def scale_tile_bytes(rows: int, K: int) -> int:
    """Bytes of the tiled scale layout: 512-byte tiles of 128 rows x 4 scales."""
    return ((rows + 127) // 128) * ((K // BLOCK + 3) // 4) * 512


def scales_to_tiled(scales: np.ndarray) -> np.ndarray:
    """Row-major [rows, K/16] scales -> the tiled layout the block-scaled MMA
    reads: tile (r // 128, c // 4), tiles ordered row-tile-major; inside a tile
    the byte of (r, c) sits at (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4.
    Padding bytes are zero."""
    rows, nb = scales.shape
    kt = (nb + 3) // 4
    out = np.zeros(scale_tile_bytes(rows, nb * BLOCK), dtype=np.uint8)
    for r in range(rows):
        for c in range(nb):
            tile = (r // 128) * kt + c // 4
            off = tile * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
            out[off] = scales[r, c]
    return out


def scales_from_tiled(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Inverse of scales_to_tiled (vectorised index arithmetic of the same rule)."""
    nb = K // BLOCK
    kt = (nb + 3) // 4
    r = np.arange(rows)[:, None]
    c = np.arange(nb)[None, :]
    off = ((r // 128) * kt + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return np.asarray(tiled, dtype=np.uint8)[off]


def storage_bits_per_element(K: int) -> float:
    """Bits per element of codes + block scales, without tile padding:
    (16*4 + 8)/16 = 4.5 [QF-NVFP4 "why 4.5 bit"]."""
    code_bytes = K // 2
    scale_bytes = K // BLOCK
    return 8.0 * (code_bytes + scale_bytes) / K


# ----------------------------------------------------------------------------
# W4A4 GEMM reference. [QWEN36-QAD "Why W4A4 rather than W4A16": only FP4
# activations reach the FP4 tensor cores]
# ----------------------------------------------------------------------------

def dequantize_f64(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """s * q per element in FP64 (exact; the global scale is left out)."""
    rows, K = codes.shape
    s = e4m3_decode(scales)
    q = e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK)
    return (s[..., None] * q).reshape(rows, K)


def gemm_reference(a_codes, a_scales, ga, b_codes, b_scales, gb, rows=None):
    """C = ga*gb * A_deq @ B_deq^T in FP64 and S = |ga*gb| * |A_deq| @ |B_deq|^T.

    a_codes [M, K] / b_codes [N, K] are unpacked 4-bit codes, *_scales the
    row-major E4M3 codes. ``rows`` optionally restricts to a subset of A's rows.
    """
    A = dequantize_f64(a_codes, a_scales)
    if rows is not None:
        A = A[rows]
    B = dequantize_f64(b_codes, b_scales)
    alpha = float(np.float64(ga) * np.float64(gb))
    C = alpha * (A @ B.T)
    S = abs(alpha) * (np.abs(A) @ np.abs(B).T)
    return C, S


def gemm_tolerance(C_ref: np.ndarray, S: np.ndarray) -> np.ndarray:
    """|C - C_ref| bound: 1e-4 * sum|a b| for accumulation, plus BF16 output
    rounding (unit roundoff 2^-8 of the value)."""
    return 1e-4 * S * (1.0 + 2.0 ** -8) + 2.0 ** -8 * np.abs(C_ref)


# ----------------------------------------------------------------------------
# Routed-expert MoE. [QWEN36-QAD "2. PTQ": routed experts are 99.2% of the
# quantized tensors, fused gate/up and down projections; QF-NVFP4: top-k
# routing, dynamic activation quantization]
# ----------------------------------------------------------------------------

def moe_permutation(topk_ids: np.ndarray, num_experts: int, pad: int = 128):
    """Stable sort of (token, slot) pairs by expert.

    Returns (order, counts, offsets): order[p] = flat pair index t*k + j of the
    p-th pair in expert-major order; counts[e] = pairs routed to e;
    offsets[e] = first padded row of expert e (segments padded to ``pad``).
    """
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    order = []
    for e in range(num_experts):                    # stable: increasing pair index
        order.extend(np.nonzero(flat == e)[0].tolist())
    order = np.asarray(order, dtype=np.int64)
    counts = np.bincount(flat, minlength=num_experts).astype(np.int64)
    padded = (counts + pad - 1) // pad * pad
    offsets = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
    return order, counts, offsets


def silu_f64(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def moe_reference(x, topk_ids, topk_w, w13, w2, experts=None):
    """Reference routed-expert forward, stage by stage (R9).

    x [T, H] FP32 (BF16 values); topk_ids/topk_w [T, k]; w13[e] and w2[e] are
    dicts from ``quantize`` of expert e's gate_up [2I, H] and down [H, I]
    weights. ``experts`` restricts the computation to a subset (the output
    then only holds those experts' contributions). Returns a dict of stages.
    """
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    k = topk_ids.shape[1]
    E = len(w13)
    order, counts, offsets = moe_permutation(topk_ids, E)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    out = np.zeros((T, H), dtype=np.float64)
    out_S = np.zeros((T, H), dtype=np.float64)
    stages = {}
    for e in (range(E) if experts is None else experts):
        pairs = order[starts[e]:starts[e] + counts[e]]
        if pairs.size == 0:
            continue
        tok = pairs // k
        rows = x[tok]
        xq = quantize(rows, "max")                              # per-expert dynamic g
        gu, gu_S = gemm_reference(xq["codes"], xq["scales"], xq["g"],
                                  w13[e]["codes"], w13[e]["scales"], w13[e]["g"])
        inter = gu.shape[1] // 2
        gate, up = gu[:, :inter], gu[:, inter:]
        h = bf16_round_f64(silu_f64(gate) * up)
        hq = quantize(h.astype(np.float32), "max")
        y, y_S = gemm_reference(hq["codes"], hq["scales"], hq["g"],
                                w2[e]["codes"], w2[e]["scales"], w2[e]["g"])
        w = np.asarray(topk_w, dtype=np.float64).reshape(-1)[pairs]
        np.add.at(out, tok, w[:, None] * y)
        np.add.at(out_S, tok, np.abs(w)[:, None] * y_S)
        stages[e] = dict(pairs=pairs, xq=xq, gate_up=gu, gate_up_S=gu_S, h=h,
                         hq=hq, y=y, y_S=y_S)
    return dict(out=out, out_S=out_S, order=order, counts=counts,
                offsets=offsets, stages=stages)
