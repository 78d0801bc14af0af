/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 library.
 *
 * The operations follow the NVFP4 two-level scaling described in
 * "How is Qwen3.8-Flash-Next-NVFP4's NVFP4 quantization done? W4A4 two-level
 * scaling and why only routed experts are quantized" (section "Core: W4A4
 * two-level scaling"): E2M1 element codes, one E4M3 block scale per 16
 * contiguous elements of the last dimension, one FP32 global scale per tensor,
 * 4.5 bits per element. Calibration modes follow Table 1 of "Developing
 * Nemotron 3.5 Lightning NVFP4 with QAD using NVIDIA Model Optimizer" (max and
 * four_over_six) and its section "Quantization scale handling during QAD"
 * (dynamic and frozen scales). The W4A4 GEMM is the operation that "Why W4A4
 * rather than W4A16" in "Model-Optimizer in practice: recovering
 * Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD" says only FP4 activations can
 * reach on Blackwell tensor cores.
 *
 * Conventions for every call
 * --------------------------
 *  - Pointers are DEVICE pointers unless a comment says otherwise. Calls are
 *    asynchronous on `stream` (0 = legacy default stream).
 *  - The caller owns and allocates every buffer. The library allocates no
 *    device memory; scratch comes from a caller-provided `workspace` whose
 *    size is returned by the matching *_workspace_bytes query.
 *  - Return value: an nvfp4_status checked synchronously on the host
 *    (argument validation, device gate, launch errors). Conditions found on
 *    the device (non-finite input, a bounded wait that ran out) are recorded
 *    in a library-owned device status word; read it with
 *    nvfp4_get_device_status(), which synchronizes `stream`.
 *  - Bounds-checking build: libnvfp4_debug.so (built with
 *    -DNVFP4_DEBUG_BOUNDS) exports the same calls; its kernels check every
 *    computed global index against the extent of its buffer, record
 *    NVFP4_ERR_BOUNDS in the device status word on a violation and skip that
 *    access (no trap). The regular library carries no checks.
 *  - Requirements: K % 64 == 0; every pointer 16-byte aligned; inputs
 *    row-major and contiguous. The device must be sm_100 (B200-class);
 *    other devices get NVFP4_ERR_UNSUPPORTED_DEVICE (the hardware gate of
 *    "check what your card supports before choosing FP8 / W4A8 / NVFP4").
 *
 * Storage formats
 * ---------------
 *  codes   [rows][K/2] bytes, two E2M1 codes per byte, element 2j in the low
 *          nibble of byte j. Code bit 3 is the sign.
 *  scales  E4M3 block scales in the tiled layout the block-scaled MMA reads:
 *          512-byte tiles of 128 rows x 4 scales (64 elements of K), tiles
 *          ordered row-tile-major (tile = (r/128) * (K/64) + c/4), and inside
 *          a tile the scale of (row r, block c) at byte
 *          (r%32)*16 + ((r%128)/32)*4 + c%4. Rows are padded to a multiple of
 *          128 with zero bytes. Size: nvfp4_scale_bytes(rows, K).
 *  g       one FP32 global scale per tensor: g = amax / (6 * 448).
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same handle as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,        /* bad pointer, size, alignment or mode */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 2, /* not an sm_100 device */
  NVFP4_ERR_CUDA = 3,               /* a CUDA runtime call failed */
  NVFP4_ERR_WORKSPACE = 4,          /* workspace missing or too small */
  NVFP4_ERR_NONFINITE_INPUT = 5,    /* device: amax of an input is Inf/NaN */
  NVFP4_ERR_TIMEOUT = 6,            /* device: a bounded wait ran out */
  NVFP4_ERR_TOO_LARGE = 7,          /* input larger than nvfp4_quantize_noalloc's static scratch */
  NVFP4_ERR_BOUNDS = 8              /* device, bounds-checking build only: a computed global index
                                       fell outside its buffer; that access was skipped */
} nvfp4_status;

typedef enum {
  NVFP4_MODE_MAX = 0,           /* every block targets the E2M1 maximum 6 */
  NVFP4_MODE_FOUR_OVER_SIX = 1, /* per block, target 6 or 4, lower block MSE */
  NVFP4_MODE_MSE = 2            /* per block, the E4M3 scale (of all 126) with the
                                   lowest block squared error, ties to the lowest
                                   code: MSE calibration, Table 1 of "Developing
                                   Nemotron 3.5 Lightning NVFP4 with QAD using
                                   NVIDIA Model Optimizer". nvfp4_quantize only. */
} nvfp4_mode;

/* Library version (major*10000 + minor*100 + patch). Host only. */
int nvfp4_version(void);

/* Hardware gate for the CURRENT device: NVFP4_OK on sm_100, else
 * NVFP4_ERR_UNSUPPORTED_DEVICE (or NVFP4_ERR_CUDA if no device). */
nvfp4_status nvfp4_check_device(void);

/* Human-readable name of a status code (static string). Host only. */
const char* nvfp4_status_string(nvfp4_status s);

/* Bytes of the tiled block-scale buffer for a [rows x K] tensor:
 * ceil(rows/128) * (K/64) * 512. Returns 0 if K % 64 != 0. Host only. */
size_t nvfp4_scale_bytes(int64_t rows, int64_t K);

/* Workspace bytes nvfp4_quantize / nvfp4_fake_quant /
 * nvfp4_fake_quant_backward need to compute a dynamic global scale for an
 * [M x K] input (0 is never returned). The workspace holds a grid-wide
 * barrier whose arrival counter assumes one CTA per SM of one device:
 *  - zero-fill it once before its first use; every completed call leaves it
 *    ready for the next;
 *  - after a call that reported NVFP4_ERR_TIMEOUT, zero-fill it again;
 *  - use one workspace per device (never hand the same buffer to calls on
 *    devices with different SM counts);
 *  - calls that share a workspace must be ordered on the GPU (one stream, or
 *    events between streams); give each stream its own workspace otherwise.
 * Host only. */
size_t nvfp4_quantize_workspace_bytes(int64_t M, int64_t K);

/*
 * nvfp4_quantize -- NVFP4 quantization of x [M x K] BF16 along K.
 *   Two-level scaling ("Core: W4A4 two-level scaling", levels 1 and 2):
 *   g = amax/2688 (or *g_in when given: a static, calibrated global scale);
 *   per block of 16, s = E4M3(bmax / (Mt * g)) floored at 2^-9, Mt = 6
 *   (mode MAX) or the better of 6 and 4 by block squared error (mode
 *   FOUR_OVER_SIX, tie -> 6), or (mode MSE, Table 1 "MSE" of "Developing
 *   Nemotron 3.5 Lightning NVFP4 with QAD using NVIDIA Model Optimizer")
 *   the E4M3 scale, of all 126 positive finite ones, with the lowest block
 *   squared error (ties -> lowest code); codes = E2M1(x * (1 / (g * s)));
 *   every rounding is to nearest even and saturating (E2M1 at +-6, E4M3 at
 *   448).
 *   Dynamic activations use g_in = NULL ("the A4 side: dynamic activations");
 *   static weights pass a precomputed g_in or let the call compute it.
 * x           [M][K] BF16, device.
 * g_in        nullable device FP32 scalar: static global scale.
 * codes       out [M][K/2] bytes.
 * scales      out nvfp4_scale_bytes(M, K) bytes (tiled layout, padding zeroed).
 * g_out       out device FP32 scalar: the global scale used.
 * fos_choice  nullable out [M][K/16] bytes: 1 where the block kept the M=4
 *             scale, else 0 (always 0 in modes MAX and MSE).
 * workspace   >= nvfp4_quantize_workspace_bytes(M, K) bytes when g_in is
 *             NULL (zero-filled before its first use, see above); may be
 *             NULL when g_in is given. Calls that share one workspace must
 *             be ordered on the GPU (same stream).
 * A dynamic call is a single cooperative launch of one CTA per SM: each CTA
 *   reduces the amax of its slice while keeping most of the slice in shared
 *   memory, the CTAs meet at a grid-wide barrier, then quantize.
 * M may be 0 (nothing is written except g_out = 1 for a dynamic call).
 * Device status: NVFP4_ERR_NONFINITE_INPUT if amax is Inf/NaN (outputs are
 * then unspecified); NVFP4_ERR_TIMEOUT if the grid barrier wait ran out.
 */
nvfp4_status nvfp4_quantize(const void* x, int64_t M, int64_t K, nvfp4_mode mode,
                            const float* g_in, uint8_t* codes, uint8_t* scales,
                            float* g_out, uint8_t* fos_choice, void* workspace,
                            size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_fake_quant -- quantize-dequantize forward of QAD's simulated
 *   quantization ("Quantization scale handling during QAD", Figure 2):
 *   y = BF16(g * s * q) elementwise, with q, s, g as in nvfp4_quantize.
 *   Scale sources:
 *     g_frozen = NULL, scales_frozen = NULL : dynamic lane, g and s
 *        recomputed from x (mode selects MAX / FOUR_OVER_SIX);
 *     g_frozen set, scales_frozen = NULL : static g, block scales from x;
 *     both set : frozen lane, s* and g* as captured by an earlier
 *        nvfp4_quantize (tiled layout); codes saturate at +-6 when x has
 *        drifted past the frozen range. mode is ignored.
 * x, y        [M][K] BF16, device (y may not alias x).
 * workspace   as for nvfp4_quantize (needed only when g_frozen is NULL).
 */
nvfp4_status nvfp4_fake_quant(const void* x, int64_t M, int64_t K, nvfp4_mode mode,
                              const float* g_frozen, const uint8_t* scales_frozen,
                              void* y, void* workspace, size_t workspace_bytes,
                              nvfp4_stream_t stream);

/*
 * nvfp4_gemm -- W4A4 block-scaled GEMM on tcgen05 tensor cores:
 *   C[m][n] = BF16( (ga*gb) * sum_k (sa*qa)[m][k] * (sb*qb)[n][k] ),
 *   FP32 accumulation in tensor memory, global-scale product and BF16
 *   rounding fused in the epilogue ("Why W4A4 rather than W4A16").
 * Aq, As, ga  activations: codes [M][K/2], tiled scales, FP32 global scale.
 * Bq, Bs, gb  weights: codes [N][K/2], tiled scales, FP32 global scale.
 * C           out [M][N] BF16 row-major.
 * Requirements: M >= 0, N % 16 == 0, K % 64 == 0, K > 0.
 * Device status: NVFP4_ERR_TIMEOUT if a pipeline wait ran out (C then
 * unspecified; the context stays usable).
 */
nvfp4_status nvfp4_gemm(const uint8_t* Aq, const uint8_t* As, const float* ga,
                        const uint8_t* Bq, const uint8_t* Bs, const float* gb,
                        int64_t M, int64_t N, int64_t K, void* C,
                        nvfp4_stream_t stream);

/*
 * nvfp4_topk_kl -- top-k logit KL distillation loss per row ("Model-Optimizer
 *   in practice: recovering Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD",
 *   section "QAD", --logit_kl_topk: the KD loss restricted to the teacher's
 *   top-k vocabulary entries, no dense [rows x V] FP32 tensor). Per row: the
 *   set is the k largest teacher logits (ties to the lower index); p_t, p_s
 *   are softmax of teacher and student logits over the set (temperature 1);
 *   loss = KL(p_t || p_s); gradient w.r.t. the student logits = p_s - p_t on
 *   the set. FP32 arithmetic with exp/log.
 * teacher, student  [rows][V] BF16, device, 16-byte aligned; V % 8 == 0.
 * k         1 <= k <= V.
 * loss      out FP32 [rows], device.
 * idx       nullable out int32 [rows][k]: the set, ascending index.
 * grad      nullable out FP32 [rows][k]: d loss / d student logit at idx
 *           (needs idx).
 * Non-finite teacher logits rank by their BF16 bit pattern: +-Inf as
 *   values, NaN with the sign bit clear above +Inf, with it set below -Inf.
 * Errors: NVFP4_ERR_INVALID_ARG for bad sizes or pointers.
 */
nvfp4_status nvfp4_topk_kl(const void* teacher, const void* student, int64_t rows, int64_t V, int k,
                           float* loss, int32_t* idx, float* grad, nvfp4_stream_t stream);

/*
 * nvfp4_dequantize -- y = BF16(g * s * q) for every element of an NVFP4
 *   tensor: the read side of an NVFP4 KV cache ("Developing Nemotron 3.5
 *   Lightning NVFP4 with QAD using NVIDIA Model Optimizer", Table 1
 *   "four_over_six + NVFP4 KV": K and V stored in NVFP4, QK^T in BF16).
 *   Products d = g*s then d*q in FP32, rounded once to BF16 (nearest even),
 *   so nvfp4_dequantize of nvfp4_quantize's output equals nvfp4_fake_quant.
 * codes   [M][K/2] bytes (element 2j in the low nibble), device, 16-aligned.
 * scales  tiled block scales (nvfp4_scale_bytes(M, K) bytes), device.
 * g       device FP32 scalar.
 * y       out [M][K] BF16, device, 16-byte aligned.
 * Errors: NVFP4_ERR_INVALID_ARG for K % 64 != 0 or bad pointers.
 */
nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t M,
                              int64_t K, void* y, nvfp4_stream_t stream);

/*
 * nvfp4_fake_quant_backward -- gradient of the QAD fake-quant w.r.t. x
 *   ("Developing Nemotron 3.5 Lightning NVFP4 with QAD using NVIDIA Model
 *   Optimizer", Figure 2: the gradient returns to the FP weights through
 *   the simulated quantization; the page does not name the estimator).
 *   Clipped straight-through estimator: grad_x = grad_y where
 *   |x * RN(1/(g*s))| <= 6 (FP32 product) for the element's block scale s,
 *   else 0. The scales are those nvfp4_fake_quant would use for the same
 *   arguments: recomputed from x (dynamic, static g), or frozen g*, s*.
 * x, grad_y   [M][K] BF16, device, 16-byte aligned.
 * mode        MAX or FOUR_OVER_SIX (used when the scales are recomputed).
 * g_frozen, scales_frozen, workspace: as for nvfp4_fake_quant.
 * grad_x      out [M][K] BF16 (distinct from x and grad_y).
 * Errors: NVFP4_ERR_INVALID_ARG for bad sizes, pointers, aliasing or mode.
 */
nvfp4_status nvfp4_fake_quant_backward(const void* x, const void* grad_y, int64_t M, int64_t K,
                                       nvfp4_mode mode, const float* g_frozen,
                                       const uint8_t* scales_frozen, void* grad_x, void* workspace,
                                       size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * Routed-expert (MoE) layer in NVFP4 W4A4 -- the layer the pages quantize
 * first ("2. PTQ": routed experts are 99.2% of the quantized tensors; the
 * Qwen3.8-Flash-Next page quantizes only the fused gate_up_proj/down_proj of
 * the routed experts, with top-k routing and dynamic activations).
 *
 *   out[t] = sum_j topk_w[t][j] * Down_e( SiLU(Gate_e(x_t)) * Up_e(x_t) ),
 *   e = topk_ids[t][j]
 *
 * with each expert's activations quantized dynamically (its own global scale
 * over the rows routed to it), h = SiLU(gate)*up rounded to BF16 and
 * quantized per expert, and the weighted combine done in FP32.
 * x         [T][H] BF16.
 * topk_ids  [T][topk] int32 in [0, E); topk_w [T][topk] FP32.
 * w13_q     [E][2I][H/2] codes; rows [0, I) are gate, [I, 2I) are up.
 * w13_s     E consecutive tiled scale buffers of nvfp4_scale_bytes(2I, H).
 * w13_g     [E] FP32 global scales.
 * w2_q      [E][H][I/2] codes; w2_s E buffers of nvfp4_scale_bytes(H, I);
 * w2_g      [E] FP32.
 * out       [T][H] FP32, overwritten.
 * workspace >= nvfp4_moe_workspace_bytes(T, H, I, E, topk) bytes, no
 *           initialisation needed; calls sharing it must be stream-ordered.
 * Requirements: H % 256 == 0, I % 128 == 0, 1 <= topk <= E <= 1024.
 */
size_t nvfp4_moe_workspace_bytes(int64_t T, int64_t H, int64_t I, int E, int topk);

nvfp4_status nvfp4_moe_grouped_gemm(const void* x, int64_t T, int64_t H,
                                    const int32_t* topk_ids, const float* topk_w,
                                    int topk, int E, int64_t I,
                                    const uint8_t* w13_q, const uint8_t* w13_s,
                                    const float* w13_g, const uint8_t* w2_q,
                                    const uint8_t* w2_s, const float* w2_g,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    nvfp4_stream_t stream);

/* Byte offsets of the intermediates the MoE call leaves in its workspace
 * (for inspection by tests and debuggers). All rows are in expert-major,
 * 128-padded order; R = padded row capacity. */
typedef struct {
  int64_t rows_capacity;    /* R */
  int64_t counts;           /* int32 [E]   pairs routed to each expert */
  int64_t offsets;          /* int32 [E+1] first padded row of each expert */
  int64_t row_pair;         /* int32 [R]   flat pair t*topk+j of a row, -1 = pad */
  int64_t xq_codes;         /* [R][H/2]    gathered, quantized x */
  int64_t xq_scales;        /* nvfp4_scale_bytes(R, H) */
  int64_t xq_g;             /* FP32 [E] */
  int64_t h;                /* BF16 [R][I]  SiLU(gate)*up */
  int64_t hq_codes;         /* [R][I/2] */
  int64_t hq_scales;        /* nvfp4_scale_bytes(R, I) */
  int64_t hq_g;             /* FP32 [E] */
  int64_t total_bytes;
} nvfp4_moe_layout;

nvfp4_status nvfp4_moe_workspace_layout(int64_t T, int64_t H, int64_t I, int E, int topk,
                                        nvfp4_moe_layout* layout /* host */);

/*
 * nvfp4_quantize_noalloc -- nvfp4_quantize without a workspace argument, for
 *   callers that cannot allocate device memory: an inference plugin whose
 *   enqueue step receives only its input and output pointers, or code that
 *   runs where the device allocator is unavailable or forbidden. (The pages
 *   have no counterpart; this is a deployment convenience.) Same arguments,
 *   outputs and device status as nvfp4_quantize, except that only modes MAX
 *   and FOUR_OVER_SIX are accepted (NVFP4_MODE_MSE returns
 *   NVFP4_ERR_INVALID_ARG).
 * Scratch: the dynamic global scale is reduced through a library-owned static
 *   device array of 4096 32-bit slots (16 KiB, held on every GPU that loads
 *   the library until exit), one slot per 2^18 input elements: M*K may be at
 *   most 2^30, larger inputs return NVFP4_ERR_TOO_LARGE before any launch.
 * The call allocates nothing. The first call on a device looks up the array's
 *   device address (make it before any stream capture on that device). All
 *   calls on a device share the array: calls whose kernels overlap on the GPU
 *   race and must be ordered (same stream). Nothing in the array needs to be
 *   cleared between calls.
 */
nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t M, int64_t K, nvfp4_mode mode,
                                    const float* g_in, uint8_t* codes, uint8_t* scales,
                                    float* g_out, uint8_t* fos_choice, nvfp4_stream_t stream);

/* Conversion primitives (diagnostics; the quantize kernels use the same
 * device code). e2m1: code of each FP32 value, one per byte, RNE, saturate
 * at +-6, sign from the value. e4m3: code of each non-negative FP32 value,
 * RNE, saturate at 448. n >= 0; in/out device arrays of n elements. */
nvfp4_status nvfp4_convert_e2m1(const float* in, int64_t n, uint8_t* out, nvfp4_stream_t stream);
nvfp4_status nvfp4_convert_e4m3(const float* in, int64_t n, uint8_t* out, nvfp4_stream_t stream);

/* Synchronize `stream`, then read (and with clear != 0 reset) the device
 * status word of the current device. *out is a host pointer. */
nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream, int clear, nvfp4_status* out);

/* Test hook for the bounded-wait path: run a kernel on `stream` whose wait
 * on a flag that nothing sets gives up after `timeout_ns` nanoseconds and
 * records NVFP4_ERR_TIMEOUT in the device status word. */
nvfp4_status nvfp4_selftest_timeout(uint64_t timeout_ns, nvfp4_stream_t stream);

/* Test hook for the GEMM's own bounded waits: nvfp4_gemm with the same
 * arguments, except that the TMA producer of the first CTA leaves the first
 * pipeline stage of its first tile unissued (nothing is copied, nothing is in
 * flight for it) and every wait gives up after `timeout_ns` (0 < timeout_ns
 * <= 10 s). The MMA warp's wait on that stage runs out, the CTA records
 * NVFP4_ERR_TIMEOUT in the device status word, lets its issued copies and
 * MMAs finish (bounded), frees its tensor memory and returns; C is then
 * unspecified and the context stays usable. Needs M > 0. The pages have no
 * counterpart: this exercises the library's failure detection. */
nvfp4_status nvfp4_selftest_gemm_timeout(const uint8_t* Aq, const uint8_t* As, const float* ga,
                                         const uint8_t* Bq, const uint8_t* Bs, const float* gb,
                                         int64_t M, int64_t N, int64_t K, void* C, uint64_t timeout_ns,
                                         nvfp4_stream_t stream);

/* FP4 tensor-core rate probe (diagnostic; the pages have no counterpart):
 * launches one CTA per SM that issues `iters` x 4 block-scaled MMAs
 * (kind::mxf4nvf4, M=128, N=256, K=64 -- the W4A4 GEMM's instruction) on
 * operands resident in shared memory, with no global-memory traffic, and
 * waits (bounded) for them. *flops_per_launch (host) receives the launch's
 * FLOP count, 2*128*256*256*iters*SMs; divided by the launch's duration it
 * is the measured dense FP4 peak. 1 <= iters <= 2^20. */
nvfp4_status nvfp4_probe_mma_peak(int iters, double* flops_per_launch, nvfp4_stream_t stream);

/* Number of kernels this library has launched in the process so far, summed
 * over all devices and threads (a host-side counter incremented at every
 * launch; it counts launches issued, not completed). Diagnostic only: the
 * method itself has no counterpart. Never fails. */
uint64_t nvfp4_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
