/*
 * hq.h -- C ABI of the B200 (sm_100a) dynamic-FP8 quantize and scaled FP8
 * GEMM library (libhq.so).
 *
 * The operations restate, in this library's own terms, the problem the
 * following pages describe:
 *   - hip-quant 0.6.0 README: "FP8 Formats" (E4M3 / E5M2 facts, OCP
 *     round-to-nearest-even), "Training-path numerical guards" (scales are
 *     pre-quant multipliers; the reciprocal is the dequant scale; non-finite
 *     amax samples are ignored), "Scale / amax tracking", "Memory Safety".
 *   - AstrAI csrc/kernels/fp8/ops.cu: quantize_bf16 (quantize with fused
 *     amax), commit "finalize fp8 scale rings inside quantize kernels" (the
 *     [hist | scale | counter] ring updated by the last block), mm_fp8 and
 *     linear_forward_fp8 (NT layout: A = XQ[M,K], B = WQ[N,K]).
 *   - hip-quant 0.6.0 README: "Stochastic E5M2 Backward Gradients" (round
 *     up or down with probability proportional to the distance, from a
 *     stateless hash of (seed, element index)), "Block-wise FP8 Scaling"
 *     (one FP32 dequant scale per block along the last dimension) and
 *     "Block-scaled Linear and Adafactor Kernel Helpers" (the linear on
 *     block-wise FP8 bytes and scales of both operands).
 *   - fuel-ir 0.22.4 src/quant_scale.rs: ScaleGranularity, scale_count,
 *     ScalePair.
 *   - ROCm/aiter PR 6437 "Technical Details": an a8w8 GEMM that writes a
 *     caller-owned, contiguous, 16-byte-aligned bf16 out[M,N], validation
 *     before launch, empty out is a no-op, out must not overlap an input.
 *   - megablocks-hip _dev/TODO-gg.md: the grouped (per-expert) GEMM; the
 *     output is overwritten, never accumulated into.
 *
 * Conventions common to every entry point:
 *   - Every buffer pointer is a DEVICE pointer on the current CUDA device,
 *     owned by the caller.  The library allocates nothing on any call.
 *   - Buffers are dense and row-major (C order); there are no stride
 *     arguments.
 *   - All work is enqueued on `stream` (0 = the legacy default stream).
 *     Calls are asynchronous: a status of HQ_OK means validation passed and
 *     the launches were enqueued.
 *   - Validation runs before any launch.  On any error the call returns a
 *     status, sets the message returned by hq_last_error(), and writes no
 *     output buffer.  Argument checks come first, then the device checks
 *     (pointer attributes), then the architecture check.
 *   - Device-side failures (a bounded wait that gave up, malformed device
 *     offsets) are recorded in a device error word that hq_check_device_error()
 *     reads back.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; no CUDA header is needed. */
typedef struct CUstream_st* hq_stream_t;

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARG = 1,      /* null pointer, bad size, bad enum, bad scale length */
  HQ_ERR_MISALIGNED = 2,       /* a pointer breaks its alignment rule */
  HQ_ERR_OVERLAP = 3,          /* an output overlaps an input or another output */
  HQ_ERR_WRONG_DEVICE = 4,     /* a pointer is not device memory of the current device */
  HQ_ERR_UNSUPPORTED_ARCH = 5, /* the current device is not compute capability 10.0 */
  HQ_ERR_CUDA = 6,             /* a CUDA runtime/driver call failed */
  HQ_ERR_TIMEOUT = 7,          /* a kernel's bounded wait gave up (device error word) */
  HQ_ERR_TOO_LARGE = 8         /* a size exceeds this library's index range */
} hq_status;

/* FP8 formats (hip-quant README "FP8 Formats"; AstrAI ops.cu `fmt` 0/1).
   E4M3: 1 sign, 4 exponent, 3 mantissa bits, bias 7, max +-448, NaN only.
   E5M2: 1 sign, 5 exponent, 2 mantissa bits, bias 15, max +-57344. */
typedef enum { HQ_E4M3 = 0, HQ_E5M2 = 1 } hq_fp8_format;

/* Scale granularity of a [rows, cols] tensor (fuel-ir quant_scale.rs
   ScaleGranularity): one scale for the tensor, one per row, one per column. */
typedef enum { HQ_PER_TENSOR = 0, HQ_PER_TOKEN = 1, HQ_PER_CHANNEL = 2 } hq_granularity;

/* Element type of a quantize input (hip-quant README: float32, float16 and
   bfloat16 inputs). */
typedef enum { HQ_F32 = 0, HQ_BF16 = 1, HQ_F16 = 2 } hq_dtype;

/* Number of f32 scales for a [rows, cols] tensor: 1, rows or cols
   (quant_scale.rs ScaleGranularity::scale_count).  Returns -1 for an
   invalid granularity or negative size. */
int64_t hq_scale_count(hq_granularity g, int64_t rows, int64_t cols);

/* "per_tensor" / "per_token" / "per_channel" (quant_scale.rs as_str), or
   NULL for an invalid value. */
const char* hq_granularity_name(hq_granularity g);

/* Writes "act_<g>_weight_<g>" (quant_scale.rs ScalePair Display) into buf
   (NUL-terminated, at most len bytes).  Returns the string length, or -1
   on an invalid granularity or a buffer that is too short. */
int hq_scale_pair_name(hq_granularity act, hq_granularity weight, char* buf, size_t len);

/* Bytes of device workspace hq_quantize_fp8 needs for this shape and mode
   (delayed != 0: the delayed per-tensor mode).  0 means no workspace.
   The caller zero-fills a workspace once before its first use; every call
   returns the whole workspace to zero, so one workspace can serve calls of
   any shape and mode that run one after another on the device.  Two calls
   that may run at the same time need two workspaces. */
size_t hq_quantize_workspace_bytes(hq_granularity g, int64_t rows, int64_t cols, int delayed);

/*
 * Dynamic (or delayed) FP8 quantization of a dense row-major x[rows, cols].
 *
 * Computes, per scale group of granularity g (tensor / row / column):
 *   amax = max |x| over the group's finite elements (NaN and +-Inf skipped)
 *   m    = fmax / amax in f32 (fmax = 448 or 57344); m = 1 when amax == 0
 *          or the quotient is not finite
 *   q    = saturating round-to-nearest-even FP8 code of f32(x) * m:
 *          |y| >= fmax and +-Inf -> +-max code, NaN -> 0x7F
 *   scales[i] = 1 / m (f32): the dequant scale the GEMM consumes
 *   amax_out[i] = amax (optional)
 * (hip-quant README "FP8 Formats" and "Training-path numerical guards";
 * AstrAI ops.cu quantize_bf16; quant_scale.rs scale_count.)
 *
 * Delayed mode (ring != NULL; only g == HQ_PER_TENSOR): ring is a device f32
 * buffer of ring_len + 2 words [hist[ring_len] | scale | counter] (AstrAI
 * ops.cu ring commit and pack_quantize_params).  The kernel quantizes with
 * m = ring[ring_len], writes scales[0] = 1/m, and its last block then
 * stores this call's amax in hist[ring_idx], takes win = max(hist) and, if
 * win is finite and > 0, forms next = f32(fmax / win) * 2^-margin; next
 * replaces ring[ring_len] only when it is finite and > 0 (a subnormal win
 * or a large |margin| can overflow it to +Inf or underflow it to 0; the old
 * scale then stays).  The counter word must be 0 on entry and is 0 on exit.
 * A fresh ring is hist = 0, scale = 1, counter = 0; the caller passes
 * ring_idx = step mod ring_len.
 *
 * Arguments:
 *   x            device, rows*cols elements of type xt
 *   q            device, rows*cols bytes (uint8 FP8 codes), row-major
 *   scales       device, hq_scale_count(g, rows, cols) f32
 *   amax_out     device or NULL, hq_scale_count(g, rows, cols) f32
 *   workspace    device, >= hq_quantize_workspace_bytes(...) bytes, 256-byte
 *                aligned, zeroed before first use (NULL if 0 bytes needed)
 * Errors: HQ_ERR_INVALID_ARG (null, negative size, bad enum, ring with
 *   g != PER_TENSOR, ring_len < 1, ring_idx outside [0, ring_len), workspace
 *   too small), HQ_ERR_MISALIGNED (x not aligned to its element size, ring
 *   or scales not 4-byte aligned, workspace not 256-byte aligned),
 *   HQ_ERR_OVERLAP (q / scales / amax_out / ring / workspace overlapping
 *   each other or x), HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH,
 *   HQ_ERR_TOO_LARGE (rows*cols >= 2^40), HQ_ERR_CUDA.
 * A shape with scale_count == 0 returns HQ_OK without a launch.  rows*cols
 * == 0 with scale_count > 0 writes scales = 1/m with amax 0 (and updates
 * the ring with amax 0).
 */
hq_status hq_quantize_fp8(const void* x, hq_dtype xt, int64_t rows, int64_t cols,
                          hq_fp8_format fmt, hq_granularity g,
                          uint8_t* q, float* scales, float* amax_out,
                          float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                          void* workspace, size_t workspace_bytes, hq_stream_t stream);

/*
 * Delayed (amax-history ring) per-tensor quantize of several tensors in one
 * launch: each tensor gets exactly what hq_quantize_fp8 in delayed mode
 * (ring != NULL, HQ_PER_TENSOR) would give it -- codes of f32(x) * m with
 * m = ring[ring_len], scale[0] = 1/m, amax_out[0] = the finite-only amax,
 * and the ring stepped (AstrAI ops.cu ring commit: every operand's ring is
 * finalized by the kernel that quantizes it; a layer quantizes its input
 * and weights this way every step).  One launch instead of `count` saves
 * the launch gaps of small tensors.
 *
 * tensors: host array of `count` descriptors (1 <= count <= 8); every
 *   tensor has element type xt and FP8 format fmt:
 *     x          device, n elements (rows*cols flattened), aligned to xt
 *     n          elements (>= 0; n == 0 steps the ring with amax 0)
 *     q          device, n bytes
 *     scale      device f32[1]
 *     amax_out   device f32[1] or NULL
 *     ring       device f32[ring_len + 2], counter word 0 on entry
 *     ring_len, ring_idx, ring_margin   as hq_quantize_fp8
 *     workspace  device, >= hq_quantize_workspace_bytes(HQ_PER_TENSOR, 1,
 *                n, 1) bytes, 256-byte aligned, zero on entry (left zero)
 * The tensors' buffers must not overlap each other (they run at once).
 * Errors: as hq_quantize_fp8 for each tensor (the message names it), plus
 *   HQ_ERR_INVALID_ARG for count outside [1, 8] or a NULL tensors array,
 *   and HQ_ERR_OVERLAP between tensors.  Nothing is launched on any error.
 */
typedef struct {
  const void* x;
  int64_t n;
  uint8_t* q;
  float* scale;
  float* amax_out;
  float* ring;
  int32_t ring_len, ring_idx, ring_margin;
  void* workspace;
  size_t workspace_bytes;
} hq_delayed_tensor;
hq_status hq_quantize_fp8_delayed_batch(const hq_delayed_tensor* tensors, int32_t count, hq_dtype xt,
                                        hq_fp8_format fmt, hq_stream_t stream);

/*
 * Block-scaled FP8 GEMM (hip-quant README "Block-scaled Linear and Adafactor
 * Kernel Helpers": the pre-quantized block-scaled linear consumes FP8 bytes
 * and FP32 per-block scales of both operands; "Block-wise FP8 Scaling": one
 * dequant scale per block of `block` elements along K, the last block the
 * short remainder):
 *   out[m,n] = bf16_rn( sum_b x_scales[m,b] * w_scales[n,b] * S_b[m,n] + bias[n] )
 * with S_b = sum over k in block b of dec(xq[m,k]) * dec(wq[n,k]), accumulated
 * in FP32 on the tensor cores, the block terms summed in FP32.
 *
 * Arguments: xq device [M, K] and wq device [N, K] FP8 codes of format fmt
 *   (K-major: the NT layout), 16-byte aligned; x_scales device f32
 *   [M, ceil(K / block)], w_scales device f32 [N, ceil(K / block)] (as
 *   hq_quantize_fp8_blockwise writes them); block a positive multiple of 32;
 *   K % 16 == 0; bias device bf16 [N] or NULL, 16-byte aligned; out
 *   caller-owned device bf16 [M, N], N % 8 == 0, 16-byte aligned, overwritten
 *   (K == 0 writes bf16(bias) or zeros).  M == 0 or N == 0 returns HQ_OK with
 *   no launch.
 * Errors: HQ_ERR_INVALID_ARG, HQ_ERR_MISALIGNED, HQ_ERR_OVERLAP,
 *   HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH, HQ_ERR_TOO_LARGE,
 *   HQ_ERR_CUDA; a stalled kernel reports HQ_ERR_TIMEOUT through
 *   hq_check_device_error.
 */
hq_status hq_gemm_blockscaled(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scales,
                              const float* w_scales, int64_t block, const void* bias, int64_t M, int64_t N, int64_t K,
                              void* out, hq_stream_t stream);

/*
 * Block-wise FP8 (hip-quant README "Block-wise FP8 Scaling"): the codes of x
 * [rows, cols] plus one f32 dequant scale per block of `block` consecutive
 * elements along the last dimension, scales [rows, ceil(cols / block)] (the
 * last block of a row may be shorter), real value ~= fp8 * block scale.  Per
 * block: amax over the finite |x|, m = fmax / amax (1 when amax is 0 or the
 * quotient is not finite), scale = 1/m, codes of f32(x) * m rounded to
 * nearest even, or, with stochastic != 0 (E5M2 only), rounded as
 * hq_quantize_e5m2_stochastic rounds (draws by row-major element index under
 * `seed`).  With block >= cols this is the per-token quantize.
 *
 * Arguments: x device [rows, cols] f32 / bf16 / f16 (xt), q device uint8
 *   [rows, cols], both 16-byte aligned; cols % 16 == 0; block % 16 == 0;
 *   scales device f32 [rows * ceil(cols / block)]; amax_out the same or NULL.
 *   rows == 0 or cols == 0 returns HQ_OK with no launch once the shape and
 *   enum checks pass (null buffers allowed then).
 * Errors: HQ_ERR_INVALID_ARG, HQ_ERR_MISALIGNED, HQ_ERR_OVERLAP,
 *   HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH, HQ_ERR_TOO_LARGE,
 *   HQ_ERR_CUDA.
 */
hq_status hq_quantize_fp8_blockwise(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                                    int64_t block, int stochastic, uint64_t seed, uint8_t* q, float* scales,
                                    float* amax_out, hq_stream_t stream);

/*
 * Block-wise dequantize: out[r, c] = f32(dec(q[r, c]) * scales[r, c / block])
 * (one f32 multiply), written as f32 (out_type HQ_F32) or rounded to bf16
 * (HQ_BF16).  Same layout rules, and the same empty-shape rule, as
 * hq_quantize_fp8_blockwise; out 16-byte aligned.
 */
hq_status hq_dequantize_fp8_blockwise(const uint8_t* q, hq_fp8_format fmt, int64_t rows, int64_t cols,
                                      int64_t block, const float* scales, hq_dtype out_type, void* out,
                                      hq_stream_t stream);

/*
 * Dynamic quantize to E5M2 with stochastic rounding, for gradients
 * (hip-quant README "Stochastic E5M2 Backward Gradients": between the two
 * adjacent E5M2 values, with probability proportional to the distance, from
 * a stateless per-element hash of (seed, element index)).
 *
 * amax, m = 57344 / amax and the exported dequant scales 1/m are exactly
 * those of hq_quantize_fp8(x, E5M2, g) for granularity g.  The cast: y =
 * f32(x) * m (one f32 multiply); with s the E5M2 spacing at |y| (2^(e-2)
 * for |y| in [2^e, 2^(e+1)), e >= -14, else 2^-16) and lo = floor(|y|/s) s,
 * |y| rounds up to lo + s iff u < floor((|y| - lo) / s * 2^32), where u is
 * the element's draw: the top 32 bits of SplitMix64's output number i + 1
 * from state `seed`, i = the element's row-major index.  NaN gives 0x7F,
 * |y| >= 57344 and +-Inf saturate, the sign is kept.  The same (x, g, seed)
 * always gives the same codes.
 *
 * Arguments: as hq_quantize_fp8 without the ring; x and q 16-byte aligned;
 * per-channel needs cols * sizeof(element) % 16 == 0; workspace >=
 * hq_quantize_workspace_bytes(g, rows, cols, 0) bytes, zero on entry and on
 * return (none for per-token).
 * Errors: HQ_ERR_INVALID_ARG, HQ_ERR_MISALIGNED, HQ_ERR_OVERLAP,
 *   HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH, HQ_ERR_TOO_LARGE,
 *   HQ_ERR_CUDA.
 */
hq_status hq_quantize_e5m2_stochastic(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_granularity g,
                                      uint64_t seed, uint8_t* q, float* scales, float* amax_out, void* workspace,
                                      size_t workspace_bytes, hq_stream_t stream);

/*
 * Per-tensor FP8 quantize that also writes the codes transposed, for the
 * backward GEMMs of AstrAI ops.cu linear_backward_fp8: dX = g @ w reads the
 * weight codes transposed and dW = g^T @ x reads the gradient and activation
 * codes transposed.  With the codes of x [rows, cols] row-major in q and
 * transposed in qt [cols, rows], both GEMMs run as the NT hq_gemm_a8w8.
 *
 * The codes are those of hq_quantize_fp8 with per-tensor granularity:
 *   - ring != NULL: the delayed mode (m = ring[ring_len], the ring stepped
 *     with this call's amax by the last CTA), exactly as hq_quantize_fp8;
 *   - multiplier != NULL: a caller's multiplier m = *multiplier (device f32),
 *     the ring-free static form the backward uses for w and x (the forward's
 *     scales; no ring is stepped); amax_out still receives the amax;
 *   - neither: the dynamic mode (m = fmax / amax of this call).
 * scales[0] receives 1/m in every mode.
 *
 * Arguments:
 *   x           device, [rows, cols] row-major, f32 / bf16 / f16 (xt),
 *               16-byte aligned; rows % 16 == 0 and cols % 16 == 0
 *   q           device uint8 [rows, cols], 16-byte aligned, or NULL
 *   qt          device uint8 [cols, rows], 16-byte aligned
 *   scales      device f32 [1]; amax_out device f32 [1] or NULL
 *   multiplier  device f32 [1] or NULL (not together with ring)
 *   ring, ring_len, ring_idx, ring_margin: as hq_quantize_fp8
 *   workspace   >= hq_quantize_workspace_bytes(PER_TENSOR, rows, cols, 1)
 *               bytes, zero on entry, zero again on return
 * Errors: HQ_ERR_INVALID_ARG (null, shape not a multiple of 16, multiplier
 *   with ring, bad ring index), HQ_ERR_MISALIGNED, HQ_ERR_OVERLAP,
 *   HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH, HQ_ERR_TOO_LARGE,
 *   HQ_ERR_CUDA.  An empty x (rows or cols 0) still writes scales (and steps
 *   the ring in the delayed mode).
 */
hq_status hq_quantize_fp8_transpose(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                                    uint8_t* q, uint8_t* qt, float* scales, float* amax_out, const float* multiplier,
                                    float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                                    void* workspace, size_t workspace_bytes, hq_stream_t stream);

/*
 * Bias gradient of a linear layer's backward pass (AstrAI
 * csrc/kernels/fp8/ops.cu linear_backward_fp8: the bias gradient is g
 * summed over dim 0 and cast back to g's dtype):
 *   out[c] = dtype( sum over r of g[r, c] ),  c in [0, cols)
 * The sum is accumulated in f32 in a fixed order (the rows of fixed bands
 * in order, then the bands in order), so repeated calls give identical
 * bits; it is rounded once to g's dtype (bf16 / f16 round-to-nearest-even,
 * or f32).  NaN and Inf propagate as in an f32 sum.  rows == 0 gives zeros.
 *
 * Arguments:
 *   g          device, [rows, cols] row-major, f32 / bf16 / f16 (gt),
 *              aligned to its element size (16-byte alignment of g and
 *              of every row takes the vector path)
 *   out        device, [cols] of gt, aligned to its element size
 *   workspace  device, >= hq_grad_bias_workspace_bytes(rows, cols) bytes,
 *              256-byte aligned, zero on entry and zero again on return (a
 *              counter per column strip; the rest holds per-band partial
 *              sums and need not be zero)
 * Errors: HQ_ERR_INVALID_ARG (null, negative shape, bad dtype, workspace
 *   too small), HQ_ERR_MISALIGNED, HQ_ERR_OVERLAP (out or workspace
 *   overlapping g or each other), HQ_ERR_WRONG_DEVICE,
 *   HQ_ERR_UNSUPPORTED_ARCH, HQ_ERR_TOO_LARGE (rows or cols >= 2^31, or
 *   rows * cols >= 2^40), HQ_ERR_CUDA.  cols == 0 is a no-op.
 */
size_t hq_grad_bias_workspace_bytes(int64_t rows, int64_t cols);
hq_status hq_grad_bias(const void* g, hq_dtype gt, int64_t rows, int64_t cols, void* out, void* workspace,
                       size_t workspace_bytes, hq_stream_t stream);

/*
 * Scaled FP8 GEMM, NT layout, into a caller-owned bf16 buffer:
 *   out[m, n] = bf16_rn( acc[m, n] * x_scale[m'] * w_scale[n'] ),
 *   acc[m, n] = sum_k dec(xq[m, k]) * dec(wq[n, k])   (FP32 accumulation)
 * with m' = m if x_scale_len == M else 0, n' = n if w_scale_len == N else 0
 * (ROCm/aiter PR 6437 "Technical Details": XQ[M,K], WQ[N,K], x_scale[M],
 * w_scale[N], bf16 out; AstrAI ops.cu mm_fp8: out = a @ b^T * (sa*sb),
 * FP32 accumulate).  Both operands use format fmt.
 *
 * Arguments:
 *   xq        device, M*K FP8 codes, row-major [M, K], 16-byte aligned
 *             (may be NULL when K == 0)
 *   wq        device, N*K FP8 codes, row-major [N, K], 16-byte aligned
 *             (may be NULL when K == 0)
 *   x_scale   device f32, x_scale_len in {1, M}
 *   w_scale   device f32, w_scale_len in {1, N}
 *   out       device bf16 (uint16 bits), dense row-major [M, N], 16-byte
 *             aligned start; it may be a view into a larger buffer, and
 *             nothing outside [out, out + M*N) is written.  Overwritten,
 *             never accumulated into.
 * Errors: HQ_ERR_INVALID_ARG (null, negative size, K % 16 != 0, N % 8 != 0,
 *   bad scale length, bad fmt), HQ_ERR_MISALIGNED (out, xq or wq not 16-byte
 *   aligned, scales not 4-byte aligned), HQ_ERR_OVERLAP (out overlapping
 *   any input), HQ_ERR_WRONG_DEVICE, HQ_ERR_UNSUPPORTED_ARCH,
 *   HQ_ERR_TOO_LARGE (M, N or K >= 2^31), HQ_ERR_CUDA.
 * M == 0 or N == 0 returns HQ_OK with no launch.  K == 0 writes
 * bf16(0 * scales).
 */
hq_status hq_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt,
                       const float* x_scale, int64_t x_scale_len,
                       const float* w_scale, int64_t w_scale_len,
                       int64_t M, int64_t N, int64_t K, void* out, hq_stream_t stream);

/*
 * The scaled FP8 GEMM with the fused epilogues of AstrAI ops.cu: mm_fp8
 * ("out_dtype" 1 = an FP8 output with its "out_scale", the output
 * quantization step) and linear_forward_fp8 (the bias added in the GEMM
 * epilogue).  Dense GEMMs only.
 *
 *   h[m, n] = bf16_rn( acc[m, n] * (x_scale[m'] * w_scale[n']) + bias[n] )
 *
 * (one f32 fused multiply-add before the rounding; no bias: as hq_gemm_a8w8).
 *
 * q_out == NULL: h is written to out, as hq_gemm_a8w8 does.
 * q_out != NULL: out must be NULL and h is not written.  Instead h is
 *   quantized per tensor with the delayed-scaling ring, exactly as
 *   hq_quantize_fp8(h, PER_TENSOR, q_fmt, ring, ring_idx, ring_margin) would
 *   quantize it: q = satfinite RNE code of f32(h) * m with m = ring[ring_len]
 *   on entry; *q_scale = 1/m; *q_amax (nullable) = max |h| over finite
 *   elements; the last CTA folds that amax into ring[ring_idx] and publishes
 *   the next multiplier in ring[ring_len] (the ring and workspace rules of
 *   hq_quantize_fp8's delayed mode).  The result is bit-identical to the two
 *   calls; the bf16 h never reaches memory.
 *
 * Arguments beyond hq_gemm_a8w8's:
 *   bias      device bf16 (uint16 bits) [N], 4-byte aligned, or NULL
 *   out       device bf16 [M, N] as in hq_gemm_a8w8, or NULL with q_out
 *   q_out     device uint8 [M, N] FP8 codes, 16-byte aligned; needs N % 16 == 0.
 *             NULL is accepted for an empty result (M == 0 or N == 0) with a
 *             ring and out == NULL: the FP8 mode is then implied
 *   q_fmt     format of the output codes
 *   q_scale   device f32 [1]: receives 1/m (the dequant scale of q_out)
 *   q_amax    device f32 [1] or NULL
 *   ring, ring_len, ring_idx, ring_margin: as hq_quantize_fp8 (required with q_out)
 *   workspace device, >= hq_quantize_workspace_bytes(PER_TENSOR, M, N, 1)
 *             bytes, all zero on entry; zero again on return (required with q_out)
 * Errors: those of hq_gemm_a8w8, plus HQ_ERR_INVALID_ARG (both or neither
 *   of out / q_out, q_out without ring / q_scale / workspace, bad ring
 *   index, N % 16 != 0 with q_out, bad q_fmt), HQ_ERR_MISALIGNED (q_out,
 *   bias, q_scale, ring, workspace) and HQ_ERR_OVERLAP among all buffers.
 * M == 0 or N == 0 with q_out runs the delayed quantize of the empty h
 * (amax 0, the ring updated, *q_scale = 1/m); with out it is a no-op.
 */
hq_status hq_gemm_a8w8_ex(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                          int64_t x_scale_len, const float* w_scale, int64_t w_scale_len, const void* bias,
                          int64_t M, int64_t N, int64_t K, void* out, uint8_t* q_out, hq_fp8_format q_fmt,
                          float* q_scale, float* q_amax, float* ring, int32_t ring_len, int32_t ring_idx,
                          int32_t ring_margin, void* workspace, size_t workspace_bytes, hq_stream_t stream);

/*
 * Scaled FP8 GEMM whose epilogue writes its result as block-wise FP8
 * (hip-quant README "Block-wise FP8 Scaling", with the output step of
 * AstrAI ops.cu mm_fp8 "out_dtype" 1): the bf16 result
 *
 *   h[m, n] = bf16_rn( acc[m, n] * (x_scale[m'] * w_scale[n']) + bias[n] )
 *
 * is quantized in blocks of 32 consecutive columns of a row, exactly as
 * hq_quantize_fp8_blockwise(h, HQ_BF16, M, N, q_fmt, 32, 0, 0, q_out,
 * q_scales, NULL) would quantize it: per block, amax over the finite |h|,
 * m = fmax / amax (1 when amax is 0 or the quotient is not finite),
 * q_scales[m, b] = 1/m, codes of f32(h) * m rounded to nearest even with
 * saturation (NaN -> 0x7F).  The result is bit-identical to the two calls;
 * the bf16 h never reaches memory.  The codes and scales are the operand
 * layout of hq_gemm_blockscaled with block 32 (K = this N), so the next
 * layer's GEMM can read them directly.  Dense GEMMs only; no ring, no
 * workspace.
 *
 * Arguments as hq_gemm_a8w8_ex, and:
 *   q_out     device uint8 [M, N] FP8 codes, 16-byte aligned, caller-owned
 *   q_fmt     format of the output codes
 *   block     the column block: 32 (the only supported value)
 *   q_scales  device f32 [M, N / 32] dequant scales, 4-byte aligned
 *   N % 32 == 0.  M == 0 or N == 0 returns HQ_OK with no launch (q_out and
 *   q_scales may then be NULL).
 * Errors: those of hq_gemm_a8w8, plus HQ_ERR_INVALID_ARG (block != 32,
 *   N % 32 != 0, null q_out / q_scales, bad q_fmt), HQ_ERR_MISALIGNED
 *   (q_out, q_scales, bias) and HQ_ERR_OVERLAP among all buffers.
 */
hq_status hq_gemm_a8w8_blockq(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                              int64_t x_scale_len, const float* w_scale, int64_t w_scale_len, const void* bias,
                              int64_t M, int64_t N, int64_t K, uint8_t* q_out, hq_fp8_format q_fmt, int64_t block,
                              float* q_scales, hq_stream_t stream);

/*
 * Grouped (per-expert) scaled FP8 GEMM (megablocks-hip TODO-gg.md gmm):
 * for each expert e and each row r in [offsets[e], offsets[e+1]):
 *   out[r, n] = bf16_rn( x_scale[r'] * w_scale[e*N + n'] *
 *                        sum_k dec(xq[r, k]) * dec(wq[e, n, k]) )
 *
 * Arguments:
 *   xq        device [M_total, K] FP8 codes, 16-byte aligned
 *   wq        device [E, N, K] FP8 codes, 16-byte aligned
 *   x_scale   device f32, x_scale_len in {1, M_total}
 *   w_scale   device f32, w_scale_len in {1, E*N}
 *   offsets   device int32 [E + 1]: offsets[0] = 0, non-decreasing,
 *             offsets[E] = M_total.  Read on the device only (no host sync).
 *   out       device bf16 [M_total, N], 16-byte aligned, overwritten.
 * Rows outside every expert's range are not written.  Malformed offsets
 * (decreasing, or outside [0, M_total]) never cause an access outside the
 * buffers: offsets are clamped and the device error word records
 * HQ_ERR_INVALID_ARG.
 * Errors as hq_gemm_a8w8, plus E outside [1, 1024] (HQ_ERR_INVALID_ARG).
 */
hq_status hq_grouped_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt,
                               const float* x_scale, int64_t x_scale_len,
                               const float* w_scale, int64_t w_scale_len,
                               const int32_t* offsets, int32_t E,
                               int64_t M_total, int64_t N, int64_t K,
                               void* out, hq_stream_t stream);

/*
 * Grouped bf16 GEMM with FP32 accumulation (megablocks-hip TODO-gg.md: the
 * per-expert bf16 product, overwritten into out):
 *   out[r, n] = bf16_rn( sum_k x[r, k] * w[e, n, k] ),  r in expert e's rows
 * x: device bf16 [M_total, K]; w: device bf16 [E, N, K]; K % 8 == 0.
 * Other arguments, rules and errors as hq_grouped_gemm_a8w8.
 */
hq_status hq_grouped_gemm_bf16(const void* x, const void* w,
                               const int32_t* offsets, int32_t E,
                               int64_t M_total, int64_t N, int64_t K,
                               void* out, hq_stream_t stream);

/*
 * hq_quantize_fp8 without a caller workspace, for callers that cannot
 * allocate device memory (no cudaMalloc in their context, or no allocator of
 * their own: they receive only input and output buffers).  No page describes
 * this entry point; it is this library's addition.
 *
 * Same arguments, computation, results and errors as hq_quantize_fp8, minus
 * `workspace` / `workspace_bytes`.  The per-tensor, per-channel and delayed
 * modes use one static device array of HQ_NOALLOC_SCRATCH_BYTES (256 KiB)
 * instead, which every GPU that loads the library holds until the process
 * exits.  Per-tensor and delayed calls always fit; a per-channel call fits
 * up to 32,764 columns; a larger one returns HQ_ERR_TOO_LARGE before any
 * launch.  The call itself allocates nothing.
 *
 * The argument checks run first, in hq_quantize_fp8's order; the size limit
 * and the array's set-up come after them.  The first call on a device that
 * needs the array looks up its device address and clears it (a synchronous
 * memset on that device); make that first call before any stream capture.
 * Every call leaves the array zero again.  After a call that returned
 * HQ_ERR_CUDA, or after hq_check_device_error() reported HQ_ERR_TIMEOUT, the
 * next call clears the array again (synchronously) before using it.  All
 * calls share the one array: two calls that may overlap on the GPU
 * (different streams, or different host threads) race on it and must be
 * serialised by the caller.
 */
#define HQ_NOALLOC_SCRATCH_BYTES (256u * 1024u)
hq_status hq_quantize_fp8_noalloc(const void* x, hq_dtype xt, int64_t rows, int64_t cols,
                                  hq_fp8_format fmt, hq_granularity g,
                                  uint8_t* q, float* scales, float* amax_out,
                                  float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                                  hq_stream_t stream);

/*
 * Test hook for the failure path of the library's bounded waits: launches
 * one warp whose lanes wait on a shared-memory barrier nothing completes,
 * lane l for limit_ns * (1 + l/32) nanoseconds (limit_ns in 1 us .. 2 s).
 * The first lane to give up records a timeout in the device error word and
 * ends the other lanes' waits; the warp agrees on giving up before a
 * warp-wide step (as the GEMM warps do before their warp-wide tensor-memory
 * loads) and the kernel returns normally (no trap, no fault).  The next
 * hq_check_device_error() returns HQ_ERR_TIMEOUT and clears the word.  Every
 * wait in the library's kernels takes this path on a stalled barrier.
 * Errors: HQ_ERR_INVALID_ARG (limit outside the range), HQ_ERR_UNSUPPORTED_ARCH,
 *   HQ_ERR_CUDA.
 */
hq_status hq_debug_bounded_wait(uint64_t limit_ns, hq_stream_t stream);

/* Synchronizes the current device, then reads and clears the device error
   word: HQ_OK, HQ_ERR_TIMEOUT (a bounded wait in a kernel gave up; that
   launch's outputs are undefined), HQ_ERR_INVALID_ARG (malformed grouped
   offsets), or HQ_ERR_CUDA. */
hq_status hq_check_device_error(void);

/* Message for the last error on this host thread ("" if none). */
const char* hq_last_error(void);

/* Library version string. */
const char* hq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
