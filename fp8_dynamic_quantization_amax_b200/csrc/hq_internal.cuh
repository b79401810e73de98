// hq_internal.cuh -- declarations shared by the translation units of
// libhq.so (api.cu, quantize.cu, gemm.cu, gemm_bs.cu, noalloc.cu, probe.cu).
// Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>

#include "../../include/hq.h"
#include <cstddef>
#include <cstdint>
#include <string>

namespace hq {

// Format facts (hip-quant README "FP8 Formats"): largest finite magnitude.
constexpr float kFmaxE4M3 = 448.0f;
constexpr float kFmaxE5M2 = 57344.0f;

struct QuantizeArgs {
  const void* x;
  int xt;            // 0 f32, 1 bf16, 2 f16
  int64_t rows, cols;
  int fmt;           // 0 E4M3, 1 E5M2
  int gran;          // 0 tensor, 1 token, 2 channel
  uint8_t* q;
  float* scales;
  float* amax_out;   // nullable
  float* ring;       // nullable (delayed mode)
  int ring_len, ring_idx, ring_margin;
  void* ws;          // workspace (may be null when none is needed)
  cudaStream_t stream;
  uint8_t* qt = nullptr;        // transposed codes [cols, rows] (launch_quantize_transpose)
  const float* mult = nullptr;  // a caller's multiplier (static per-tensor form)
  uint64_t seed = 0;            // stochastic rounding (launch_quantize_sr)
};

size_t quantize_workspace_bytes(int gran, int64_t rows, int64_t cols, int delayed);
cudaError_t launch_quantize(const QuantizeArgs& a);

// One tensor of a batched delayed (ring) per-tensor quantize.
struct DelayedTensorArgs {
  const void* x;
  int64_t n;          // elements
  uint8_t* q;
  float* scale;       // f32[1]: 1/m
  float* amax_out;    // nullable
  float* ring;        // [ring_len | scale | counter]
  int ring_len, ring_idx, ring_margin;
  void* ws;           // the delayed workspace (one amax word), zero between calls
};
// Up to 8 tensors of one dtype (xt) and format in one launch.
cudaError_t launch_quantize_delayed_batch(int xt, int fmt, const DelayedTensorArgs* t, int count,
                                          cudaStream_t stream);
// Per-tensor quantize writing the codes row-major (a.q, nullable) and
// transposed (a.qt); rows % 16 == 0, cols % 16 == 0, x 16-byte aligned.
cudaError_t launch_quantize_transpose(const QuantizeArgs& a);
// Dynamic E5M2 quantize with stochastic rounding (a.seed); x 16-byte aligned,
// cols a multiple of the 16-byte vector for the per-channel form.
cudaError_t launch_quantize_sr(const QuantizeArgs& a);
// Block-wise quantize (scales [rows, ceil(cols / block)]) and dequantize;
// block % 16 == 0, cols % 16 == 0, 16-byte aligned buffers.
cudaError_t launch_quantize_blockwise(const QuantizeArgs& a, int64_t block, bool stochastic);
// Bias gradient: column sums of g [rows, cols] (xt 0 f32, 1 bf16, 2 f16) in
// f32, written in g's dtype; ws as grad_bias_workspace_bytes, its counters
// zero between calls.
size_t grad_bias_workspace_bytes(int64_t rows, int64_t cols);
cudaError_t launch_grad_bias(const void* g, int xt, int64_t rows, int64_t cols, void* out, void* ws,
                             cudaStream_t stream);
cudaError_t launch_dequantize_blockwise(const uint8_t* q, int fmt, int64_t rows, int64_t cols, int64_t block,
                                        const float* scales, bool bf16_out, void* out, cudaStream_t stream);

struct GemmArgs {
  int kind;                 // 0: fp8 a8w8 (kind::f8f6f4), 1: bf16 (kind::f16)
  int fmt;                  // fp8 format of both operands (kind 0)
  const void* a;            // [M_total, K]
  const void* b;            // [E, N, K] (E = 1 for the dense GEMM)
  const float* x_scale;     // nullable for kind 1
  int64_t x_scale_len;
  const float* w_scale;     // nullable for kind 1
  int64_t w_scale_len;
  const int32_t* offsets;   // null: dense GEMM (one group of M rows)
  int E;
  int64_t M, N, K;
  void* out;                // bf16 [M, N]; null when q_out is set
  cudaStream_t stream;
  // fused epilogues (dense only)
  const void* bias = nullptr;   // bf16 [N]
  uint8_t* q_out = nullptr;     // FP8 codes [M, N]: the delayed per-tensor quantize of the bf16 result
  int q_fmt = 0;
  float* q_scale = nullptr;
  float* q_amax = nullptr;
  float* ring = nullptr;
  int ring_len = 0, ring_idx = 0, ring_margin = 0;
  uint32_t* q_ws = nullptr;     // amax accumulator word (zero between calls)
  float* q_bscales = nullptr;   // set: q_out holds block-wise codes (32-column blocks, no ring), scales [M, N/32]
};

// Returns cudaSuccess or the failing call's error; *msg gets a description.
cudaError_t launch_gemm(const GemmArgs& a, std::string* msg);

// Block-scaled FP8 GEMM: out = bf16(sum_b xs[m,b] ws[n,b] S_b (+ bias[n])),
// scales [M | N, ceil(K / block)], block % 32 == 0, K % 16 == 0, N % 8 == 0,
// A, B, out and bias 16-byte aligned.
struct BlockScaledGemmArgs {
  int fmt;
  const void* a;            // FP8 [M, K]
  const void* b;            // FP8 [N, K]
  const float* x_scales;    // [M, nb]
  const float* w_scales;    // [N, nb]
  int64_t block;
  const void* bias;         // bf16 [N] or null
  int64_t M, N, K;
  void* out;                // bf16 [M, N]
  cudaStream_t stream;
};
cudaError_t launch_gemm_blockscaled(const BlockScaledGemmArgs& a, std::string* msg);
// The same GEMM with the block scales applied while converting the codes to
// bf16 MMA operands (gemm.cu): no per-block round trip through TMEM.
cudaError_t launch_gemm_blockscaled_bf16(const BlockScaledGemmArgs& a, std::string* msg);

// Device error word (set by bounded waits and by offset validation).
enum : unsigned { kDevErrTimeout = 1u, kDevErrBadOffsets = 2u };
cudaError_t read_and_clear_device_error(unsigned* word);
// Device address of that word on the current device (nullptr if unavailable).
unsigned* device_error_word();

int device_sm_count(int dev);

// One bounded wait that nothing completes (probe.cu): sets kDevErrTimeout.
cudaError_t launch_bounded_wait_probe(unsigned long long limit_ns, cudaStream_t stream);

// Records a printf-style message for hq_last_error() and returns s.
hq_status set_error(hq_status s, const char* fmt, ...);

// The argument checks of hq_quantize_fp8 that do not involve the workspace
// (api.cu); *empty is set for a call with no scale group.
hq_status quantize_check_args(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                              hq_granularity g, const uint8_t* q, const float* scales, const float* amax_out,
                              const float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                              bool* empty);

// Marks the no-allocation entry point's static scratch for clearing on its
// next call on every device (noalloc.cu).
void noalloc_scratch_invalidate();

}  // namespace hq
