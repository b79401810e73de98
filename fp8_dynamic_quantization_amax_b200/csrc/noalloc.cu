// noalloc.cu -- hq_quantize_fp8_noalloc: the quantize entry point for callers
// that cannot allocate device memory.
//
// The per-tensor, per-channel and delayed modes of hq_quantize_fp8 need a
// small device workspace for their cross-CTA amax accumulators, counter and
// published multipliers.  Some callers cannot provide one, because they may
// not call cudaMalloc: for example code that runs inside a host framework's
// enqueue callback where allocation after set-up is forbidden, or a library
// that owns no allocator and receives only its input and output buffers.
// For them the workspace lives here, in one file-scope device array that
// every GPU which loads this library holds until the process exits.
#include "../../include/hq.h"
#include "hq_internal.cuh"

#include <mutex>

namespace {

// Fixed size of the shared scratch: per-tensor and delayed calls need 256
// bytes; a per-channel call needs 16 + 8 bytes per column (rounded up to 256),
// so up to 32,764 columns fit.
constexpr size_t kScratchBytes = HQ_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device.  The first call
// on a device looks the address up (the array's name is only a host-side
// handle) and clears the array; every quantize call leaves it zero again.
// After a failed call the address is forgotten, so the next call clears the
// array before using it.
hq_status scratch_for_current_device(int* dev_out, void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return hq::set_error(HQ_ERR_CUDA, "cudaGetDevice failed");
  }
  if (dev < 0 || dev >= 64) return hq::set_error(HQ_ERR_INVALID_ARG, "device index out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return hq::set_error(HQ_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
    }
    e = cudaMemset(p, 0, kScratchBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
      cudaGetLastError();  // leave no stale error for a later, unrelated launch check
      return hq::set_error(HQ_ERR_CUDA, "clearing the static scratch failed: %s", cudaGetErrorString(e));
    }
    g_scratch_ptr[dev] = p;
  }
  *dev_out = dev;
  *out = g_scratch_ptr[dev];
  return HQ_OK;
}

}  // namespace

namespace hq {
void noalloc_scratch_invalidate() {
  std::lock_guard<std::mutex> lk(g_mu);
  for (void*& p : g_scratch_ptr) p = nullptr;
}
}  // namespace hq

extern "C" hq_status hq_quantize_fp8_noalloc(const void* x, hq_dtype xt, int64_t rows, int64_t cols,
                                             hq_fp8_format fmt, hq_granularity g, uint8_t* q, float* scales,
                                             float* amax_out, float* ring, int32_t ring_len, int32_t ring_idx,
                                             int32_t ring_margin, hq_stream_t stream) {
  // the same argument checks, in the same order, as hq_quantize_fp8
  bool empty = false;
  hq_status s = hq::quantize_check_args(x, xt, rows, cols, fmt, g, q, scales, amax_out, ring, ring_len, ring_idx,
                                        ring_margin, &empty);
  if (s != HQ_OK || empty) return s;
  const size_t need = hq_quantize_workspace_bytes(g, rows, cols, ring != nullptr);
  if (need > kScratchBytes)
    return hq::set_error(HQ_ERR_TOO_LARGE,
                         "this shape needs %zu bytes of scratch; the static scratch holds %zu "
                         "(per-channel: at most 32764 columns)",
                         need, kScratchBytes);
  void* ws = nullptr;
  int dev = -1;
  if (need > 0) {
    s = scratch_for_current_device(&dev, &ws);
    if (s != HQ_OK) return s;
  }
  s = hq_quantize_fp8(x, xt, rows, cols, fmt, g, q, scales, amax_out, ring, ring_len, ring_idx, ring_margin, ws,
                      need > 0 ? kScratchBytes : 0, stream);
  if (s == HQ_ERR_CUDA && need > 0) {
    // a launch that failed part-way can leave counters or published
    // multipliers in the array: clear it again on the next call
    std::lock_guard<std::mutex> lk(g_mu);
    g_scratch_ptr[dev] = nullptr;
  }
  return s;
}
