// api.cu -- the extern "C" boundary of libhq.so: argument validation,
// device and architecture checks, dispatch to the kernels, error strings.
//
// Validation order follows ROCm/aiter PR 6437 "Technical Details": every
// argument check runs before any launch and before the architecture check,
// so invalid arguments always report INVALID_ARG / MISALIGNED / OVERLAP
// even on an unsupported device, and no output is touched on error.  An
// empty output returns after validation without a launch.  Operands must be
// on the current device (the PR's non-current-device rule).
#include "../../include/hq.h"
#include "hq_internal.cuh"

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

namespace {

thread_local std::string g_last_error;

hq_status fail(hq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

hq_status ok() {
  g_last_error.clear();
  return HQ_OK;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
  const void* p;
  size_t bytes;
  const char* name;
};

bool overlaps(const Range& a, const Range& b) {
  if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
  return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// Every output range against every other range listed after it.
hq_status check_overlaps(const Range* outs, int n_out, const Range* ins, int n_in) {
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j)
      if (overlaps(outs[i], ins[j]))
        return fail(HQ_ERR_OVERLAP, "%s overlaps input %s", outs[i].name, ins[j].name);
    for (int j = i + 1; j < n_out; ++j)
      if (overlaps(outs[i], outs[j]))
        return fail(HQ_ERR_OVERLAP, "%s overlaps %s", outs[i].name, outs[j].name);
  }
  return HQ_OK;
}

// Device pointers of the current device only (managed memory included).
hq_status check_device_ptrs(const Range* rs, int n) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(HQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  for (int i = 0; i < n; ++i) {
    if (!rs[i].p) continue;
    cudaPointerAttributes attr;
    e = cudaPointerGetAttributes(&attr, rs[i].p);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(HQ_ERR_WRONG_DEVICE, "%s: cudaPointerGetAttributes: %s", rs[i].name, cudaGetErrorString(e));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
      return fail(HQ_ERR_WRONG_DEVICE, "%s is not device memory", rs[i].name);
    if (attr.device != dev)
      return fail(HQ_ERR_WRONG_DEVICE, "%s lives on device %d, current device is %d", rs[i].name, attr.device, dev);
  }
  return HQ_OK;
}

// Compute capability 10.0 (B200, sm_100a) only; cached per device.
hq_status check_arch() {
  static std::mutex mu;
  static int cache[64];
  static bool init = false;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(HQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(mu);
  if (!init) {
    for (int& c : cache) c = -1;
    init = true;
  }
  if (dev < 0 || dev >= 64) return fail(HQ_ERR_UNSUPPORTED_ARCH, "device index %d out of range", dev);
  if (cache[dev] < 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return fail(HQ_ERR_CUDA, "cudaDeviceGetAttribute failed");
    cache[dev] = major * 10 + minor;
  }
  if (cache[dev] != 100)
    return fail(HQ_ERR_UNSUPPORTED_ARCH, "compute capability %d.%d; this library is built for sm_100a (10.0)",
                cache[dev] / 10, cache[dev] % 10);
  return HQ_OK;
}

hq_status launched(cudaError_t e, const char* what, const std::string& extra = std::string()) {
  if (e != cudaSuccess)
    return fail(HQ_ERR_CUDA, "%s: %s%s%s", what, cudaGetErrorString(e), extra.empty() ? "" : " -- ", extra.c_str());
  return ok();
}

constexpr int64_t k2p31 = int64_t(1) << 31;
constexpr int64_t k2p40 = int64_t(1) << 40;

}  // namespace

namespace hq {
hq_status set_error(hq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

int device_sm_count(int dev) {
  static std::mutex mu;
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}
}  // namespace hq

extern "C" {

int64_t hq_scale_count(hq_granularity g, int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return -1;
  switch (g) {
    case HQ_PER_TENSOR: return 1;
    case HQ_PER_TOKEN: return rows;
    case HQ_PER_CHANNEL: return cols;
    default: return -1;
  }
}

const char* hq_granularity_name(hq_granularity g) {
  switch (g) {
    case HQ_PER_TENSOR: return "per_tensor";
    case HQ_PER_TOKEN: return "per_token";
    case HQ_PER_CHANNEL: return "per_channel";
    default: return nullptr;
  }
}

int hq_scale_pair_name(hq_granularity act, hq_granularity weight, char* buf, size_t len) {
  const char* a = hq_granularity_name(act);
  const char* w = hq_granularity_name(weight);
  if (!a || !w || !buf) return -1;
  const int n = snprintf(buf, len, "act_%s_weight_%s", a, w);
  if (n < 0 || static_cast<size_t>(n) >= len) return -1;
  return n;
}

size_t hq_quantize_workspace_bytes(hq_granularity g, int64_t rows, int64_t cols, int delayed) {
  if (hq_scale_count(g, rows, cols) < 0) return 0;
  return hq::quantize_workspace_bytes(static_cast<int>(g), rows, cols, delayed);
}

}  // extern "C"

namespace hq {
// The argument checks of hq_quantize_fp8 that do not involve the workspace,
// in the order that entry point applies them.  *empty is set when the call
// has no scale group (scale_count == 0): such a call returns HQ_OK without
// a launch.
hq_status quantize_check_args(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                              hq_granularity g, const uint8_t* q, const float* scales, const float* amax_out,
                              const float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                              bool* empty) {
  *empty = false;
  if (xt != HQ_F32 && xt != HQ_BF16 && xt != HQ_F16) return fail(HQ_ERR_INVALID_ARG, "invalid dtype %d", (int)xt);
  if (fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", (int)fmt);
  if (g != HQ_PER_TENSOR && g != HQ_PER_TOKEN && g != HQ_PER_CHANNEL)
    return fail(HQ_ERR_INVALID_ARG, "invalid granularity %d", (int)g);
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  if (ring) {
    if (g != HQ_PER_TENSOR) return fail(HQ_ERR_INVALID_ARG, "a delayed-scaling ring needs per-tensor granularity");
    if (ring_len < 1 || ring_len > (1 << 20)) return fail(HQ_ERR_INVALID_ARG, "ring_len %d outside [1, 2^20]", ring_len);
    if (ring_idx < 0 || ring_idx >= ring_len)
      return fail(HQ_ERR_INVALID_ARG, "ring_idx %d outside [0, %d)", ring_idx, ring_len);
    if (ring_margin < -126 || ring_margin > 126) return fail(HQ_ERR_INVALID_ARG, "ring_margin %d outside [-126, 126]", ring_margin);
  }
  const int64_t ns = hq_scale_count(g, rows, cols);
  const int64_t n = rows * cols;
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  if (ns == 0) {
    *empty = true;
    return ok();
  }
  if (n > 0 && (!x || !q)) return fail(HQ_ERR_INVALID_ARG, "x and q must not be null");
  if (!scales) return fail(HQ_ERR_INVALID_ARG, "scales must not be null");
  if (!is_aligned(x, esize)) return fail(HQ_ERR_MISALIGNED, "x is not aligned to its element size");
  if (!is_aligned(scales, 4) || !is_aligned(amax_out, 4) || !is_aligned(ring, 4))
    return fail(HQ_ERR_MISALIGNED, "scales, amax_out and ring must be 4-byte aligned");
  const Range outs[] = {{q, static_cast<size_t>(n), "q"},
                        {scales, static_cast<size_t>(ns) * 4, "scales"},
                        {amax_out, amax_out ? static_cast<size_t>(ns) * 4 : 0, "amax_out"},
                        {ring, ring ? static_cast<size_t>(ring_len + 2) * 4 : 0, "ring"}};
  const Range ins[] = {{x, static_cast<size_t>(n) * esize, "x"}};
  return check_overlaps(outs, 4, ins, 1);
}
}  // namespace hq

extern "C" {

hq_status hq_quantize_fp8(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                          hq_granularity g, uint8_t* q, float* scales, float* amax_out, float* ring,
                          int32_t ring_len, int32_t ring_idx, int32_t ring_margin, void* workspace,
                          size_t workspace_bytes, hq_stream_t stream) {
  // ---- arguments
  bool empty = false;
  hq_status s = hq::quantize_check_args(x, xt, rows, cols, fmt, g, q, scales, amax_out, ring, ring_len, ring_idx,
                                        ring_margin, &empty);
  if (s != HQ_OK || empty) return s;
  const int64_t ns = hq_scale_count(g, rows, cols);
  const int64_t n = rows * cols;
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  const size_t need = hq::quantize_workspace_bytes(static_cast<int>(g), rows, cols, ring != nullptr);
  if (need > 0 && !workspace) return fail(HQ_ERR_INVALID_ARG, "this mode needs a workspace of %zu bytes", need);
  if (need > 0 && workspace_bytes < need)
    return fail(HQ_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes, need);
  if (need > 0 && !is_aligned(workspace, 256)) return fail(HQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  const Range outs[] = {{q, static_cast<size_t>(n), "q"},
                        {scales, static_cast<size_t>(ns) * 4, "scales"},
                        {amax_out, amax_out ? static_cast<size_t>(ns) * 4 : 0, "amax_out"},
                        {ring, ring ? static_cast<size_t>(ring_len + 2) * 4 : 0, "ring"},
                        {workspace, need, "workspace"}};
  const Range ins[] = {{x, static_cast<size_t>(n) * esize, "x"}};
  s = check_overlaps(outs, 5, ins, 1);
  if (s != HQ_OK) return s;
  // ---- device
  const Range devs[] = {{n > 0 ? x : nullptr, 0, "x"}, {n > 0 ? q : nullptr, 0, "q"}, {scales, 0, "scales"},
                        {amax_out, 0, "amax_out"}, {ring, 0, "ring"}, {need > 0 ? workspace : nullptr, 0, "workspace"}};
  s = check_device_ptrs(devs, 6);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  // ---- launch
  hq::QuantizeArgs a;
  a.x = x; a.xt = xt; a.rows = rows; a.cols = cols; a.fmt = fmt; a.gran = g;
  a.q = q; a.scales = scales; a.amax_out = amax_out;
  a.ring = ring; a.ring_len = ring_len; a.ring_idx = ring_idx; a.ring_margin = ring_margin;
  a.ws = workspace;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return launched(hq::launch_quantize(a), "quantize launch");
}

hq_status hq_quantize_fp8_delayed_batch(const hq_delayed_tensor* tensors, int32_t count, hq_dtype xt,
                                        hq_fp8_format fmt, hq_stream_t stream) {
  // ---- arguments
  if (!tensors) return fail(HQ_ERR_INVALID_ARG, "tensors must not be null");
  if (count < 1 || count > 8) return fail(HQ_ERR_INVALID_ARG, "count = %d outside [1, 8]", count);
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  Range all[8][6];  // per tensor: x, q, scale, amax_out, ring, workspace
  for (int i = 0; i < count; ++i) {
    const hq_delayed_tensor& t = tensors[i];
    bool empty = false;
    hq_status s = hq::quantize_check_args(t.x, xt, 1, t.n, fmt, HQ_PER_TENSOR, t.q, t.scale, t.amax_out, t.ring,
                                          t.ring_len, t.ring_idx, t.ring_margin, &empty);
    if (s != HQ_OK) return fail(s, "tensor %d: %s", i, hq_last_error());
    if (!t.ring) return fail(HQ_ERR_INVALID_ARG, "tensor %d: a delayed quantize needs a ring", i);
    const size_t need = hq::quantize_workspace_bytes(HQ_PER_TENSOR, 1, t.n, 1);
    if (need > 0 && !t.workspace) return fail(HQ_ERR_INVALID_ARG, "tensor %d: a workspace of %zu bytes is needed", i, need);
    if (need > 0 && t.workspace_bytes < need)
      return fail(HQ_ERR_INVALID_ARG, "tensor %d: workspace of %zu bytes is smaller than the %zu needed", i,
                  t.workspace_bytes, need);
    if (need > 0 && !is_aligned(t.workspace, 256))
      return fail(HQ_ERR_MISALIGNED, "tensor %d: workspace must be 256-byte aligned", i);
    all[i][0] = {t.x, static_cast<size_t>(t.n) * esize, "x"};
    all[i][1] = {t.q, static_cast<size_t>(t.n), "q"};
    all[i][2] = {t.scale, 4, "scale"};
    all[i][3] = {t.amax_out, t.amax_out ? 4u : 0u, "amax_out"};
    all[i][4] = {t.ring, static_cast<size_t>(t.ring_len + 2) * 4, "ring"};
    all[i][5] = {t.workspace, need, "workspace"};
    // the workspace against this tensor's other buffers
    for (int k = 0; k < 5; ++k)
      if (overlaps(all[i][5], all[i][k]))
        return fail(HQ_ERR_OVERLAP, "tensor %d: workspace overlaps %s", i, all[i][k].name);
  }
  // tensors run at once: no output of one may overlap any buffer of another
  for (int i = 0; i < count; ++i)
    for (int j = 0; j < count; ++j) {
      if (i == j) continue;
      for (int a = 1; a < 6; ++a)
        for (int b = 0; b < 6; ++b)
          if (overlaps(all[i][a], all[j][b]))
            return fail(HQ_ERR_OVERLAP, "tensor %d's %s overlaps tensor %d's %s", i, all[i][a].name, j,
                        all[j][b].name);
    }
  // ---- device
  for (int i = 0; i < count; ++i) {
    const hq_delayed_tensor& t = tensors[i];
    const Range devs[] = {{t.n > 0 ? t.x : nullptr, 0, "x"}, {t.n > 0 ? t.q : nullptr, 0, "q"}, {t.scale, 0, "scale"},
                          {t.amax_out, 0, "amax_out"}, {t.ring, 0, "ring"}, {t.workspace, 0, "workspace"}};
    hq_status s = check_device_ptrs(devs, 6);
    if (s != HQ_OK) return fail(s, "tensor %d: %s", i, hq_last_error());
  }
  hq_status s = check_arch();
  if (s != HQ_OK) return s;
  // ---- launch
  hq::DelayedTensorArgs a[8];
  for (int i = 0; i < count; ++i) {
    const hq_delayed_tensor& t = tensors[i];
    a[i].x = t.x; a[i].n = t.n; a[i].q = t.q; a[i].scale = t.scale; a[i].amax_out = t.amax_out;
    a[i].ring = t.ring; a[i].ring_len = t.ring_len; a[i].ring_idx = t.ring_idx; a[i].ring_margin = t.ring_margin;
    a[i].ws = t.workspace;
  }
  return launched(hq::launch_quantize_delayed_batch(static_cast<int>(xt), static_cast<int>(fmt), a, count,
                                                    reinterpret_cast<cudaStream_t>(stream)),
                  "batched delayed quantize launch");
}

hq_status hq_quantize_fp8_blockwise(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                                    int64_t block, int stochastic, uint64_t seed, uint8_t* q, float* scales,
                                    float* amax_out, hq_stream_t stream) {
  if (xt != HQ_F32 && xt != HQ_BF16 && xt != HQ_F16) return fail(HQ_ERR_INVALID_ARG, "invalid dtype %d", (int)xt);
  if (fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", (int)fmt);
  if (stochastic && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "stochastic rounding is for E5M2");
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  if (block < 16 || block % 16 != 0 || block >= k2p31)
    return fail(HQ_ERR_INVALID_ARG, "block = %lld must be a positive multiple of 16", (long long)block);
  if (cols % 16 != 0) return fail(HQ_ERR_INVALID_ARG, "cols must be a multiple of 16");
  const int64_t n = rows * cols;
  const int64_t ns = rows * ((cols + block - 1) / block);
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  if (n == 0) return ok();
  if (!x || !q || !scales) return fail(HQ_ERR_INVALID_ARG, "x, q and scales must not be null");
  if (!is_aligned(x, 16) || !is_aligned(q, 16)) return fail(HQ_ERR_MISALIGNED, "x and q must be 16-byte aligned");
  if (!is_aligned(scales, 4) || !is_aligned(amax_out, 4))
    return fail(HQ_ERR_MISALIGNED, "scales and amax_out must be 4-byte aligned");
  const Range outs[] = {{q, static_cast<size_t>(n), "q"},
                        {scales, static_cast<size_t>(ns) * 4, "scales"},
                        {amax_out, amax_out ? static_cast<size_t>(ns) * 4 : 0, "amax_out"}};
  const Range ins[] = {{x, static_cast<size_t>(n) * esize, "x"}};
  hq_status s = check_overlaps(outs, 3, ins, 1);
  if (s != HQ_OK) return s;
  const Range devs[] = {{x, 0, "x"}, {q, 0, "q"}, {scales, 0, "scales"}, {amax_out, 0, "amax_out"}};
  s = check_device_ptrs(devs, 4);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  hq::QuantizeArgs a;
  a.x = x; a.xt = xt; a.rows = rows; a.cols = cols; a.fmt = fmt; a.gran = HQ_PER_TOKEN;
  a.q = q; a.scales = scales; a.amax_out = amax_out;
  a.ring = nullptr; a.ring_len = 0; a.ring_idx = 0; a.ring_margin = 0;
  a.ws = nullptr;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.seed = seed;
  return launched(hq::launch_quantize_blockwise(a, block, stochastic != 0), "block-wise quantize launch");
}

hq_status hq_dequantize_fp8_blockwise(const uint8_t* q, hq_fp8_format fmt, int64_t rows, int64_t cols,
                                      int64_t block, const float* scales, hq_dtype out_type, void* out,
                                      hq_stream_t stream) {
  if (fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", (int)fmt);
  if (out_type != HQ_F32 && out_type != HQ_BF16) return fail(HQ_ERR_INVALID_ARG, "out_type must be F32 or BF16");
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  if (block < 16 || block % 16 != 0 || block >= k2p31)
    return fail(HQ_ERR_INVALID_ARG, "block = %lld must be a positive multiple of 16", (long long)block);
  if (cols % 16 != 0) return fail(HQ_ERR_INVALID_ARG, "cols must be a multiple of 16");
  const int64_t n = rows * cols;
  const int64_t ns = rows * ((cols + block - 1) / block);
  if (n == 0) return ok();
  if (!q || !scales || !out) return fail(HQ_ERR_INVALID_ARG, "q, scales and out must not be null");
  if (!is_aligned(q, 16) || !is_aligned(out, 16)) return fail(HQ_ERR_MISALIGNED, "q and out must be 16-byte aligned");
  if (!is_aligned(scales, 4)) return fail(HQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  const size_t osize = out_type == HQ_F32 ? 4 : 2;
  const Range outs[] = {{out, static_cast<size_t>(n) * osize, "out"}};
  const Range ins[] = {{q, static_cast<size_t>(n), "q"}, {scales, static_cast<size_t>(ns) * 4, "scales"}};
  hq_status s = check_overlaps(outs, 1, ins, 2);
  if (s != HQ_OK) return s;
  const Range devs[] = {{q, 0, "q"}, {scales, 0, "scales"}, {out, 0, "out"}};
  s = check_device_ptrs(devs, 3);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  return launched(hq::launch_dequantize_blockwise(q, fmt, rows, cols, block, scales, out_type == HQ_BF16, out,
                                                  reinterpret_cast<cudaStream_t>(stream)),
                  "block-wise dequantize launch");
}

size_t hq_grad_bias_workspace_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return 0;
  return hq::grad_bias_workspace_bytes(rows, cols);
}

hq_status hq_grad_bias(const void* g, hq_dtype gt, int64_t rows, int64_t cols, void* out, void* workspace,
                       size_t workspace_bytes, hq_stream_t stream) {
  if (gt != HQ_F32 && gt != HQ_BF16 && gt != HQ_F16) return fail(HQ_ERR_INVALID_ARG, "invalid dtype %d", (int)gt);
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  if (cols == 0) return ok();
  const size_t esize = (gt == HQ_F32) ? 4 : 2;
  const size_t need = hq::grad_bias_workspace_bytes(rows, cols);
  if (!out || !workspace || (rows > 0 && !g)) return fail(HQ_ERR_INVALID_ARG, "g, out and workspace must not be null");
  if (workspace_bytes < need)
    return fail(HQ_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  if ((g && !is_aligned(g, esize)) || !is_aligned(out, esize))
    return fail(HQ_ERR_MISALIGNED, "g and out must be aligned to their element size");
  if (!is_aligned(workspace, 256)) return fail(HQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  const Range outs[] = {{out, static_cast<size_t>(cols) * esize, "out"}, {workspace, need, "workspace"}};
  const Range ins[] = {{g, static_cast<size_t>(rows) * static_cast<size_t>(cols) * esize, "g"}};
  hq_status s = check_overlaps(outs, 2, ins, 1);
  if (s != HQ_OK) return s;
  const Range devs[] = {{g, 0, "g"}, {out, 0, "out"}, {workspace, 0, "workspace"}};
  s = check_device_ptrs(devs, 3);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  return launched(hq::launch_grad_bias(g, static_cast<int>(gt), rows, cols, out, workspace,
                                       reinterpret_cast<cudaStream_t>(stream)),
                  "bias gradient launch");
}

hq_status hq_quantize_e5m2_stochastic(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_granularity g,
                                      uint64_t seed, uint8_t* q, float* scales, float* amax_out, void* workspace,
                                      size_t workspace_bytes, hq_stream_t stream) {
  if (xt != HQ_F32 && xt != HQ_BF16 && xt != HQ_F16) return fail(HQ_ERR_INVALID_ARG, "invalid dtype %d", (int)xt);
  if (g != HQ_PER_TENSOR && g != HQ_PER_TOKEN && g != HQ_PER_CHANNEL)
    return fail(HQ_ERR_INVALID_ARG, "invalid granularity %d", (int)g);
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  const int64_t ns = hq_scale_count(g, rows, cols);
  const int64_t n = rows * cols;
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  const size_t need = hq::quantize_workspace_bytes(static_cast<int>(g), rows, cols, 0);
  if (ns == 0) return ok();
  if (n > 0 && (!x || !q)) return fail(HQ_ERR_INVALID_ARG, "x and q must not be null");
  if (!scales) return fail(HQ_ERR_INVALID_ARG, "scales must not be null");
  if (g == HQ_PER_CHANNEL && (static_cast<size_t>(cols) * esize) % 16 != 0)
    return fail(HQ_ERR_INVALID_ARG, "per-channel rows must be whole 16-byte units");
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(HQ_ERR_INVALID_ARG, "this mode needs a zeroed workspace of %zu bytes", need);
  if (!is_aligned(x, 16) || !is_aligned(q, 16)) return fail(HQ_ERR_MISALIGNED, "x and q must be 16-byte aligned");
  if (!is_aligned(scales, 4) || !is_aligned(amax_out, 4))
    return fail(HQ_ERR_MISALIGNED, "scales and amax_out must be 4-byte aligned");
  if (need > 0 && !is_aligned(workspace, 256)) return fail(HQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  const Range outs[] = {{q, static_cast<size_t>(n), "q"},
                        {scales, static_cast<size_t>(ns) * 4, "scales"},
                        {amax_out, amax_out ? static_cast<size_t>(ns) * 4 : 0, "amax_out"},
                        {need > 0 ? workspace : nullptr, need, "workspace"}};
  const Range ins[] = {{x, static_cast<size_t>(n) * esize, "x"}};
  hq_status s = check_overlaps(outs, 4, ins, 1);
  if (s != HQ_OK) return s;
  const Range devs[] = {{n > 0 ? x : nullptr, 0, "x"}, {n > 0 ? q : nullptr, 0, "q"}, {scales, 0, "scales"},
                        {amax_out, 0, "amax_out"}, {need > 0 ? workspace : nullptr, 0, "workspace"}};
  s = check_device_ptrs(devs, 5);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  hq::QuantizeArgs a;
  a.x = x; a.xt = xt; a.rows = rows; a.cols = cols; a.fmt = HQ_E5M2; a.gran = g;
  a.q = q; a.scales = scales; a.amax_out = amax_out;
  a.ring = nullptr; a.ring_len = 0; a.ring_idx = 0; a.ring_margin = 0;
  a.ws = workspace;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.seed = seed;
  return launched(hq::launch_quantize_sr(a), "stochastic quantize launch");
}

hq_status hq_quantize_fp8_transpose(const void* x, hq_dtype xt, int64_t rows, int64_t cols, hq_fp8_format fmt,
                                    uint8_t* q, uint8_t* qt, float* scales, float* amax_out, const float* multiplier,
                                    float* ring, int32_t ring_len, int32_t ring_idx, int32_t ring_margin,
                                    void* workspace, size_t workspace_bytes, hq_stream_t stream) {
  // ---- arguments
  if (xt != HQ_F32 && xt != HQ_BF16 && xt != HQ_F16) return fail(HQ_ERR_INVALID_ARG, "invalid dtype %d", (int)xt);
  if (fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", (int)fmt);
  if (rows < 0 || cols < 0) return fail(HQ_ERR_INVALID_ARG, "negative shape [%lld, %lld]", (long long)rows, (long long)cols);
  if (rows >= k2p31 || cols >= k2p31 || (cols > 0 && rows > (k2p40 - 1) / cols))
    return fail(HQ_ERR_TOO_LARGE, "shape [%lld, %lld] is beyond the supported range", (long long)rows, (long long)cols);
  if (rows % 16 != 0 || cols % 16 != 0)
    return fail(HQ_ERR_INVALID_ARG, "rows and cols must be multiples of 16 (16-byte code rows both ways)");
  if (multiplier && ring) return fail(HQ_ERR_INVALID_ARG, "give a multiplier or a ring, not both");
  if (ring) {
    if (ring_len < 1 || ring_len > (1 << 20)) return fail(HQ_ERR_INVALID_ARG, "ring_len %d outside [1, 2^20]", ring_len);
    if (ring_idx < 0 || ring_idx >= ring_len)
      return fail(HQ_ERR_INVALID_ARG, "ring_idx %d outside [0, %d)", ring_idx, ring_len);
    if (ring_margin < -126 || ring_margin > 126) return fail(HQ_ERR_INVALID_ARG, "ring_margin %d outside [-126, 126]", ring_margin);
  }
  const int64_t n = rows * cols;
  const size_t esize = (xt == HQ_F32) ? 4 : 2;
  const size_t need = hq::quantize_workspace_bytes(0, rows, cols, 1);
  if (n > 0 && (!x || !qt)) return fail(HQ_ERR_INVALID_ARG, "x and qt must not be null");
  if (!scales) return fail(HQ_ERR_INVALID_ARG, "scales must not be null");
  if (!workspace || workspace_bytes < need)
    return fail(HQ_ERR_INVALID_ARG, "a zeroed workspace of %zu bytes is needed", need);
  if (!is_aligned(x, 16) || !is_aligned(q, 16) || !is_aligned(qt, 16))
    return fail(HQ_ERR_MISALIGNED, "x, q and qt must start on 16-byte boundaries");
  if (!is_aligned(scales, 4) || !is_aligned(amax_out, 4) || !is_aligned(ring, 4) || !is_aligned(multiplier, 4))
    return fail(HQ_ERR_MISALIGNED, "scales, amax_out, multiplier and ring must be 4-byte aligned");
  if (!is_aligned(workspace, 256)) return fail(HQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  const Range outs[] = {{q, q ? static_cast<size_t>(n) : 0, "q"},
                        {qt, static_cast<size_t>(n), "qt"},
                        {scales, 4, "scales"},
                        {amax_out, amax_out ? 4u : 0u, "amax_out"},
                        {ring, ring ? static_cast<size_t>(ring_len + 2) * 4 : 0, "ring"},
                        {workspace, need, "workspace"}};
  const Range ins[] = {{x, static_cast<size_t>(n) * esize, "x"}, {multiplier, multiplier ? 4u : 0u, "multiplier"}};
  hq_status s = check_overlaps(outs, 6, ins, 2);
  if (s != HQ_OK) return s;
  // ---- device
  const Range devs[] = {{n > 0 ? x : nullptr, 0, "x"}, {q, 0, "q"}, {n > 0 ? qt : nullptr, 0, "qt"},
                        {scales, 0, "scales"}, {amax_out, 0, "amax_out"}, {multiplier, 0, "multiplier"},
                        {ring, 0, "ring"}, {workspace, 0, "workspace"}};
  s = check_device_ptrs(devs, 8);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  // ---- launch
  hq::QuantizeArgs a;
  a.x = x; a.xt = xt; a.rows = rows; a.cols = cols; a.fmt = fmt; a.gran = HQ_PER_TENSOR;
  a.q = q; a.scales = scales; a.amax_out = amax_out;
  a.ring = ring; a.ring_len = ring_len; a.ring_idx = ring_idx; a.ring_margin = ring_margin;
  a.ws = workspace;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.qt = qt;
  a.mult = multiplier;
  return launched(hq::launch_quantize_transpose(a), "quantize-transpose launch");
}

namespace {

// Fused epilogue arguments of hq_gemm_a8w8_ex (dense a8w8 only).
struct GemmEx {
  const void* bias;
  uint8_t* q_out;
  int q_fmt;
  float* q_scale;
  float* q_amax;
  float* ring;
  int32_t ring_len, ring_idx, ring_margin;
  void* workspace;
  size_t workspace_bytes;
  bool blockq = false;         // block-wise FP8 output (no ring) into q_out and q_bscales
  float* q_bscales = nullptr;  // dequant scales [M, N / q_block]
  int64_t q_block = 0;
};

hq_status gemm_common(int kind, const void* a, const void* b, int fmt, const float* xs, int64_t xs_len,
                      const float* ws, int64_t ws_len, const int32_t* offsets, int32_t E, int64_t M, int64_t N,
                      int64_t K, void* out, hq_stream_t stream, const GemmEx* ex = nullptr) {
  // FP8 output: q_out given, or (an empty result has no codes to point at)
  // a ring with no bf16 out
  const bool empty = M == 0 || N == 0;
  const bool bq = ex != nullptr && ex->blockq;  // block-wise FP8 output
  const bool fp8o = ex != nullptr && (ex->q_out != nullptr || (empty && (ex->ring != nullptr || bq) && out == nullptr));
  const bool grouped = offsets != nullptr || E != 1 || kind == 1;
  if (kind == 0 && fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", fmt);
  if (M < 0 || N < 0 || K < 0) return fail(HQ_ERR_INVALID_ARG, "negative size");
  if (M >= k2p31 || N >= k2p31 || K >= k2p31) return fail(HQ_ERR_TOO_LARGE, "M, N and K must be below 2^31");
  if (grouped) {
    if (E < 1 || E > 1024) return fail(HQ_ERR_INVALID_ARG, "E = %d outside [1, 1024]", E);
    if (!offsets) return fail(HQ_ERR_INVALID_ARG, "offsets must not be null");
    if (static_cast<int64_t>(E) * N >= k2p31) return fail(HQ_ERR_TOO_LARGE, "E*N must be below 2^31");
  }
  const int esize = kind == 0 ? 1 : 2;
  if ((K * esize) % 16 != 0)
    return fail(HQ_ERR_INVALID_ARG, "K = %lld: rows of A and B must be a multiple of 16 bytes", (long long)K);
  if (N % 8 != 0) return fail(HQ_ERR_INVALID_ARG, "N = %lld must be a multiple of 8 (16-byte output rows)", (long long)N);
  if (kind == 0) {
    if (!xs || !ws) return fail(HQ_ERR_INVALID_ARG, "x_scale and w_scale must not be null");
    if (xs_len != 1 && xs_len != M)
      return fail(HQ_ERR_INVALID_ARG, "x_scale_len %lld must be 1 or M = %lld", (long long)xs_len, (long long)M);
    const int64_t wn = grouped ? static_cast<int64_t>(E) * N : N;
    if (ws_len != 1 && ws_len != wn)
      return fail(HQ_ERR_INVALID_ARG, "w_scale_len %lld must be 1 or %lld", (long long)ws_len, (long long)wn);
    if (!is_aligned(xs, 4) || !is_aligned(ws, 4)) return fail(HQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  }
  size_t need = 0;
  if (ex) {
    if (grouped) return fail(HQ_ERR_INVALID_ARG, "fused epilogues are for the dense GEMM");
    if (fp8o == (out != nullptr)) return fail(HQ_ERR_INVALID_ARG, "exactly one of out and q_out must be given");
    if (ex->bias && !is_aligned(ex->bias, 4)) return fail(HQ_ERR_MISALIGNED, "bias must be 4-byte aligned");
    if (fp8o && bq) {
      if (ex->q_fmt != HQ_E4M3 && ex->q_fmt != HQ_E5M2)
        return fail(HQ_ERR_INVALID_ARG, "invalid q_fmt %d", ex->q_fmt);
      if (ex->q_block != 32) return fail(HQ_ERR_INVALID_ARG, "block = %lld: only 32 is supported", (long long)ex->q_block);
      if (N % 32 != 0) return fail(HQ_ERR_INVALID_ARG, "N = %lld must be a multiple of the block (32)", (long long)N);
      if (!empty && !ex->q_bscales) return fail(HQ_ERR_INVALID_ARG, "q_scales must not be null");
      if (!is_aligned(ex->q_out, 16)) return fail(HQ_ERR_MISALIGNED, "q_out must start on a 16-byte boundary");
      if (!is_aligned(ex->q_bscales, 4)) return fail(HQ_ERR_MISALIGNED, "q_scales must be 4-byte aligned");
    } else if (fp8o) {
      if (ex->q_fmt != HQ_E4M3 && ex->q_fmt != HQ_E5M2)
        return fail(HQ_ERR_INVALID_ARG, "invalid q_fmt %d", ex->q_fmt);
      if (!ex->ring) return fail(HQ_ERR_INVALID_ARG, "q_out needs a delayed-scaling ring");
      if (ex->ring_len < 1 || ex->ring_len > (1 << 20))
        return fail(HQ_ERR_INVALID_ARG, "ring_len %d outside [1, 2^20]", ex->ring_len);
      if (ex->ring_idx < 0 || ex->ring_idx >= ex->ring_len)
        return fail(HQ_ERR_INVALID_ARG, "ring_idx %d outside [0, %d)", ex->ring_idx, ex->ring_len);
      if (ex->ring_margin < -126 || ex->ring_margin > 126)
        return fail(HQ_ERR_INVALID_ARG, "ring_margin %d outside [-126, 126]", ex->ring_margin);
      if (!ex->q_scale) return fail(HQ_ERR_INVALID_ARG, "q_scale must not be null");
      need = hq::quantize_workspace_bytes(0, M, N, 1);
      if (!ex->workspace || ex->workspace_bytes < need)
        return fail(HQ_ERR_INVALID_ARG, "q_out needs a zeroed workspace of %zu bytes", need);
      if (N % 16 != 0) return fail(HQ_ERR_INVALID_ARG, "N = %lld must be a multiple of 16 with q_out", (long long)N);
      if (!is_aligned(ex->q_out, 16)) return fail(HQ_ERR_MISALIGNED, "q_out must start on a 16-byte boundary");
      if (!is_aligned(ex->q_scale, 4) || !is_aligned(ex->q_amax, 4) || !is_aligned(ex->ring, 4))
        return fail(HQ_ERR_MISALIGNED, "q_scale, q_amax and ring must be 4-byte aligned");
      if (!is_aligned(ex->workspace, 256)) return fail(HQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
    }
  }
  void* dst = fp8o ? static_cast<void*>(ex->q_out) : out;
  if ((!dst && !(fp8o && empty)) || (K > 0 && ((!a && M > 0) || (!b && N > 0))))
    return fail(HQ_ERR_INVALID_ARG, "operand and output pointers must not be null");
  if (!is_aligned(dst, 16)) return fail(HQ_ERR_MISALIGNED, "out must start on a 16-byte boundary");
  if (!is_aligned(a, 16) || !is_aligned(b, 16)) return fail(HQ_ERR_MISALIGNED, "A and B must be 16-byte aligned");
  if (offsets && !is_aligned(offsets, 4)) return fail(HQ_ERR_MISALIGNED, "offsets must be 4-byte aligned");
  const int64_t ebatch = grouped ? E : 1;
  const bool dq = fp8o && !bq;  // delayed per-tensor FP8 output
  const Range outs[] = {{dst, static_cast<size_t>(M) * static_cast<size_t>(N) * (fp8o ? 1 : 2), fp8o ? "q_out" : "out"},
                        {dq ? ex->q_scale : nullptr, 4, "q_scale"},
                        {dq ? ex->q_amax : nullptr, 4, "q_amax"},
                        {dq ? ex->ring : nullptr, dq ? static_cast<size_t>(ex->ring_len + 2) * 4 : 0, "ring"},
                        {dq ? ex->workspace : nullptr, need, "workspace"},
                        {bq ? ex->q_bscales : nullptr, bq ? static_cast<size_t>(M) * static_cast<size_t>(N / 32) * 4 : 0,
                         "q_scales"}};
  const Range ins[] = {{a, static_cast<size_t>(M * K * esize), "A"},
                       {b, static_cast<size_t>(ebatch * N * K * esize), "B"},
                       {xs, kind == 0 ? static_cast<size_t>(xs_len) * 4 : 0, "x_scale"},
                       {ws, kind == 0 ? static_cast<size_t>(ws_len) * 4 : 0, "w_scale"},
                       {offsets, offsets ? static_cast<size_t>(E + 1) * 4 : 0, "offsets"},
                       {ex ? ex->bias : nullptr, static_cast<size_t>(N) * 2, "bias"}};
  hq_status s = check_overlaps(outs, 6, ins, 6);
  if (s != HQ_OK) return s;
  const Range devs[] = {{a, 0, "A"}, {b, 0, "B"}, {xs, 0, "x_scale"}, {ws, 0, "w_scale"},
                        {offsets, 0, "offsets"}, {dst, 0, "out"}, {ex ? ex->bias : nullptr, 0, "bias"},
                        {dq ? ex->q_scale : nullptr, 0, "q_scale"}, {dq ? ex->q_amax : nullptr, 0, "q_amax"},
                        {dq ? ex->ring : nullptr, 0, "ring"}, {dq ? ex->workspace : nullptr, 0, "workspace"},
                        {bq ? ex->q_bscales : nullptr, 0, "q_scales"}};
  s = check_device_ptrs(devs, 12);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  if ((M == 0 || N == 0) && dq) {
    // the delayed quantize of the empty result: amax 0, the ring still steps
    hq::QuantizeArgs qa;
    qa.x = ex->workspace; qa.xt = HQ_BF16; qa.rows = M; qa.cols = N; qa.fmt = ex->q_fmt; qa.gran = HQ_PER_TENSOR;
    qa.q = ex->q_out; qa.scales = ex->q_scale; qa.amax_out = ex->q_amax;
    qa.ring = ex->ring; qa.ring_len = ex->ring_len; qa.ring_idx = ex->ring_idx; qa.ring_margin = ex->ring_margin;
    qa.ws = ex->workspace;
    qa.stream = reinterpret_cast<cudaStream_t>(stream);
    return launched(hq::launch_quantize(qa), "quantize launch");
  }
  if (M == 0 || N == 0) return ok();
  hq::GemmArgs g;
  g.kind = kind; g.fmt = fmt; g.a = a; g.b = b;
  g.x_scale = xs; g.x_scale_len = xs_len; g.w_scale = ws; g.w_scale_len = ws_len;
  g.offsets = offsets; g.E = grouped ? E : 1;
  g.M = M; g.N = N; g.K = K; g.out = out;
  g.stream = reinterpret_cast<cudaStream_t>(stream);
  if (ex) {
    g.bias = ex->bias;
    if (bq) {
      g.out = nullptr;
      g.q_out = ex->q_out; g.q_fmt = ex->q_fmt; g.q_bscales = ex->q_bscales;
    } else if (fp8o) {
      g.out = nullptr;
      g.q_out = ex->q_out; g.q_fmt = ex->q_fmt; g.q_scale = ex->q_scale; g.q_amax = ex->q_amax;
      g.ring = ex->ring; g.ring_len = ex->ring_len; g.ring_idx = ex->ring_idx; g.ring_margin = ex->ring_margin;
      g.q_ws = static_cast<uint32_t*>(ex->workspace);
    }
  }
  std::string msg;
  return launched(hq::launch_gemm(g, &msg), "gemm launch", msg);
}

}  // namespace

hq_status hq_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                       int64_t x_scale_len, const float* w_scale, int64_t w_scale_len, int64_t M, int64_t N,
                       int64_t K, void* out, hq_stream_t stream) {
  return gemm_common(0, xq, wq, fmt, x_scale, x_scale_len, w_scale, w_scale_len, nullptr, 1, M, N, K, out, stream);
}

hq_status hq_gemm_a8w8_ex(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                          int64_t x_scale_len, const float* w_scale, int64_t w_scale_len, const void* bias,
                          int64_t M, int64_t N, int64_t K, void* out, uint8_t* q_out, hq_fp8_format q_fmt,
                          float* q_scale, float* q_amax, float* ring, int32_t ring_len, int32_t ring_idx,
                          int32_t ring_margin, void* workspace, size_t workspace_bytes, hq_stream_t stream) {
  const GemmEx ex{bias, q_out, static_cast<int>(q_fmt), q_scale, q_amax, ring, ring_len, ring_idx, ring_margin,
                  workspace, workspace_bytes};
  return gemm_common(0, xq, wq, fmt, x_scale, x_scale_len, w_scale, w_scale_len, nullptr, 1, M, N, K, out, stream,
                     &ex);
}

hq_status hq_gemm_a8w8_blockq(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                              int64_t x_scale_len, const float* w_scale, int64_t w_scale_len, const void* bias,
                              int64_t M, int64_t N, int64_t K, uint8_t* q_out, hq_fp8_format q_fmt, int64_t block,
                              float* q_scales, hq_stream_t stream) {
  GemmEx ex{bias, q_out, static_cast<int>(q_fmt), nullptr, nullptr, nullptr, 0, 0, 0, nullptr, 0};
  ex.blockq = true;
  ex.q_bscales = q_scales;
  ex.q_block = block;
  return gemm_common(0, xq, wq, fmt, x_scale, x_scale_len, w_scale, w_scale_len, nullptr, 1, M, N, K, nullptr, stream,
                     &ex);
}

hq_status hq_gemm_blockscaled(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scales,
                              const float* w_scales, int64_t block, const void* bias, int64_t M, int64_t N, int64_t K,
                              void* out, hq_stream_t stream) {
  if (fmt != HQ_E4M3 && fmt != HQ_E5M2) return fail(HQ_ERR_INVALID_ARG, "invalid fp8 format %d", (int)fmt);
  if (M < 0 || N < 0 || K < 0) return fail(HQ_ERR_INVALID_ARG, "negative size");
  if (M >= k2p31 || N >= k2p31 || K >= k2p31) return fail(HQ_ERR_TOO_LARGE, "M, N and K must be below 2^31");
  if (block < 32 || block % 32 != 0 || block >= k2p31)
    return fail(HQ_ERR_INVALID_ARG, "block = %lld must be a positive multiple of 32", (long long)block);
  if (K % 16 != 0) return fail(HQ_ERR_INVALID_ARG, "K = %lld must be a multiple of 16", (long long)K);
  if (N % 8 != 0) return fail(HQ_ERR_INVALID_ARG, "N = %lld must be a multiple of 8 (16-byte output rows)", (long long)N);
  const int64_t nb = (K + block - 1) / block;
  if (!out || (K > 0 && ((!xq && M > 0) || (!wq && N > 0) || (!x_scales && M > 0) || (!w_scales && N > 0))))
    return fail(HQ_ERR_INVALID_ARG, "operands, scales and out must not be null");
  if (!is_aligned(out, 16) || !is_aligned(xq, 16) || !is_aligned(wq, 16) || !is_aligned(bias, 16))
    return fail(HQ_ERR_MISALIGNED, "A, B, bias and out must be 16-byte aligned");
  if (!is_aligned(x_scales, 4) || !is_aligned(w_scales, 4)) return fail(HQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  const Range outs[] = {{out, static_cast<size_t>(M) * static_cast<size_t>(N) * 2, "out"}};
  const Range ins[] = {{xq, static_cast<size_t>(M * K), "A"},
                       {wq, static_cast<size_t>(N * K), "B"},
                       {x_scales, static_cast<size_t>(M * nb) * 4, "x_scales"},
                       {w_scales, static_cast<size_t>(N * nb) * 4, "w_scales"},
                       {bias, bias ? static_cast<size_t>(N) * 2 : 0, "bias"}};
  hq_status s = check_overlaps(outs, 1, ins, 5);
  if (s != HQ_OK) return s;
  const Range devs[] = {{xq, 0, "A"}, {wq, 0, "B"}, {x_scales, 0, "x_scales"}, {w_scales, 0, "w_scales"},
                        {bias, 0, "bias"}, {out, 0, "out"}};
  s = check_device_ptrs(devs, 6);
  if (s != HQ_OK) return s;
  s = check_arch();
  if (s != HQ_OK) return s;
  if (M == 0 || N == 0) return ok();
  hq::BlockScaledGemmArgs g;
  g.fmt = fmt; g.a = xq; g.b = wq; g.x_scales = x_scales; g.w_scales = w_scales; g.block = block; g.bias = bias;
  g.M = M; g.N = N; g.K = K; g.out = out;
  g.stream = reinterpret_cast<cudaStream_t>(stream);
  std::string msg;
  return launched(hq::launch_gemm_blockscaled(g, &msg), "block-scaled gemm launch", msg);
}

hq_status hq_grouped_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, hq_fp8_format fmt, const float* x_scale,
                               int64_t x_scale_len, const float* w_scale, int64_t w_scale_len,
                               const int32_t* offsets, int32_t E, int64_t M_total, int64_t N, int64_t K, void* out,
                               hq_stream_t stream) {
  if (!offsets) return fail(HQ_ERR_INVALID_ARG, "offsets must not be null");
  return gemm_common(0, xq, wq, fmt, x_scale, x_scale_len, w_scale, w_scale_len, offsets, E, M_total, N, K, out,
                     stream);
}

hq_status hq_grouped_gemm_bf16(const void* x, const void* w, const int32_t* offsets, int32_t E, int64_t M_total,
                               int64_t N, int64_t K, void* out, hq_stream_t stream) {
  if (!offsets) return fail(HQ_ERR_INVALID_ARG, "offsets must not be null");
  return gemm_common(1, x, w, 0, nullptr, 0, nullptr, 0, offsets, E, M_total, N, K, out, stream);
}

hq_status hq_debug_bounded_wait(uint64_t limit_ns, hq_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 2000000000ull)
    return fail(HQ_ERR_INVALID_ARG, "limit_ns = %llu outside [1 us, 2 s]", (unsigned long long)limit_ns);
  hq_status s = check_arch();
  if (s != HQ_OK) return s;
  return launched(hq::launch_bounded_wait_probe(limit_ns, reinterpret_cast<cudaStream_t>(stream)),
                  "bounded-wait probe launch");
}

hq_status hq_check_device_error(void) {
  unsigned w = 0;
  const cudaError_t e = hq::read_and_clear_device_error(&w);
  if (e != cudaSuccess) return fail(HQ_ERR_CUDA, "device error check: %s", cudaGetErrorString(e));
  if (w & hq::kDevErrTimeout) {
    // a kernel that gave up may have left its scratch words set
    hq::noalloc_scratch_invalidate();
    return fail(HQ_ERR_TIMEOUT, "a kernel's bounded wait gave up");
  }
  if (w & hq::kDevErrBadOffsets) return fail(HQ_ERR_INVALID_ARG, "grouped GEMM offsets were malformed");
  return ok();
}

const char* hq_last_error(void) { return g_last_error.c_str(); }

const char* hq_version(void) { return "hq 0.1.0 (sm_100a)"; }

}  // extern "C"
