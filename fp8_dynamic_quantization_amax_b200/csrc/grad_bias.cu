// grad_bias.cu -- the bias gradient of a linear layer's backward pass:
// out[c] = dtype( sum over r of g[r, c] ), accumulated in f32 (AstrAI
// csrc/kernels/fp8/ops.cu linear_backward_fp8: the bias gradient is g summed
// over dim 0 and cast back to g's dtype).  sm_100a only.
//
// One launch over [column strip x row band] tiles.  A strip is 256 column
// vectors (16-byte vectors when every row starts 16-byte aligned, else
// single elements); a band is a fixed share of the rows.  Thread t of CTA
// (strip, band) sums column vector t of the strip over the band's rows in
// order (eight rows' loads in flight) and writes the f32 partial sums to the
// workspace.  The last CTA of a strip to finish (one counter per strip)
// adds the bands' partials in band order and rounds each column once to g's
// dtype, then returns its counter to zero.  The summation order is fixed,
// so results do not depend on which CTA finishes last.
#include "hq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace hq {
namespace {

constexpr int kGbThreads = 256;   // column vectors per strip
constexpr int64_t kGbMaxBands = 64;
constexpr int64_t kGbBandRows = 32;   // at least this many rows per band
constexpr int kGbRowsInFlight = 8;    // a thread's row loads in flight
constexpr int kGbBandsInFlight = 8;   // the final sum's partial loads in flight

__host__ __device__ inline int64_t gb_bands(int64_t rows) {
  int64_t b = (rows + kGbBandRows - 1) / kGbBandRows;
  return b < 1 ? 1 : (b > kGbMaxBands ? kGbMaxBands : b);
}

template <int XT>
__device__ __forceinline__ float gb_load1(const void* g, int64_t i) {
  if (XT == 0) return __ldg(static_cast<const float*>(g) + i);
  const unsigned short h = __ldg(static_cast<const unsigned short*>(g) + i);
  if (XT == 1) return __uint_as_float(static_cast<uint32_t>(h) << 16);
  return __half2float(__ushort_as_half(h));
}

// the 16-byte vector at element i, and its 4 f32 or 8 16-bit values widened
// (volatile asm: a run of these stays in program order, ahead of the adds
// that consume them, so a thread keeps all of a run's loads in flight)
template <int XT>
__device__ __forceinline__ uint4 gb_load_raw(const void* g, int64_t i) {
  uint4 u;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
               : "l"(static_cast<const char*>(g) + i * (XT == 0 ? 4 : 2)));
  return u;
}
template <int XT>
__device__ __forceinline__ void gb_widen(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if (XT == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) f[j] = __uint_as_float(w[j]);
  } else if (XT == 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = __uint_as_float(w[j] << 16);
      f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xFFFFu)));
      f[2 * j + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
    }
  }
}

template <int XT>
__device__ __forceinline__ void gb_store1(void* out, int64_t c, float v) {
  if (XT == 0) static_cast<float*>(out)[c] = v;
  else if (XT == 1) static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(v);
  else static_cast<__half*>(out)[c] = __float2half_rn(v);
}

// VEC: elements per column vector (16 / element size on the vector path, 1
// otherwise).  Workspace: counters [strips] (padded to 256 bytes), then the
// partials [bands][cols] f32.
template <int XT, int VEC>
__global__ void __launch_bounds__(kGbThreads) k_grad_bias(const void* __restrict__ g, int64_t rows, int64_t cols,
                                                          int strips, int64_t band_rows, void* __restrict__ out,
                                                          uint32_t* __restrict__ counters,
                                                          float* __restrict__ part) {
  __shared__ int s_last;
  const int strip = static_cast<int>(blockIdx.x % strips);
  const int64_t band = blockIdx.x / strips;
  const int64_t bands = gridDim.x / strips;
  const int64_t nvc = cols / VEC;                                   // column vectors
  const int64_t cv = static_cast<int64_t>(strip) * kGbThreads + threadIdx.x;
  const bool active = cv < nvc;
  const int64_t r0 = band * band_rows;
  const int64_t r1 = min(rows, r0 + band_rows);
  float acc[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) acc[j] = 0.0f;
  if (active) {
    int64_t r = r0;
    for (; r + (kGbRowsInFlight - 1) < r1; r += kGbRowsInFlight) {  // loads in flight, added in row order
      if (VEC == 1) {
        float f[kGbRowsInFlight];
#pragma unroll
        for (int k = 0; k < kGbRowsInFlight; ++k) f[k] = gb_load1<XT>(g, (r + k) * cols + cv);
#pragma unroll
        for (int k = 0; k < kGbRowsInFlight; ++k) acc[0] = __fadd_rn(acc[0], f[k]);
      } else {
        uint4 u[kGbRowsInFlight];  // all the loads first, then the adds in row order
#pragma unroll
        for (int k = 0; k < kGbRowsInFlight; ++k) u[k] = gb_load_raw<XT>(g, (r + k) * cols + cv * VEC);
        // the adds read acc through this (volatile, so after the loads) empty
        // asm: none of them is scheduled between the loads
#pragma unroll
        for (int j = 0; j < VEC; ++j) asm volatile("" : "+f"(acc[j]));
#pragma unroll
        for (int k = 0; k < kGbRowsInFlight; ++k) {
          float f[VEC];
          gb_widen<XT>(u[k], f);
#pragma unroll
          for (int j = 0; j < VEC; ++j) acc[j] = __fadd_rn(acc[j], f[j]);
        }
      }
    }
    for (; r < r1; ++r) {
      float f[VEC];
      if (VEC == 1) f[0] = gb_load1<XT>(g, r * cols + cv);
      else gb_widen<XT>(gb_load_raw<XT>(g, r * cols + cv * VEC), f);
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[j] = __fadd_rn(acc[j], f[j]);
    }
    float* pp = part + band * cols + cv * VEC;
    if (VEC == 1) {
      pp[0] = acc[0];
    } else {
#pragma unroll
      for (int j = 0; j < VEC; j += 4) *reinterpret_cast<float4*>(pp + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
  }
  // the last CTA of the strip (acquire-release counter) reduces the bands
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(counters + strip) : "memory");
    s_last = (prev == static_cast<uint32_t>(bands - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (active) {
    // the bands' partials of this column vector, kGbBandsInFlight bands'
    // loads at a time, added in band order
    float s[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) s[j] = 0.0f;
    const float* pp = part + cv * VEC;
    int64_t b = 0;
    for (; b + (kGbBandsInFlight - 1) < bands; b += kGbBandsInFlight) {
      float f[kGbBandsInFlight][VEC];
#pragma unroll
      for (int k = 0; k < kGbBandsInFlight; ++k) {
        if (VEC == 1) {
          f[k][0] = __ldcg(pp + (b + k) * cols);
        } else {
#pragma unroll
          for (int j = 0; j < VEC; j += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pp + (b + k) * cols + j));
            f[k][j] = v.x; f[k][j + 1] = v.y; f[k][j + 2] = v.z; f[k][j + 3] = v.w;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kGbBandsInFlight; ++k)
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[j] = __fadd_rn(s[j], f[k][j]);
    }
    for (; b < bands; ++b)
#pragma unroll
      for (int j = 0; j < VEC; ++j) s[j] = __fadd_rn(s[j], __ldcg(pp + b * cols + j));
#pragma unroll
    for (int j = 0; j < VEC; ++j) gb_store1<XT>(out, cv * VEC + j, s[j]);
  }
  if (threadIdx.x == 0) atomicExch(counters + strip, 0u);
}

template <int XT, int VEC>
cudaError_t launch_gb(const void* g, int64_t rows, int64_t cols, void* out, void* ws, cudaStream_t stream) {
  const int64_t nvc = cols / VEC;
  const int strips = static_cast<int>((nvc + kGbThreads - 1) / kGbThreads);
  const int64_t bands = gb_bands(rows);
  const int64_t band_rows = (rows + bands - 1) / bands;
  uint32_t* counters = static_cast<uint32_t*>(ws);
  const int64_t ncnt = (cols + kGbThreads - 1) / kGbThreads;  // the scalar path's strip count bounds both
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + (ncnt * 4 + 255) / 256 * 256);
  k_grad_bias<XT, VEC><<<static_cast<unsigned>(strips * bands), kGbThreads, 0, stream>>>(
      g, rows, cols, strips, band_rows, out, counters, part);
  return cudaGetLastError();
}

}  // namespace

size_t grad_bias_workspace_bytes(int64_t rows, int64_t cols) {
  const int64_t ncnt = (cols + kGbThreads - 1) / kGbThreads;
  return static_cast<size_t>((ncnt * 4 + 255) / 256 * 256) +
         static_cast<size_t>(gb_bands(rows)) * static_cast<size_t>(cols) * 4;
}

cudaError_t launch_grad_bias(const void* g, int xt, int64_t rows, int64_t cols, void* out, void* ws,
                             cudaStream_t stream) {
  const int esize = (xt == 0) ? 4 : 2;
  const int vec = 16 / esize;
  const bool vpath = (reinterpret_cast<uintptr_t>(g) % 16 == 0) && ((cols * esize) % 16 == 0);
  if (xt == 0) return vpath ? launch_gb<0, 4>(g, rows, cols, out, ws, stream) : launch_gb<0, 1>(g, rows, cols, out, ws, stream);
  if (xt == 1) return vpath ? launch_gb<1, 8>(g, rows, cols, out, ws, stream) : launch_gb<1, 1>(g, rows, cols, out, ws, stream);
  (void)vec;
  return vpath ? launch_gb<2, 8>(g, rows, cols, out, ws, stream) : launch_gb<2, 1>(g, rows, cols, out, ws, stream);
}

}  // namespace hq
