// quantize.cu -- dynamic FP8 quantization kernels for sm_100a.
//
// What is computed (hip-quant README "FP8 Formats" and "Training-path
// numerical guards"; AstrAI ops.cu quantize_bf16 and the ring commit;
// fuel-ir quant_scale.rs ScaleGranularity):
//   amax  = max |x| over the finite elements of a scale group
//   m     = fmax / amax (IEEE f32 division), 1 when amax == 0 or m is inf
//   q     = satfinite round-to-nearest-even FP8 code of f32(x) * m
//   scale = 1 / m (the dequant scale), amax_out = amax
//
// Kernel family (all memory bound; 16-byte vector loads, warp-shuffle
// reductions):
//   per-token   one pass: a warp (short rows) or a CTA (long rows) holds the
//               row in registers, reduces its amax, then casts it.
//   per-tensor  two launches: phase 1 reduces amax with per-CTA partials and
//               an atomicMax on the f32 bit pattern; the last CTA (threadfence
//               + counter election) publishes m.  Phase 2 casts, walking the
//               tensor backwards so its first reads hit what phase 1 left in L2.
//   per-channel the same two phases on [column strip x row band] tiles.
//   delayed     one pass with the multiplier already in the ring; the last
//               CTA folds amax into hist[idx] and publishes the next scale.
// No kernel here waits on another CTA: the last-CTA election only counts.
#include "hq_internal.cuh"

#include <cfloat>
#include <cuda_fp16.h>

namespace hq {
namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------ element types
// DT: 0 f32, 1 bf16, 2 f16.  VEC = elements per 16-byte vector.
template <int DT> struct Dt;
template <> struct Dt<0> {
  static constexpr int kSize = 4, kVec = 4;
  __device__ static float load1(const void* p, int64_t i) { return __ldg(static_cast<const float*>(p) + i); }
  __device__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};
template <> struct Dt<1> {
  static constexpr int kSize = 2, kVec = 8;
  __device__ static float load1(const void* p, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(p) + i)) << 16);
  }
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <> struct Dt<2> {
  static constexpr int kSize = 2, kVec = 8;
  __device__ static float load1(const void* p, int64_t i) {
    return __half2float(__ushort_as_half(__ldg(static_cast<const unsigned short*>(p) + i)));
  }
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  }
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

template <int FMT> struct Fmt;
template <> struct Fmt<0> { static constexpr float kMax = kFmaxE4M3; };
template <> struct Fmt<1> { static constexpr float kMax = kFmaxE5M2; };

// Two f32 values -> two FP8 codes (lo in the low byte), saturating
// round-to-nearest-even.  A NaN input gives the canonical code 0x7F.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  unsigned short r;
  if (FMT == 0)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  uint32_t v = r;
  v = isnan(lo) ? ((v & 0xFF00u) | 0x7Fu) : v;
  v = isnan(hi) ? ((v & 0x00FFu) | 0x7F00u) : v;
  return v;
}

template <int FMT>
__device__ __forceinline__ uint8_t cvt1(float y) {
  return static_cast<uint8_t>(cvt2<FMT>(y, 0.0f) & 0xFFu);
}

// |v| if finite, else 0 (NaN and +-Inf do not take part in amax).
__device__ __forceinline__ float finite_abs(float v) {
  const float a = fabsf(v);
  return (a <= FLT_MAX) ? a : 0.0f;
}

template <int DT>
__device__ __forceinline__ float vec_amax(const uint4& u, float acc) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
#pragma unroll
  for (int i = 0; i < Dt<DT>::kVec; ++i) acc = fmaxf(acc, finite_abs(f[i]));
  return acc;
}

// Scale the vector by m and store its codes (VEC bytes at dst).
template <int DT, int FMT>
__device__ __forceinline__ void vec_store_codes(uint8_t* dst, const uint4& u, float m) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
  if constexpr (Dt<DT>::kVec == 8) {
    uint2 o;
    o.x = cvt2<FMT>(__fmul_rn(f[0], m), __fmul_rn(f[1], m)) |
          (cvt2<FMT>(__fmul_rn(f[2], m), __fmul_rn(f[3], m)) << 16);
    o.y = cvt2<FMT>(__fmul_rn(f[4], m), __fmul_rn(f[5], m)) |
          (cvt2<FMT>(__fmul_rn(f[6], m), __fmul_rn(f[7], m)) << 16);
    *reinterpret_cast<uint2*>(dst) = o;
  } else {
    *reinterpret_cast<uint32_t*>(dst) =
        cvt2<FMT>(__fmul_rn(f[0], m), __fmul_rn(f[1], m)) |
        (cvt2<FMT>(__fmul_rn(f[2], m), __fmul_rn(f[3], m)) << 16);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Max over the whole CTA (kThreads threads); every thread gets the result.
__device__ __forceinline__ float block_max(float v, float* sh) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) sh[w] = v;
  __syncthreads();
  float r = (l < kThreads / 32) ? sh[l] : 0.0f;
  r = warp_max(r);
  return r;
}

// m = fmax / amax, with m = 1 for amax == 0 or a non-finite quotient.
__device__ __forceinline__ float multiplier(float amax, float fmax) {
  if (!(amax > 0.0f)) return 1.0f;
  const float m = __fdiv_rn(fmax, amax);
  return (m <= FLT_MAX) ? m : 1.0f;
}

// ---------------------------------------------------------------- per-token
// Vector path: TPR threads per row (32: a warp per row, 8 rows per CTA;
// 256: a CTA per row).  Each thread holds up to MAXV 16-byte vectors.
template <int DT, int FMT, int TPR, int MAXV>
__global__ void __launch_bounds__(kThreads) k_token_vec(
    const void* __restrict__ x, int64_t rows, int64_t cols, uint8_t* __restrict__ q,
    float* __restrict__ scales, float* __restrict__ amax_out) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int RPC = kThreads / TPR;
  __shared__ float sh[kThreads / 32];
  const int sub = threadIdx.x / TPR, t = threadIdx.x % TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + sub;
  const bool active = row < rows;
  const int64_t nv = cols / VEC;
  const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const char*>(x) +
                                                   (active ? row : 0) * cols * Dt<DT>::kSize);
  uint4 buf[MAXV];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int64_t v = static_cast<int64_t>(i) * TPR + t;
    if (active && v < nv) {
      buf[i] = ld_stream(xr + v);
      amax = vec_amax<DT>(buf[i], amax);
    }
  }
  if (TPR == 32) amax = warp_max(amax);
  else amax = block_max(amax, sh);
  const float m = multiplier(amax, Fmt<FMT>::kMax);
  if (active && t == 0) {
    scales[row] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[row] = amax;
  }
  uint8_t* qr = q + (active ? row : 0) * cols;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int64_t v = static_cast<int64_t>(i) * TPR + t;
    if (active && v < nv) vec_store_codes<DT, FMT>(qr + v * VEC, buf[i], m);
  }
}

// Any shape and alignment: one CTA per row, scalar loads, two passes over the
// row (the second pass reads it back from L1/L2).
template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads) k_token_generic(
    const void* __restrict__ x, int64_t rows, int64_t cols, uint8_t* __restrict__ q,
    float* __restrict__ scales, float* __restrict__ amax_out) {
  __shared__ float sh[kThreads / 32];
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  float amax = 0.0f;
  for (int64_t c = threadIdx.x; c < cols; c += kThreads)
    amax = fmaxf(amax, finite_abs(Dt<DT>::load1(x, row * cols + c)));
  amax = block_max(amax, sh);
  const float m = multiplier(amax, Fmt<FMT>::kMax);
  if (threadIdx.x == 0) {
    scales[row] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[row] = amax;
  }
  for (int64_t c = threadIdx.x; c < cols; c += kThreads)
    q[row * cols + c] = cvt1<FMT>(__fmul_rn(Dt<DT>::load1(x, row * cols + c), m));
}

// --------------------------------------------------------------- per-tensor
// Workspace words: [0] amax bits, [1] CTA counter, [2] the multiplier m
// published by phase 1 for phase 2.  All three are zero between calls.
constexpr int kUnroll = 4;

template <int DT, bool VECP>
__device__ __forceinline__ float flat_amax(const void* x, int64_t n) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  float amax = 0.0f;
  int64_t done = 0;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    int64_t v = gtid;
    for (; v + (kUnroll - 1) * gstride < nv; v += kUnroll * gstride) {
      uint4 u[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) u[j] = __ldg(xv + v + j * gstride);
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) amax = vec_amax<DT>(u[j], amax);
    }
    for (; v < nv; v += gstride) amax = vec_amax<DT>(__ldg(xv + v), amax);
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) amax = fmaxf(amax, finite_abs(Dt<DT>::load1(x, i)));
  return amax;
}

template <int DT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_tensor_amax(
    const void* __restrict__ x, int64_t n, uint32_t* __restrict__ ws, float fmax,
    float* __restrict__ scales, float* __restrict__ amax_out) {
  __shared__ float sh[kThreads / 32];
  __shared__ bool is_last;
  float amax = flat_amax<DT, VECP>(x, n);
  amax = block_max(amax, sh);
  if (threadIdx.x == 0) {
    atomicMax(&ws[0], __float_as_uint(amax));  // non-negative: bit order = value order
    __threadfence();
    is_last = atomicAdd(&ws[1], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    __threadfence();
    const float a = __uint_as_float(atomicExch(&ws[0], 0u));
    const float m = multiplier(a, fmax);
    ws[2] = __float_as_uint(m);
    scales[0] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[0] = a;
    atomicExch(&ws[1], 0u);
  }
}

// Cast with one multiplier; walks the vectors from the end backwards.
template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_tensor_cast(
    const void* __restrict__ x, int64_t n, uint32_t* __restrict__ ws, uint8_t* __restrict__ q) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ bool is_last;
  const float m = __uint_as_float(__ldcg(&ws[2]));
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t done = 0;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    int64_t i = gtid;
    for (; i + (kUnroll - 1) * gstride < nv; i += kUnroll * gstride) {
      uint4 u[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) u[j] = ld_stream(xv + (nv - 1 - (i + j * gstride)));
#pragma unroll
      for (int j = 0; j < kUnroll; ++j)
        vec_store_codes<DT, FMT>(q + (nv - 1 - (i + j * gstride)) * VEC, u[j], m);
    }
    for (; i < nv; i += gstride) {
      const int64_t v = nv - 1 - i;
      vec_store_codes<DT, FMT>(q + v * VEC, ld_stream(xv + v), m);
    }
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) q[i] = cvt1<FMT>(__fmul_rn(Dt<DT>::load1(x, i), m));
  // Every CTA has read m: the last one returns the workspace to zero.
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&ws[1], 1u) == gridDim.x - 1;
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    atomicExch(&ws[2], 0u);
    atomicExch(&ws[1], 0u);
  }
}

// -------------------------------------------------------------- per-channel
// Tile: a strip of 32 column vectors (32*VEC columns) x a band of rows.  Warp
// w of the CTA takes rows w, w+8, ... of the band; lane l owns column vector
// strip*32 + l.  Workspace: [0] counter, then amax bits[cols] (aligned to
// 16 bytes), then m[cols].
template <int DT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_channel_amax(
    const void* __restrict__ x, int64_t rows, int64_t cols, int64_t band_rows,
    uint32_t* __restrict__ counter, uint32_t* __restrict__ ws_amax, float* __restrict__ ws_m,
    float fmax, float* __restrict__ scales, float* __restrict__ amax_out) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ float sh[kThreads / 32][32 * VEC];
  __shared__ bool is_last;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t nvc = cols / VEC;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + l;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * band_rows;
  const int64_t r1 = min(rows, r0 + band_rows);
  float am[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) am[j] = 0.0f;
  if (cv < nvc) {
    if (VECP) {
      for (int64_t r = r0 + w; r < r1; r += kThreads / 32) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const char*>(x) +
                                                             (r * cols + cv * VEC) * Dt<DT>::kSize));
        float f[Dt<DT>::kVec];
        Dt<DT>::unpack(u, f);
#pragma unroll
        for (int j = 0; j < VEC; ++j) am[j] = fmaxf(am[j], finite_abs(f[j]));
      }
    } else {
      for (int64_t r = r0 + w; r < r1; r += kThreads / 32)
        am[0] = fmaxf(am[0], finite_abs(Dt<DT>::load1(x, r * cols + cv)));
    }
  }
#pragma unroll
  for (int j = 0; j < VEC; ++j) sh[w][l * VEC + j] = am[j];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * VEC; c += kThreads) {
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 * VEC + c;
    if (col < cols) {
      float a = sh[0][c];
#pragma unroll
      for (int ww = 1; ww < kThreads / 32; ++ww) a = fmaxf(a, sh[ww][c]);
      atomicMax(&ws_amax[col], __float_as_uint(a));
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(counter, 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int64_t c = threadIdx.x; c < cols; c += kThreads) {
      const float a = __uint_as_float(atomicExch(&ws_amax[c], 0u));
      const float m = multiplier(a, fmax);
      ws_m[c] = m;
      scales[c] = __fdiv_rn(1.0f, m);
      if (amax_out) amax_out[c] = a;
    }
    if (threadIdx.x == 0) atomicExch(counter, 0u);
  }
}

template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_channel_cast(
    const void* __restrict__ x, int64_t rows, int64_t cols, int64_t band_rows,
    uint32_t* __restrict__ counter, float* __restrict__ ws_m, uint8_t* __restrict__ q) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ bool is_last;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t nvc = cols / VEC;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + l;
  if (cv < nvc) {
    // bands in reverse launch order: the last band read by phase 1 goes first
    const int64_t band = static_cast<int64_t>(gridDim.y) - 1 - blockIdx.y;
    const int64_t r0 = band * band_rows;
    const int64_t r1 = min(rows, r0 + band_rows);
    float m[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) m[j] = __ldcg(&ws_m[cv * VEC + j]);
    const int64_t nrows = r1 - r0;
    for (int64_t i = w; i < nrows; i += kThreads / 32) {
      const int64_t r = r1 - 1 - i;
      if (VECP) {
        const uint4 u = ld_stream(reinterpret_cast<const uint4*>(static_cast<const char*>(x) +
                                                                 (r * cols + cv * VEC) * Dt<DT>::kSize));
        float f[Dt<DT>::kVec];
        Dt<DT>::unpack(u, f);
        if constexpr (Dt<DT>::kVec == 8) {
          uint2 o;
          o.x = cvt2<FMT>(__fmul_rn(f[0], m[0]), __fmul_rn(f[1], m[1])) |
                (cvt2<FMT>(__fmul_rn(f[2], m[2]), __fmul_rn(f[3], m[3])) << 16);
          o.y = cvt2<FMT>(__fmul_rn(f[4], m[4]), __fmul_rn(f[5], m[5])) |
                (cvt2<FMT>(__fmul_rn(f[6], m[6]), __fmul_rn(f[7], m[7])) << 16);
          *reinterpret_cast<uint2*>(q + r * cols + cv * VEC) = o;
        } else {
          *reinterpret_cast<uint32_t*>(q + r * cols + cv * VEC) =
              cvt2<FMT>(__fmul_rn(f[0], m[0]), __fmul_rn(f[1], m[1])) |
              (cvt2<FMT>(__fmul_rn(f[2], m[2]), __fmul_rn(f[3], m[3])) << 16);
        }
      } else {
        q[r * cols + cv] = cvt1<FMT>(__fmul_rn(Dt<DT>::load1(x, r * cols + cv), m[0]));
      }
    }
  }
  // Every CTA has read its multipliers: the last one zeroes them and the
  // counter, so the whole workspace is zero again when the call ends.
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(counter, 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (is_last) {
    for (int64_t c = threadIdx.x; c < cols; c += kThreads) ws_m[c] = 0.0f;
    __syncthreads();
    if (threadIdx.x == 0) atomicExch(counter, 0u);
  }
}

// ------------------------------------------------------------------ delayed
// Ring: [hist[len] | scale | counter].  Workspace word [0]: amax accumulator.
template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_delayed(
    const void* __restrict__ x, int64_t n, uint8_t* __restrict__ q, float* __restrict__ ring,
    int len, int idx, int margin, uint32_t* __restrict__ ws, float* __restrict__ scales,
    float* __restrict__ amax_out) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ float sh[kThreads / 32];
  __shared__ bool is_last;
  const float m = __ldcg(&ring[len]);
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  float amax = 0.0f;
  int64_t done = 0;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    int64_t v = gtid;
    for (; v + (kUnroll - 1) * gstride < nv; v += kUnroll * gstride) {
      uint4 u[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) u[j] = ld_stream(xv + v + j * gstride);
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) {
        amax = vec_amax<DT>(u[j], amax);
        vec_store_codes<DT, FMT>(q + (v + j * gstride) * VEC, u[j], m);
      }
    }
    for (; v < nv; v += gstride) {
      const uint4 u = ld_stream(xv + v);
      amax = vec_amax<DT>(u, amax);
      vec_store_codes<DT, FMT>(q + v * VEC, u, m);
    }
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) {
    const float f = Dt<DT>::load1(x, i);
    amax = fmaxf(amax, finite_abs(f));
    q[i] = cvt1<FMT>(__fmul_rn(f, m));
  }
  amax = block_max(amax, sh);
  uint32_t* counter = reinterpret_cast<uint32_t*>(ring + len + 1);
  if (threadIdx.x == 0) {
    atomicMax(&ws[0], __float_as_uint(amax));
    __threadfence();
    is_last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  __shared__ float a_sh;
  if (threadIdx.x == 0) {
    const float a = __uint_as_float(atomicExch(&ws[0], 0u));
    a_sh = a;
    ring[idx] = a;  // fold this step's amax into the history slot
    __threadfence_block();
  }
  __syncthreads();
  float win = 0.0f;
  for (int i = threadIdx.x; i < len; i += kThreads) win = fmaxf(win, __ldcg(&ring[i]));
  win = block_max(win, sh);
  if (threadIdx.x == 0) {
    const float a = a_sh;
    if (win <= FLT_MAX && win > 0.0f) {
      const float next = ldexpf(__fdiv_rn(Fmt<FMT>::kMax, win), -margin);
      if (next <= FLT_MAX && next > 0.0f) ring[len] = next;
    }
    scales[0] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[0] = a;
    atomicExch(counter, 0u);
  }
}

// ------------------------------------------------------------------- launch
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int flat_grid(int64_t nvec, int dev) {
  const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
  int64_t g = (nvec + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(device_sm_count(dev)) * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

template <int DT, int FMT, int TPR>
cudaError_t launch_token_vec(const QuantizeArgs& a, int maxv) {
  const int rpc = kThreads / TPR;
  const dim3 grid(static_cast<unsigned>((a.rows + rpc - 1) / rpc));
  switch (maxv) {
#define HQ_TOKEN_CASE(MV)                                                                   \
  case MV:                                                                                 \
    k_token_vec<DT, FMT, TPR, MV><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q, \
                                                                  a.scales, a.amax_out);   \
    break;
    HQ_TOKEN_CASE(1)
    HQ_TOKEN_CASE(2)
    HQ_TOKEN_CASE(4)
    HQ_TOKEN_CASE(8)
    HQ_TOKEN_CASE(16)
#undef HQ_TOKEN_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

inline int pow2_at_least(int64_t v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

template <int DT, int FMT>
cudaError_t launch_typed(const QuantizeArgs& a) {
  constexpr int VEC = Dt<DT>::kVec;
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t n = a.rows * a.cols;
  const float fmax = Fmt<FMT>::kMax;
  const bool flat_vec = aligned(a.x, 16) && aligned(a.q, VEC);
  const bool row_vec = flat_vec && ((a.cols * Dt<DT>::kSize) % 16 == 0);

  if (a.ring) {  // delayed per-tensor
    uint32_t* ws = static_cast<uint32_t*>(a.ws);
    const int grid = flat_grid(flat_vec ? n / VEC : n, dev);
    if (flat_vec)
      k_delayed<DT, FMT, true><<<grid, kThreads, 0, a.stream>>>(a.x, n, a.q, a.ring, a.ring_len, a.ring_idx,
                                                                a.ring_margin, ws, a.scales, a.amax_out);
    else
      k_delayed<DT, FMT, false><<<grid, kThreads, 0, a.stream>>>(a.x, n, a.q, a.ring, a.ring_len, a.ring_idx,
                                                                 a.ring_margin, ws, a.scales, a.amax_out);
    return cudaGetLastError();
  }

  if (a.gran == 1) {  // per-token
    if (row_vec) {
      const int64_t nv = a.cols / VEC;
      if (nv <= 32 * 8) return launch_token_vec<DT, FMT, 32>(a, pow2_at_least((nv + 31) / 32));
      if (nv <= static_cast<int64_t>(kThreads) * 16)
        return launch_token_vec<DT, FMT, kThreads>(a, pow2_at_least((nv + kThreads - 1) / kThreads));
    }
    k_token_generic<DT, FMT><<<static_cast<unsigned>(a.rows), kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q,
                                                                                        a.scales, a.amax_out);
    return cudaGetLastError();
  }

  if (a.gran == 0) {  // per-tensor, two phases
    uint32_t* ws = static_cast<uint32_t*>(a.ws);
    const int grid = flat_grid(flat_vec ? n / VEC : n, dev);
    if (flat_vec)
      k_tensor_amax<DT, true><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, fmax, a.scales, a.amax_out);
    else
      k_tensor_amax<DT, false><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, fmax, a.scales, a.amax_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || n == 0) return e;
    if (flat_vec)
      k_tensor_cast<DT, FMT, true><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, a.q);
    else
      k_tensor_cast<DT, FMT, false><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, a.q);
    return cudaGetLastError();
  }

  // per-channel, two phases
  const int vec = row_vec ? VEC : 1;
  const int64_t nvc = a.cols / vec;
  const int64_t strips = (nvc + 31) / 32;
  const int64_t target = static_cast<int64_t>(device_sm_count(dev)) * 4;
  int64_t bands = (target + strips - 1) / strips;
  if (bands > a.rows) bands = a.rows;
  if (bands < 1) bands = 1;
  if (bands > 65535) bands = 65535;
  const int64_t band_rows = a.rows > 0 ? (a.rows + bands - 1) / bands : 1;
  bands = a.rows > 0 ? (a.rows + band_rows - 1) / band_rows : 1;
  if (strips > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(bands));
  uint32_t* counter = static_cast<uint32_t*>(a.ws);
  uint32_t* ws_amax = counter + 4;
  float* ws_m = reinterpret_cast<float*>(ws_amax + ((a.cols + 3) / 4) * 4);
  if (row_vec)
    k_channel_amax<DT, true><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, counter, ws_amax,
                                                              ws_m, fmax, a.scales, a.amax_out);
  else
    k_channel_amax<DT, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, counter, ws_amax,
                                                               ws_m, fmax, a.scales, a.amax_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n == 0) return e;
  if (row_vec)
    k_channel_cast<DT, FMT, true><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, counter, ws_m,
                                                                   a.q);
  else
    k_channel_cast<DT, FMT, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, counter, ws_m,
                                                                    a.q);
  return cudaGetLastError();
}

}  // namespace

size_t quantize_workspace_bytes(int gran, int64_t rows, int64_t cols, int delayed) {
  (void)rows;
  if (delayed) return 256;
  if (gran == 0) return 256;
  if (gran == 1) return 0;
  // counter (16 bytes), amax bits[cols] padded to 16 bytes, m[cols]
  const size_t c4 = static_cast<size_t>((cols + 3) / 4) * 4;
  size_t b = 16 + c4 * 4 + static_cast<size_t>(cols) * 4;
  return (b + 255) / 256 * 256;
}

cudaError_t launch_quantize(const QuantizeArgs& a) {
  const int key = a.xt * 2 + a.fmt;
  switch (key) {
    case 0: return launch_typed<0, 0>(a);
    case 1: return launch_typed<0, 1>(a);
    case 2: return launch_typed<1, 0>(a);
    case 3: return launch_typed<1, 1>(a);
    case 4: return launch_typed<2, 0>(a);
    case 5: return launch_typed<2, 1>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
