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
// Kernel family (memory bound; every kernel keeps several 16-byte loads or
// bulk copies in flight per thread; only the single-launch kernels wait on
// other CTAs, at one bounded grid barrier of a cooperative launch):
//   per-token   one pass, persistent CTAs: a ring of shared-memory stages is
//               filled by 1-D bulk copies (TMA), each stage a group of whole
//               rows; a stage is reduced and cast while the next ones load.
//               Unaligned or very long rows take a scalar path.
//   per-tensor  large aligned inputs: one cooperative launch that keeps the
//               first part of each CTA's range in shared and tensor memory
//               across the grid barrier and re-reads the rest from L2.
//               Otherwise two launches: phase 1 reduces amax with per-CTA
//               partials and an atomicMax on the f32 bit pattern, the last
//               CTA (threadfence + counter election) publishes m; phase 2
//               casts, walking the tensor backwards to reuse L2.
//   per-channel the same two forms on [column strip x row band] tiles.
//   delayed     one pass with the multiplier already in the ring; the last
//               CTA folds amax into hist[idx] and publishes the next scale.
//   transposed  per-tensor codes written row-major and transposed through
//               64 x 64 shared-memory tiles (the backward GEMMs' operands).
//   stochastic  E5M2 with one counter-based SplitMix64 draw per element.
//   block-wise  one scale per block along the last dimension: the per-token
//               stage pipeline with warp-level block reductions.
//
// Instruction economy (the kernels are ALU-issue bound otherwise):
//   - amax runs on raw bit patterns: for non-negative floats the unsigned
//     order of the bits is the numeric order, so |x| is one AND and the max
//     is one max.u16x2 per two bf16/f16 elements (one max.u32 per f32).
//   - Inf/NaN have the all-ones exponent, so the raw maximum also tells
//     whether any non-finite element was seen.  Only then does a thread redo
//     its range on the exact path (finite-only amax, canonical NaN codes).
//   - the cast is one FMUL per element plus one cvt.rn.satfinite per pair.
#include "fp8_cvt.cuh"
#include "hq_internal.cuh"
#include "launch.cuh"
#include "ptx.cuh"

#include <algorithm>
#include <cstring>
#include <cfloat>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <type_traits>
#include <mutex>

namespace hq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;        // delayed kernel (casts and reduces: register bound)
constexpr int kUnrollFlat = 8;    // per-tensor phases: eight 16-byte loads in flight per thread
constexpr int kMaxStages = 4;
constexpr int kRowUnroll = 8;     // per-channel: rows loaded per step

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ------------------------------------------------------------ element types
// DT: 0 f32, 1 bf16, 2 f16.  kVec = elements per 16-byte vector.  A "raw
// magnitude word" is a 32-bit word of the input with the sign bits cleared;
// lmax takes the lane-wise maximum of two such words (2 lanes for 16-bit
// types, 1 for f32).
template <int DT> struct Dt;
template <> struct Dt<0> {
  static constexpr int kSize = 4, kVec = 4, kLanes = 1;
  __device__ static float load1(const void* p, int64_t i) { return __ldg(static_cast<const float*>(p) + i); }
  __device__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static uint32_t mag(uint32_t w) { return w & 0x7FFFFFFFu; }
  __device__ static uint32_t lmax(uint32_t a, uint32_t b) { return max(a, b); }
  __device__ static bool nonfinite(uint32_t m) { return m >= 0x7F800000u; }
  __device__ static float lane_value(uint32_t m, int) { return __uint_as_float(m); }
  __device__ static float value(uint32_t m) { return __uint_as_float(m); }
};
template <> struct Dt<1> {
  static constexpr int kSize = 2, kVec = 8, kLanes = 2;
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
  __device__ static uint32_t mag(uint32_t w) { return w & 0x7FFF7FFFu; }
  __device__ static uint32_t lmax(uint32_t a, uint32_t b) { return max_u16x2(a, b); }
  // a lane >= 0x7F80 (exponent all ones) carries into its bit 15
  __device__ static bool nonfinite(uint32_t m) { return ((m + 0x00800080u) & 0x80008000u) != 0; }
  __device__ static float lane_value(uint32_t m, int lane) {
    return __uint_as_float(((m >> (16 * lane)) & 0xFFFFu) << 16);
  }
  __device__ static float value(uint32_t m) { return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16); }
};
template <> struct Dt<2> {
  static constexpr int kSize = 2, kVec = 8, kLanes = 2;
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
  __device__ static uint32_t mag(uint32_t w) { return w & 0x7FFF7FFFu; }
  __device__ static uint32_t lmax(uint32_t a, uint32_t b) { return max_u16x2(a, b); }
  // a lane >= 0x7C00 (exponent all ones) carries into its bit 15
  __device__ static bool nonfinite(uint32_t m) { return ((m + 0x04000400u) & 0x80008000u) != 0; }
  __device__ static float lane_value(uint32_t m, int lane) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>((m >> (16 * lane)) & 0xFFFFu)));
  }
  __device__ static float value(uint32_t m) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(max(m & 0xFFFFu, m >> 16))));
  }
};

// Raw magnitude maximum of the elements of one 16-byte vector.
template <int DT>
__device__ __forceinline__ uint32_t vec_mag(const uint4& u) {
  return Dt<DT>::lmax(Dt<DT>::lmax(Dt<DT>::mag(u.x), Dt<DT>::mag(u.y)),
                      Dt<DT>::lmax(Dt<DT>::mag(u.z), Dt<DT>::mag(u.w)));
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

template <int FMT> struct Fmt;
template <> struct Fmt<0> { static constexpr float kMax = kFmaxE4M3; };
template <> struct Fmt<1> { static constexpr float kMax = kFmaxE5M2; };

// Four f32 values -> four FP8 codes in one word (a0 in the low byte),
// saturating round-to-nearest-even.  Inputs must not be NaN.
template <int FMT>
__device__ __forceinline__ uint32_t cvt4(float a0, float a1, float a2, float a3) {
  uint32_t d;
  if (FMT == 0)
    asm("{\n\t.reg .b16 l, h;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\t"
        "mov.b32 %0, {l, h};\n\t}"
        : "=r"(d) : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  else
    asm("{\n\t.reg .b16 l, h;\n\t"
        "cvt.rn.satfinite.e5m2x2.f32 l, %2, %1;\n\t"
        "cvt.rn.satfinite.e5m2x2.f32 h, %4, %3;\n\t"
        "mov.b32 %0, {l, h};\n\t}"
        : "=r"(d) : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return d;
}

template <int DT>
__device__ __forceinline__ float vec_amax_exact(const uint4& u, float acc) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
#pragma unroll
  for (int i = 0; i < Dt<DT>::kVec; ++i) acc = fmaxf(acc, finite_abs(f[i]));
  return acc;
}

// Four f32 codes-to-be (already scaled) -> one word, on the fast (no NaN) or
// the exact path.
template <int FMT, bool FAST>
__device__ __forceinline__ uint32_t pack4(float a0, float a1, float a2, float a3) {
  if (FAST) return cvt4<FMT>(a0, a1, a2, a3);
  return cvt2_exact<FMT>(a0, a1) | (cvt2_exact<FMT>(a2, a3) << 16);
}

// Scale one vector by m and store its codes (kVec bytes at dst).  FAST: the
// vector holds no NaN (checked by the caller) and m is finite.
template <int DT, int FMT, bool FAST>
__device__ __forceinline__ void vec_store(uint8_t* dst, const uint4& u, float m) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
#pragma unroll
  for (int i = 0; i < Dt<DT>::kVec; ++i) f[i] = __fmul_rn(f[i], m);
  if constexpr (Dt<DT>::kVec == 8) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack4<FMT, FAST>(f[0], f[1], f[2], f[3]), pack4<FMT, FAST>(f[4], f[5], f[6], f[7]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack4<FMT, FAST>(f[0], f[1], f[2], f[3]);
  }
}

// The same with one multiplier per element (per-channel).
template <int DT, int FMT, bool FAST>
__device__ __forceinline__ void vec_store_m(uint8_t* dst, const uint4& u, const float (&m)[Dt<DT>::kVec]) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
#pragma unroll
  for (int i = 0; i < Dt<DT>::kVec; ++i) f[i] = __fmul_rn(f[i], m[i]);
  if constexpr (Dt<DT>::kVec == 8) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack4<FMT, FAST>(f[0], f[1], f[2], f[3]), pack4<FMT, FAST>(f[4], f[5], f[6], f[7]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack4<FMT, FAST>(f[0], f[1], f[2], f[3]);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Max over the whole CTA; every thread gets the result.
__device__ __forceinline__ float block_max(float v, float* sh) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) sh[w] = v;
  __syncthreads();
  float r = (l < kThreads / 32) ? sh[l] : 0.0f;
  return warp_max(r);
}

// m = fmax / amax, with m = 1 for amax == 0 or a non-finite quotient.
__device__ __forceinline__ float multiplier(float amax, float fmax) {
  if (!(amax > 0.0f)) return 1.0f;
  const float m = __fdiv_rn(fmax, amax);
  return (m <= FLT_MAX) ? m : 1.0f;
}

// ---------------------------------------------------------------- per-token
// TMA-staged path.  Persistent CTAs walk groups of R consecutive rows (one
// bulk copy per group: the rows are contiguous); S stages are in flight.
// Within a stage each row is owned by 8/R warps (a "team").
constexpr int kHeld = 4;  // vectors per thread kept in registers between the passes

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads, 4) k_token_tma(
    const void* __restrict__ x, int64_t rows, int64_t cols, int R, int S, uint8_t* __restrict__ q,
    float* __restrict__ scales, float* __restrict__ amax_out, unsigned* err) {
  constexpr int VEC = Dt<DT>::kVec;
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kMaxStages];
  __shared__ float red[kThreads / 32];
  __shared__ int rednf[kThreads / 32];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_bytes = cols * Dt<DT>::kSize;
  const int64_t stage_bytes = static_cast<int64_t>(R) * row_bytes;
  const int64_t ngroups = (rows + R - 1) / R;
  const int wpr = (kThreads / 32) / R;  // warps per row
  const int team = warp / wpr;
  const int tt = threadIdx.x - team * wpr * 32;
  const int team_threads = wpr * 32;
  const int64_t nv = cols / VEC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) ptx::mbar_init(&full[s], 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();

  // Thread 0 tracks which stages have a copy in flight (for the abort drain).
  uint32_t pend_mask = 0, pend_parity = 0;
  auto issue = [&](int64_t g, int s, uint32_t parity) {
    const int64_t r0 = g * R;
    const int64_t nr = min(static_cast<int64_t>(R), rows - r0);
    const uint32_t bytes = static_cast<uint32_t>(nr * row_bytes);
    ptx::mbar_arrive_expect_tx(&full[s], bytes);
    ptx::bulk_load(stage_mem + s * stage_bytes, static_cast<const char*>(x) + r0 * row_bytes, bytes, &full[s]);
    pend_mask |= 1u << s;
    pend_parity = (pend_parity & ~(1u << s)) | (parity << s);
  };
  if (threadIdx.x == 0)
    for (int s = 0; s < S; ++s) {
      const int64_t g = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
      if (g < ngroups) issue(g, s, 0);
    }

  int64_t i = 0;
  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x, ++i) {
    const int s = static_cast<int>(i % S);
    const uint32_t parity = static_cast<uint32_t>((i / S) & 1);
    // One thread waits on the stage's barrier (spinning warps would take
    // issue slots from the working ones); the others park at __syncthreads.
    if (threadIdx.x == 0) {
      if (ptx::mbar_wait(&full[s], parity, &abort_flag, err, kDevErrTimeout)) pend_mask &= ~(1u << s);
    }
    __syncthreads();
    if (abort_flag) break;
    const int64_t row = g * R + team;
    const bool valid = row < rows;
    const uint4* src = reinterpret_cast<const uint4*>(stage_mem + s * stage_bytes + team * row_bytes);
    // the first kHeld vectors of this thread stay in registers for the cast
    uint4 held[kHeld];
    uint32_t mraw = 0;
    if (valid) {
#pragma unroll
      for (int k = 0; k < kHeld; ++k) {
        const int64_t v = tt + static_cast<int64_t>(k) * team_threads;
        if (v < nv) {
          held[k] = src[v];
          mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(held[k]));
        }
      }
      for (int64_t v = tt + static_cast<int64_t>(kHeld) * team_threads; v < nv; v += team_threads)
        mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(src[v]));
    }
    const bool nf = Dt<DT>::nonfinite(mraw);
    float amax;
    if (!nf) {
      amax = Dt<DT>::value(mraw);
    } else {  // rare: finite-only maximum on the exact path
      amax = 0.0f;
      for (int64_t v = tt; v < nv; v += team_threads) amax = vec_amax_exact<DT>(src[v], amax);
    }
    amax = warp_max(amax);
    bool row_nf = __any_sync(0xFFFFFFFFu, nf) != 0;
    if (wpr > 1) {  // combine the team's warps through shared memory
      if (lane == 0) {
        red[warp] = amax;
        rednf[warp] = row_nf ? 1 : 0;
      }
      __syncthreads();
      amax = red[team * wpr];
      int any = rednf[team * wpr];
      for (int k = 1; k < wpr; ++k) {
        amax = fmaxf(amax, red[team * wpr + k]);
        any |= rednf[team * wpr + k];
      }
      row_nf = any != 0;
    }
    const float m = multiplier(amax, Fmt<FMT>::kMax);
    if (valid) {
      if (tt == 0) {
        scales[row] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[row] = amax;
      }
      uint8_t* qr = q + row * cols;
      if (!row_nf) {
#pragma unroll
        for (int k = 0; k < kHeld; ++k) {
          const int64_t v = tt + static_cast<int64_t>(k) * team_threads;
          if (v < nv) vec_store<DT, FMT, true>(qr + v * VEC, held[k], m);
        }
        for (int64_t v = tt + static_cast<int64_t>(kHeld) * team_threads; v < nv; v += team_threads)
          vec_store<DT, FMT, true>(qr + v * VEC, src[v], m);
      } else {
        for (int64_t v = tt; v < nv; v += team_threads) vec_store<DT, FMT, false>(qr + v * VEC, src[v], m);
      }
    }
    __syncthreads();  // stage s fully read; red[] free again
    if (threadIdx.x == 0) {
      const int64_t g2 = g + static_cast<int64_t>(S) * gridDim.x;
      if (g2 < ngroups) {
        ptx::fence_proxy_async_smem();
        issue(g2, s, parity ^ 1u);
      }
    }
  }
  if (abort_flag && threadIdx.x == 0) {
    // copies still in flight must land before the CTA's shared memory goes
    int dummy = 0;
    for (int s = 0; s < S; ++s)
      if (pend_mask & (1u << s))
        ptx::mbar_wait(&full[s], (pend_parity >> s) & 1u, &dummy, nullptr, 0, ptx::kDrainLimitNs);
  }
}

// Register-resident path for rows of up to 32 * VPL 16-byte vectors.  A warp
// takes RPW whole rows at a time: lane l loads vectors l, l + 32, ... of each
// row (one warp load instruction covers 512 contiguous bytes) and keeps them
// in registers; the row's raw maximum is reduced by shuffles, and the codes
// are cast from the same registers.  x is read from DRAM exactly once, with
// no shared memory and no block-wide barrier; the persistent warps of other
// rows keep the loads in flight while one warp reduces and casts.
constexpr int kRegThreads = 128;

template <int DT>
__device__ __forceinline__ uint32_t warp_lmax(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = Dt<DT>::lmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

template <int DT, int FMT, int VPL, int RPW>
__global__ void __launch_bounds__(kRegThreads) k_token_reg(const void* __restrict__ x, int64_t rows, int64_t nv,
                                                           uint8_t* __restrict__ q, float* __restrict__ scales,
                                                           float* __restrict__ amax_out) {
  constexpr int VEC = Dt<DT>::kVec;
  pdl_wait();  // launched with programmatic stream serialization
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kRegThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kRegThreads) >> 5;
  const uint4* xv = static_cast<const uint4*>(x);
  for (int64_t r0 = warp0 * RPW; r0 < rows; r0 += nwarps * RPW) {
    uint4 u[RPW][VPL];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int64_t v = lane + 32 * j;
        u[r][j] = (r0 + r < rows && v < nv) ? ld_stream(xv + (r0 + r) * nv + v) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int64_t row = r0 + r;
      if (row >= rows) break;  // warp-uniform
      uint32_t mraw = 0;
#pragma unroll
      for (int j = 0; j < VPL; ++j) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u[r][j]));
      mraw = warp_lmax<DT>(mraw);
      const bool nf = Dt<DT>::nonfinite(mraw);  // the same on every lane
      float amax;
      if (!nf) {
        amax = Dt<DT>::value(mraw);
      } else {  // rare: finite-only maximum on the exact path
        amax = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) amax = vec_amax_exact<DT>(u[r][j], amax);
        amax = warp_max(amax);
      }
      const float m = multiplier(amax, Fmt<FMT>::kMax);
      if (lane == 0) {
        scales[row] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[row] = amax;
      }
      uint8_t* qr = q + row * nv * VEC;
      if (!nf) {
#pragma unroll
        for (int j = 0; j < VPL; ++j)
          if (lane + 32 * j < nv) vec_store<DT, FMT, true>(qr + (lane + 32 * j) * VEC, u[r][j], m);
      } else {
#pragma unroll
        for (int j = 0; j < VPL; ++j)
          if (lane + 32 * j < nv) vec_store<DT, FMT, false>(qr + (lane + 32 * j) * VEC, u[r][j], m);
      }
    }
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
    q[row * cols + c] = cvt1_exact<FMT>(__fmul_rn(Dt<DT>::load1(x, row * cols + c), m));
}

// --------------------------------------------------------------- per-tensor
// Workspace words: [0] amax bits, [1] CTA counter, [2] the multiplier m
// published by phase 1 for phase 2, [3] "a non-finite element was seen".
// All four are zero between calls.

// This thread's share of a flat amax: vectors gtid, gtid + stride, ... then
// the scalar tail.  *nf reports a non-finite element.
template <int DT, bool VECP>
__device__ __forceinline__ float flat_amax(const void* x, int64_t n, bool* nf) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  float amax = 0.0f;
  int64_t done = 0;
  *nf = false;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    uint32_t mraw = 0;
    int64_t v = gtid;
    for (; v + (kUnrollFlat - 1) * gstride < nv; v += kUnrollFlat * gstride) {
      uint4 u[kUnrollFlat];
#pragma unroll
      for (int j = 0; j < kUnrollFlat; ++j) u[j] = __ldg(xv + v + j * gstride);
#pragma unroll
      for (int j = 0; j < kUnrollFlat; ++j) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u[j]));
    }
    for (; v < nv; v += gstride) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(__ldg(xv + v)));
    if (!Dt<DT>::nonfinite(mraw)) {
      amax = Dt<DT>::value(mraw);
    } else {  // rare: redo this thread's vectors on the exact path
      *nf = true;
      for (v = gtid; v < nv; v += gstride) amax = vec_amax_exact<DT>(__ldg(xv + v), amax);
    }
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) {
    const float f = Dt<DT>::load1(x, i);
    if (!(fabsf(f) <= FLT_MAX)) *nf = true;
    amax = fmaxf(amax, finite_abs(f));
  }
  return amax;
}

template <int DT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_tensor_amax(
    const void* __restrict__ x, int64_t n, uint32_t* __restrict__ ws, float fmax,
    float* __restrict__ scales, float* __restrict__ amax_out) {
  __shared__ float sh[kThreads / 32];
  __shared__ bool is_last;
  bool nf;
  float amax = flat_amax<DT, VECP>(x, n, &nf);
  if (__syncthreads_or(nf) && threadIdx.x == 0) atomicOr(&ws[3], 1u);
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
template <int DT, int FMT, bool VECP, bool FAST>
__device__ __forceinline__ void flat_cast(const void* x, int64_t n, float m, uint8_t* q) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t done = 0;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    int64_t i = gtid;
    for (; i + (kUnrollFlat - 1) * gstride < nv; i += kUnrollFlat * gstride) {
      uint4 u[kUnrollFlat];
#pragma unroll
      for (int j = 0; j < kUnrollFlat; ++j) u[j] = ld_stream(xv + (nv - 1 - (i + j * gstride)));
#pragma unroll
      for (int j = 0; j < kUnrollFlat; ++j) vec_store<DT, FMT, FAST>(q + (nv - 1 - (i + j * gstride)) * VEC, u[j], m);
    }
    for (; i < nv; i += gstride) {
      const int64_t v = nv - 1 - i;
      vec_store<DT, FMT, FAST>(q + v * VEC, ld_stream(xv + v), m);
    }
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) q[i] = cvt1_exact<FMT>(__fmul_rn(Dt<DT>::load1(x, i), m));
}

template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_tensor_cast(
    const void* __restrict__ x, int64_t n, uint32_t* __restrict__ ws, uint8_t* __restrict__ q) {
  __shared__ bool is_last;
  const float m = __uint_as_float(__ldcg(&ws[2]));
  const bool any_nf = __ldcg(&ws[3]) != 0u;
  if (!any_nf) flat_cast<DT, FMT, VECP, true>(x, n, m, q);
  else flat_cast<DT, FMT, VECP, false>(x, n, m, q);
  // Every CTA has read m and the flag: the last one returns them to zero.
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&ws[1], 1u) == gridDim.x - 1;
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    atomicExch(&ws[2], 0u);
    atomicExch(&ws[3], 0u);
    atomicExch(&ws[1], 0u);
  }
}

// ------------------------------------------------- per-tensor, one launch
// The same two phases in one cooperative launch (all CTAs resident, one per
// SM).  CTA b owns the contiguous vectors [b0, b1).  Phase 1 keeps the first
// part of its range on chip -- up to 208 KB bulk-copied into shared memory,
// then 256 KB parked in tensor memory (TMEM, tcgen05.st) -- and streams the
// rest through registers with an L2 evict_last hint, so that phase 2 finds it
// in L2.  A grid barrier (a counter, bounded wait) publishes the global amax;
// phase 2 casts the L2 part again, newest lines first, then the TMEM and
// shared-memory parts.  DRAM sees x about once.  Workspace words: [0] amax
// bits, [1] arrivals, [2] departures, [3] non-finite flag; the last CTA to
// leave returns all four to zero.
constexpr int kFusedThreads = 1024;
constexpr int kFusedUnroll = 4;  // 16-byte loads in flight per thread (64 registers at 1024 threads)

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint4* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          ptx::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(ptx::smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Arrival at the grid barrier by one thread after a CTA-wide barrier: the
// release fence orders every write the CTA made before it (the maxima
// folded in with relaxed atomics) ahead of the arrival.
__device__ __forceinline__ void grid_arrive(uint32_t* arrivals) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(arrivals) : "memory");
}
// Departure counter: returns the count before this CTA's increment, with
// acquire-release order (the last CTA sees every other CTA's earlier reads
// of the workspace as done before it clears it).
__device__ __forceinline__ uint32_t grid_depart(uint32_t* departures) {
  uint32_t v;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(v) : "l"(departures) : "memory");
  return v;
}
__device__ __forceinline__ bool grid_barrier(uint32_t* arrivals, unsigned* err_word) {
  const unsigned long long t0 = ptx::globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_u32(arrivals) >= gridDim.x) return true;
    if ((it & 15u) == 15u && ptx::globaltimer() - t0 > ptx::kWaitLimitNs) {
      atomicOr(err_word, kDevErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
}

// Tensor memory as a staging store: each warp owns 64 of the 512 columns of
// its 32-lane quadrant; vector j of a thread sits in columns 4j..4j+3 of its
// lane.  kTmemVecs vectors per thread (256 KB per CTA).
constexpr int kTmemVecs = 16;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ void tmem_alloc_warp(uint32_t* slot) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ptx::smem_u32(slot)),
               "r"(kTmemCols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_warp(uint32_t base) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(kTmemCols) : "memory");
}
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// this thread's column base in its warp's quadrant
__device__ __forceinline__ uint32_t tmem_thread_base(uint32_t base) {
  const uint32_t w = threadIdx.x >> 5;
  return base + ((32u * (w & 3u)) << 16) + (w >> 2) * (4u * kTmemVecs);
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint4& u) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(u.x), "r"(u.y),
               "r"(u.z), "r"(u.w)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint4 tmem_ld4(uint32_t taddr) {
  uint4 u;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
      : "r"(taddr)
      : "memory");
  return u;
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kFusedThreads, 1) k_tensor_fused(
    const void* __restrict__ x, int64_t n, int64_t per_cta, int64_t held_max, uint8_t* __restrict__ q,
    uint32_t* __restrict__ ws, float fmax, float* __restrict__ scales, float* __restrict__ amax_out,
    unsigned* __restrict__ err_word) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int T = kFusedThreads;
  constexpr int U = kFusedUnroll;
  extern __shared__ __align__(128) uint4 held[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ float sh[T / 32];
  __shared__ float s_amax;
  __shared__ int s_flags;  // bit 0: a non-finite element somewhere, bit 1: abort
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;

  const int tid = threadIdx.x;
  const uint4* xv = static_cast<const uint4*>(x);
  const int64_t nv = n / VEC;
  const int64_t b0 = min(nv, static_cast<int64_t>(blockIdx.x) * per_cta);
  const int64_t b1 = min(nv, b0 + per_cta);
  const int64_t nheld = min(b1 - b0, held_max);
  const int64_t s0 = b0 + nheld;                               // TMEM part [s0, s1)
  const int64_t s1 = min(b1, s0 + static_cast<int64_t>(kTmemVecs) * T);  // L2 part [s1, b1)
  const bool tail_cta = blockIdx.x == gridDim.x - 1;
  pdl_wait();  // launched with programmatic stream serialization
  pdl_launch_dependents();

  if (tid == 0) {
    abort_flag = 0;
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbarrier_init();
    if (nheld > 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t bytes = static_cast<uint32_t>(nheld * 16);
      ptx::mbar_arrive_expect_tx(&bar, bytes);
      for (uint32_t off = 0; off < bytes; off += 65536u)
        bulk_load_hint(reinterpret_cast<char*>(held) + off, reinterpret_cast<const char*>(xv + b0) + off,
                       min(65536u, bytes - off), &bar, pol);
    }
  }
  if (tid < 32) tmem_alloc_warp(&tmem_slot);
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tq = tmem_thread_base(tmem_slot);

  // ---- phase 1: amax
  const uint64_t keep = policy_evict_last();
  const uint64_t once = policy_evict_first();
  uint32_t mraw = 0;
#pragma unroll
  for (int j0 = 0; j0 < kTmemVecs; j0 += U) {  // the TMEM part: read once from DRAM
    uint4 u[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t v = s0 + static_cast<int64_t>(j0 + j) * T + tid;
      u[j] = (v < s1) ? ld_hint(xv + v, once) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();  // tcgen05.st is warp-wide
#pragma unroll
    for (int j = 0; j < U; ++j) {
      mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u[j]));
      tmem_st4(tq + 4u * (j0 + j), u[j]);
    }
  }
  int64_t v = s1 + tid;
  for (; v + (U - 1) * T < b1; v += U * T) {
    uint4 u[U];
#pragma unroll
    for (int j = 0; j < U; ++j) u[j] = ld_hint(xv + v + j * T, keep);
#pragma unroll
    for (int j = 0; j < U; ++j) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u[j]));
  }
  for (; v < b1; v += T) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(ld_hint(xv + v, keep)));
  bool landed = true;
  if (nheld > 0) {
    landed = ptx::mbar_wait(&bar, 0, &abort_flag, err_word, kDevErrTimeout);
    if (landed)
      for (int64_t i = tid; i < nheld; i += T) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(held[i]));
  }
  tmem_wait_st();
  float amax = 0.0f;
  bool nf = false;
  if (!Dt<DT>::nonfinite(mraw)) {
    amax = Dt<DT>::value(mraw);
  } else {  // rare: this thread's vectors again on the exact path
    nf = true;
    for (v = s0 + tid; v < b1; v += T) amax = vec_amax_exact<DT>(__ldg(xv + v), amax);
    if (landed)
      for (int64_t i = tid; i < nheld; i += T) amax = vec_amax_exact<DT>(held[i], amax);
  }
  if (tail_cta)
    for (int64_t i = nv * VEC + tid; i < n; i += T) {
      const float f = Dt<DT>::load1(x, i);
      if (!(fabsf(f) <= FLT_MAX)) nf = true;
      amax = fmaxf(amax, finite_abs(f));
    }
  nf = __syncthreads_or(nf);
  amax = warp_max(amax);
  if ((tid & 31) == 0) sh[tid >> 5] = amax;
  __syncthreads();
  if (tid < 32) {
    float r = (tid < T / 32) ? sh[tid] : 0.0f;
    r = warp_max(r);
    if (tid == 0) {
      if (nf) atomicOr(&ws[3], 1u);
      atomicMax(&ws[0], __float_as_uint(r));
      grid_arrive(&ws[1]);
      // grid barrier: every CTA has published its amax
      const bool ok = !abort_flag && grid_barrier(&ws[1], err_word);
      s_amax = __uint_as_float(__ldcg(&ws[0]));
      s_flags = (__ldcg(&ws[3]) != 0u ? 1 : 0) | (ok ? 0 : 2);
    }
  }
  __syncthreads();

  if (!(s_flags & 2)) {
    // ---- phase 2: cast
    const float a = s_amax;
    const float m = multiplier(a, fmax);
    if (blockIdx.x == 0 && tid == 0) {
      scales[0] = __fdiv_rn(1.0f, m);
      if (amax_out) amax_out[0] = a;
    }
    const uint64_t drop = policy_evict_first();
    const int64_t ns = b1 - s1;
    auto cast_range = [&](auto fast) {
      constexpr bool FAST = decltype(fast)::value;
      int64_t i = tid;
      for (; i + (U - 1) * T < ns; i += U * T) {  // the L2 part, from its end backwards
        uint4 u[U];
#pragma unroll
        for (int j = 0; j < U; ++j) u[j] = ld_hint(xv + (b1 - 1 - (i + j * T)), drop);
#pragma unroll
        for (int j = 0; j < U; ++j) vec_store<DT, FMT, FAST>(q + (b1 - 1 - (i + j * T)) * VEC, u[j], m);
      }
      for (; i < ns; i += T) vec_store<DT, FMT, FAST>(q + (b1 - 1 - i) * VEC, ld_hint(xv + (b1 - 1 - i), drop), m);
      __syncwarp();  // tcgen05.ld is warp-wide
#pragma unroll 4
      for (int j = 0; j < kTmemVecs; ++j) {  // the TMEM part
        const uint4 u = tmem_ld4(tq + 4u * j);
        const int64_t vv = s0 + static_cast<int64_t>(j) * T + tid;
        if (vv < s1) vec_store<DT, FMT, FAST>(q + vv * VEC, u, m);
      }
      for (int64_t k = tid; k < nheld; k += T) vec_store<DT, FMT, FAST>(q + (b0 + k) * VEC, held[k], m);
    };
    if (!(s_flags & 1)) cast_range(std::true_type{});
    else cast_range(std::false_type{});
    if (tail_cta)
      for (int64_t i = nv * VEC + tid; i < n; i += T) q[i] = cvt1_exact<FMT>(__fmul_rn(Dt<DT>::load1(x, i), m));
  } else if (tid == 0 && nheld > 0 && !landed) {  // gave up: let the copy land before shared memory goes
    int dummy = 0;
    ptx::mbar_wait(&bar, 0, &dummy, nullptr, 0, ptx::kDrainLimitNs);
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  // departure, off the critical path: the last CTA to leave clears the
  // workspace (every CTA read it right after the barrier)
  if (tid == 0 && grid_depart(&ws[2]) == gridDim.x - 1) {
    atomicExch(&ws[0], 0u);
    atomicExch(&ws[3], 0u);
    atomicExch(&ws[1], 0u);
    atomicExch(&ws[2], 0u);
  }
  __syncwarp();
  if (tid < 32) tmem_dealloc_warp(tmem_slot);
}

// -------------------------------------------------------------- per-channel
// Tile: a strip of 32 column vectors (32*VEC columns) x a band of rows.  Warp
// w of the CTA takes rows w, w+8, ... of the band, eight rows per step; lane
// l owns column vector strip*32 + l.  Workspace: [0] counter, [1] the
// non-finite flag, then amax bits[cols] (from word 4), then m[cols].
template <int DT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_channel_amax(
    const void* __restrict__ x, int64_t rows, int64_t cols, int64_t band_rows,
    uint32_t* __restrict__ header, uint32_t* __restrict__ ws_amax, float* __restrict__ ws_m,
    float fmax, float* __restrict__ scales, float* __restrict__ amax_out) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  constexpr int W = kThreads / 32;
  __shared__ float sh[W][32 * VEC];
  __shared__ bool is_last;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t nvc = cols / VEC;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + l;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * band_rows;
  const int64_t r1 = min(rows, r0 + band_rows);
  float am[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) am[j] = 0.0f;
  bool nf = false;
  if (cv < nvc) {
    if constexpr (VECP) {
      const char* base = static_cast<const char*>(x) + cv * VEC * Dt<DT>::kSize;
      const int64_t rstride = cols * Dt<DT>::kSize;
      uint32_t acc[4] = {0, 0, 0, 0};  // lane-wise raw maxima of the thread's columns
      int64_t r = r0 + w;
      for (; r + (kRowUnroll - 1) * W < r1; r += kRowUnroll * W) {
        uint4 u[kRowUnroll];
#pragma unroll
        for (int j = 0; j < kRowUnroll; ++j)
          u[j] = __ldg(reinterpret_cast<const uint4*>(base + (r + j * W) * rstride));
#pragma unroll
        for (int j = 0; j < kRowUnroll; ++j) {
          acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u[j].x));
          acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u[j].y));
          acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u[j].z));
          acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u[j].w));
        }
      }
      for (; r < r1; r += W) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + r * rstride));
        acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u.x));
        acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u.y));
        acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u.z));
        acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u.w));
      }
      nf = Dt<DT>::nonfinite(Dt<DT>::lmax(Dt<DT>::lmax(acc[0], acc[1]), Dt<DT>::lmax(acc[2], acc[3])));
      if (!nf) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int ln = 0; ln < Dt<DT>::kLanes; ++ln) am[k * Dt<DT>::kLanes + ln] = Dt<DT>::lane_value(acc[k], ln);
      } else {  // rare: exact finite-only maxima
        for (r = r0 + w; r < r1; r += W) {
          float f[Dt<DT>::kVec];
          Dt<DT>::unpack(__ldg(reinterpret_cast<const uint4*>(base + r * rstride)), f);
#pragma unroll
          for (int j = 0; j < VEC; ++j) am[j] = fmaxf(am[j], finite_abs(f[j]));
        }
      }
    } else {
      for (int64_t r = r0 + w; r < r1; r += W) {
        const float f = Dt<DT>::load1(x, r * cols + cv);
        if (!(fabsf(f) <= FLT_MAX)) nf = true;
        am[0] = fmaxf(am[0], finite_abs(f));
      }
    }
  }
  if (__syncthreads_or(nf) && threadIdx.x == 0) atomicOr(&header[1], 1u);
#pragma unroll
  for (int j = 0; j < VEC; ++j) sh[w][l * VEC + j] = am[j];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * VEC; c += kThreads) {
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 32 * VEC + c;
    if (col < cols) {
      float a = sh[0][c];
#pragma unroll
      for (int ww = 1; ww < W; ++ww) a = fmaxf(a, sh[ww][c]);
      atomicMax(&ws_amax[col], __float_as_uint(a));
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&header[0], 1u) == gridDim.x * gridDim.y - 1;
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
    if (threadIdx.x == 0) atomicExch(&header[0], 0u);
  }
}

template <int DT, int FMT, bool VECP, bool FAST>
__device__ __forceinline__ void channel_cast_band(const void* x, int64_t cols, int64_t r0, int64_t r1,
                                                  int64_t cv, const float* ws_m, uint8_t* q) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  constexpr int W = kThreads / 32;
  const int w = threadIdx.x >> 5;
  const int64_t nrows = r1 - r0;
  if constexpr (VECP) {
    float m[Dt<DT>::kVec];
#pragma unroll
    for (int j = 0; j < Dt<DT>::kVec; ++j) m[j] = __ldcg(&ws_m[cv * VEC + j]);
    const char* base = static_cast<const char*>(x) + cv * VEC * Dt<DT>::kSize;
    const int64_t rstride = cols * Dt<DT>::kSize;
    int64_t i = w;
    for (; i + (kRowUnroll - 1) * W < nrows; i += kRowUnroll * W) {  // rows from the band's end backwards
      uint4 u[kRowUnroll];
#pragma unroll
      for (int j = 0; j < kRowUnroll; ++j)
        u[j] = ld_stream(reinterpret_cast<const uint4*>(base + (r1 - 1 - i - j * W) * rstride));
#pragma unroll
      for (int j = 0; j < kRowUnroll; ++j)
        vec_store_m<DT, FMT, FAST>(q + (r1 - 1 - i - j * W) * cols + cv * VEC, u[j], m);
    }
    for (; i < nrows; i += W) {
      const int64_t r = r1 - 1 - i;
      vec_store_m<DT, FMT, FAST>(q + r * cols + cv * VEC,
                                 ld_stream(reinterpret_cast<const uint4*>(base + r * rstride)), m);
    }
  } else {
    const float m0 = __ldcg(&ws_m[cv]);
    for (int64_t i = w; i < nrows; i += W) {
      const int64_t r = r1 - 1 - i;
      q[r * cols + cv] = cvt1_exact<FMT>(__fmul_rn(Dt<DT>::load1(x, r * cols + cv), m0));
    }
  }
}

template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_channel_cast(
    const void* __restrict__ x, int64_t rows, int64_t cols, int64_t band_rows,
    uint32_t* __restrict__ header, float* __restrict__ ws_m, uint8_t* __restrict__ q) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ bool is_last;
  const int l = threadIdx.x & 31;
  const int64_t nvc = cols / VEC;
  const int64_t cv = static_cast<int64_t>(blockIdx.x) * 32 + l;
  const bool any_nf = __ldcg(&header[1]) != 0u;
  if (cv < nvc) {
    // bands in reverse launch order: the last band read by phase 1 goes first
    const int64_t band = static_cast<int64_t>(gridDim.y) - 1 - blockIdx.y;
    const int64_t r0 = band * band_rows;
    const int64_t r1 = min(rows, r0 + band_rows);
    if (!any_nf) channel_cast_band<DT, FMT, VECP, true>(x, cols, r0, r1, cv, ws_m, q);
    else channel_cast_band<DT, FMT, VECP, false>(x, cols, r0, r1, cv, ws_m, q);
  }
  // Every CTA has read its multipliers: the last one zeroes them, the flag
  // and the counter, so the whole workspace is zero again when the call ends.
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&header[0], 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (is_last) {
    for (int64_t c = threadIdx.x; c < cols; c += kThreads) ws_m[c] = 0.0f;
    __syncthreads();
    if (threadIdx.x == 0) {
      atomicExch(&header[1], 0u);
      atomicExch(&header[0], 0u);
    }
  }
}

// ------------------------------------------------ per-channel, one launch
// Cooperative, one CTA per SM.  The matrix is cut into S column strips of
// kStripVecs 16-byte column vectors and B row bands (S * B <= SMs); CTA
// (strip, band) owns that tile.  Thread t owns column vector t % kStripVecs
// of the strip and rows t / kStripVecs, + kRowLanes, ... of the band.  The
// band's first rows of the strip are bulk-copied into shared memory and kept,
// each lane's next kTmemVecs rows are parked in tensor memory, and the rest
// stream through registers with an L2 evict_last hint.  The row
// lanes' maxima meet in shared memory and one atomicMax per column per CTA
// folds them into the workspace, B atomics per column.  After a grid barrier
// each CTA derives its strip's multipliers into shared memory and casts its
// tile: streamed rows again (newest first, evict_first), then held rows.
// Workspace: header [0] arrivals, [1] non-finite flag, [2] departures;
// amax bits[cols].  The last CTA to leave returns them to zero.
constexpr int kStripVecs = 256;
constexpr int kRowLanes = kFusedThreads / kStripVecs;
constexpr int64_t kMaxHeldRows = 128;  // bulk copies per CTA (one per held row)

template <int DT, int FMT>
__global__ void __launch_bounds__(kFusedThreads, 1) k_channel_fused(
    const void* __restrict__ x, int64_t rows, int64_t cols, int strips, int64_t band_rows, int64_t held_rows,
    uint8_t* __restrict__ q, uint32_t* __restrict__ header, uint32_t* __restrict__ ws_amax, float fmax,
    float* __restrict__ scales, float* __restrict__ amax_out, unsigned* __restrict__ err_word) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int T = kFusedThreads;
  constexpr int U = kFusedUnroll;
  constexpr int RL = kRowLanes;
  constexpr int SC = kStripVecs * VEC;  // columns per strip
  extern __shared__ __align__(128) uint8_t fsm[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_flags;  // bit 0: non-finite somewhere, bit 1: give up, bit 2: last to leave
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;

  const int tid = threadIdx.x;
  const int lv = tid % kStripVecs;  // column vector within the strip
  const int rl = tid / kStripVecs;  // row lane
  const int64_t nvc = cols / VEC;
  const int strip = static_cast<int>(blockIdx.x % strips);
  const int64_t band = blockIdx.x / strips;
  const int64_t c0 = static_cast<int64_t>(strip) * kStripVecs;
  const int64_t sv = min(static_cast<int64_t>(kStripVecs), nvc - c0);  // vectors in this strip
  const int64_t r0 = min(rows, band * band_rows);
  const int64_t r1 = min(rows, r0 + band_rows);
  const int64_t nh = min(r1 - r0, held_rows);
  const int64_t rs0 = r0 + nh;                 // rows [rs0, rs1) go through TMEM,
  const int64_t rs1 = rs0 + kTmemVecs * RL;    // rows [rs1, r1) through L2
  float* red = reinterpret_cast<float*>(fsm);  // [RL][SC] row-lane maxima; later the strip's multipliers
  uint4* held = reinterpret_cast<uint4*>(fsm + RL * SC * 4);  // [nh][sv]
  const uint4* xv = static_cast<const uint4*>(x);  // row r, column vector c: xv[r * nvc + c]
  pdl_wait();  // launched with programmatic stream serialization
  pdl_launch_dependents();

  if (tid < 32) {  // warp 0: the held rows' bulk copies, one per row, spread over the lanes
    if (tid == 0) {
      abort_flag = 0;
      ptx::mbar_init(&bar, 1);
      ptx::fence_mbarrier_init();
      if (nh > 0 && sv > 0) ptx::mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nh * sv * 16));
    }
    __syncwarp();
    if (nh > 0 && sv > 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t row_bytes = static_cast<uint32_t>(sv * 16);
      for (int64_t i = tid; i < nh; i += 32) bulk_load_hint(held + i * sv, xv + (r0 + i) * nvc + c0, row_bytes, &bar, pol);
    }
  }
  if (tid < 32) tmem_alloc_warp(&tmem_slot);
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tq = tmem_thread_base(tmem_slot);

  // ---- phase 1: column maxima of the tile
  const uint64_t keep = policy_evict_last();
  const uint64_t once = policy_evict_first();
  const bool active = lv < sv;
  const int64_t c = c0 + lv;
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i0 = 0; i0 < kTmemVecs; i0 += U) {  // this lane's first rows: read once, parked in TMEM
    uint4 u[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t r = rs0 + rl + static_cast<int64_t>(i0 + j) * RL;
      u[j] = (active && r < r1) ? ld_hint(xv + r * nvc + c, once) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();  // tcgen05.st is warp-wide
#pragma unroll
    for (int j = 0; j < U; ++j) {
      acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u[j].x));
      acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u[j].y));
      acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u[j].z));
      acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u[j].w));
      tmem_st4(tq + 4u * (i0 + j), u[j]);
    }
  }
  if (active) {
    int64_t r = rs1 + rl;
    for (; r + (U - 1) * RL < r1; r += U * RL) {
      uint4 u[U];
#pragma unroll
      for (int j = 0; j < U; ++j) u[j] = ld_hint(xv + (r + j * RL) * nvc + c, keep);
#pragma unroll
      for (int j = 0; j < U; ++j) {
        acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u[j].x));
        acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u[j].y));
        acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u[j].z));
        acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u[j].w));
      }
    }
    for (; r < r1; r += RL) {
      const uint4 u = ld_hint(xv + r * nvc + c, keep);
      acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u.x));
      acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u.y));
      acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u.z));
      acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u.w));
    }
  }
  tmem_wait_st();
  bool landed = true;
  if (nh > 0 && sv > 0) landed = ptx::mbar_wait(&bar, 0, &abort_flag, err_word, kDevErrTimeout);
  if (active && landed)
    for (int64_t i = rl; i < nh; i += RL) {
      const uint4 u = held[i * sv + lv];
      acc[0] = Dt<DT>::lmax(acc[0], Dt<DT>::mag(u.x));
      acc[1] = Dt<DT>::lmax(acc[1], Dt<DT>::mag(u.y));
      acc[2] = Dt<DT>::lmax(acc[2], Dt<DT>::mag(u.z));
      acc[3] = Dt<DT>::lmax(acc[3], Dt<DT>::mag(u.w));
    }
  float am[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) am[j] = 0.0f;
  bool nf = false;
  if (active) {
    if (!Dt<DT>::nonfinite(Dt<DT>::lmax(Dt<DT>::lmax(acc[0], acc[1]), Dt<DT>::lmax(acc[2], acc[3])))) {
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int ln = 0; ln < Dt<DT>::kLanes; ++ln) am[w * Dt<DT>::kLanes + ln] = Dt<DT>::lane_value(acc[w], ln);
    } else {  // rare: finite-only maxima of this lane's rows on the exact path
      nf = true;
      for (int64_t r = r0 + rl; r < r1; r += RL) {
        float f[VEC];
        Dt<DT>::unpack((r < rs0 && landed) ? held[(r - r0) * sv + lv] : __ldg(xv + r * nvc + c), f);
#pragma unroll
        for (int j = 0; j < VEC; ++j) am[j] = fmaxf(am[j], finite_abs(f[j]));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < VEC; ++j) red[rl * SC + lv * VEC + j] = am[j];
  nf = __syncthreads_or(nf);
  for (int64_t e = tid; e < sv * VEC; e += T) {  // one atomicMax per column of the strip
    float a = red[e];
#pragma unroll
    for (int l = 1; l < RL; ++l) a = fmaxf(a, red[l * SC + e]);
    atomicMax(&ws_amax[c0 * VEC + e], __float_as_uint(a));
  }
  __syncthreads();
  if (tid == 0) {
    if (nf) atomicOr(&header[1], 1u);
    grid_arrive(&header[0]);
    const bool ok = !abort_flag && grid_barrier(&header[0], err_word);
    s_flags = (__ldcg(&header[1]) != 0u ? 1 : 0) | (ok ? 0 : 2);
  }
  __syncthreads();
  const bool ok = !(s_flags & 2);
  // the strip's multipliers; the CTAs of band 0 publish the scales
  float* m_s = red;
  if (ok)
    for (int64_t e = tid; e < sv * VEC; e += T) {
      const int64_t col = c0 * VEC + e;
      const float a = __uint_as_float(__ldcg(&ws_amax[col]));
      const float m = multiplier(a, fmax);
      m_s[e] = m;
      if (band == 0) {
        scales[col] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[col] = a;
      }
    }
  __syncthreads();
  if (ok) {
    // ---- phase 2: cast the tile: this lane's L2 rows from the end backwards,
    // then its TMEM rows, then the held rows
    const uint64_t drop = policy_evict_first();
    float m[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) m[j] = active ? m_s[lv * VEC + j] : 0.0f;
    auto cast_tile = [&](auto fast) {
      constexpr bool FAST = decltype(fast)::value;
      if (active && r1 - 1 >= rs1 + rl) {
        int64_t r = rs1 + rl + ((r1 - 1 - rs1 - rl) / RL) * RL;  // this lane's last L2 row
        for (; r - (U - 1) * RL >= rs1; r -= U * RL) {
          uint4 u[U];
#pragma unroll
          for (int j = 0; j < U; ++j) u[j] = ld_hint(xv + (r - j * RL) * nvc + c, drop);
#pragma unroll
          for (int j = 0; j < U; ++j) vec_store_m<DT, FMT, FAST>(q + (r - j * RL) * cols + c * VEC, u[j], m);
        }
        for (; r >= rs1; r -= RL)
          vec_store_m<DT, FMT, FAST>(q + r * cols + c * VEC, ld_hint(xv + r * nvc + c, drop), m);
      }
      __syncwarp();  // tcgen05.ld is warp-wide
#pragma unroll 4
      for (int i = 0; i < kTmemVecs; ++i) {
        const uint4 u = tmem_ld4(tq + 4u * i);
        const int64_t r = rs0 + rl + static_cast<int64_t>(i) * RL;
        if (active && r < r1) vec_store_m<DT, FMT, FAST>(q + r * cols + c * VEC, u, m);
      }
      if (active)
        for (int64_t i = rl; i < nh; i += RL)
          vec_store_m<DT, FMT, FAST>(q + (r0 + i) * cols + c * VEC, held[i * sv + lv], m);
    };
    if (!(s_flags & 1)) cast_tile(std::true_type{});
    else cast_tile(std::false_type{});
  } else if (tid == 0 && nh > 0 && sv > 0 && !landed) {  // gave up: let the copy land before shared memory goes
    int dummy = 0;
    ptx::mbar_wait(&bar, 0, &dummy, nullptr, 0, ptx::kDrainLimitNs);
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  // departure, off the critical path: the last CTA to leave clears the
  // maxima and the header (every CTA read them right after the barrier)
  if (tid == 0) s_flags = (grid_depart(&header[2]) == gridDim.x - 1) ? 4 : 0;
  __syncthreads();
  if (s_flags & 4) {
    for (int64_t col = tid; col < cols; col += T) ws_amax[col] = 0u;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      atomicExch(&header[1], 0u);
      atomicExch(&header[0], 0u);
      atomicExch(&header[2], 0u);
    }
  }
  if (tid < 32) tmem_dealloc_warp(tmem_slot);
}

// ------------------------------------------------------------------ delayed
// Ring: [hist[len] | scale | counter].  Workspace word [0]: amax accumulator.
// One pass: cast with the ring's multiplier while reducing amax.  A thread
// whose raw maximum shows a non-finite element redoes its vectors on the
// exact path (finite-only amax, canonical NaN codes).  The body runs as CTA
// `cta` of `ncta` CTAs given one tensor (the single launch, or one tensor's
// share of a batched launch); the last of them to finish steps the ring.
// The ring's history is read at the start (only the last CTA writes it, at
// the end), so the last CTA's tail is one acquire-release increment and one
// exchange.
constexpr int kRingPrefetch = 64;  // history words read ahead into shared memory

template <int DT, int FMT, bool VECP>
__device__ __forceinline__ void delayed_body(const void* __restrict__ x, int64_t n, uint8_t* __restrict__ q,
                                             float* __restrict__ ring, int len, int idx, int margin,
                                             uint32_t* __restrict__ ws, float* __restrict__ scales,
                                             float* __restrict__ amax_out, int64_t cta, int64_t ncta) {
  constexpr int VEC = VECP ? Dt<DT>::kVec : 1;
  __shared__ float sh[kThreads / 32];
  __shared__ bool is_last;
  __shared__ float hist_sh[kRingPrefetch];
  const float m = __ldcg(&ring[len]);
  const bool m_finite = fabsf(m) <= FLT_MAX;
  if (threadIdx.x < kRingPrefetch && static_cast<int>(threadIdx.x) < len) hist_sh[threadIdx.x] = __ldcg(&ring[threadIdx.x]);
  const int64_t gtid = cta * kThreads + threadIdx.x;
  const int64_t gstride = ncta * kThreads;
  float amax = 0.0f;
  int64_t done = 0;
  if (VECP) {
    const uint4* xv = static_cast<const uint4*>(x);
    const int64_t nv = n / VEC;
    uint32_t mraw = 0;
    if (m_finite) {
      int64_t v = gtid;
      for (; v + (kUnroll - 1) * gstride < nv; v += kUnroll * gstride) {
        uint4 u[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) u[j] = ld_stream(xv + v + j * gstride);
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
          mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u[j]));
          vec_store<DT, FMT, true>(q + (v + j * gstride) * VEC, u[j], m);
        }
      }
      for (; v < nv; v += gstride) {
        const uint4 u = ld_stream(xv + v);
        mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(u));
        vec_store<DT, FMT, true>(q + v * VEC, u, m);
      }
    }
    if (m_finite && !Dt<DT>::nonfinite(mraw)) {
      amax = Dt<DT>::value(mraw);
    } else {  // rare: redo this thread's vectors on the exact path
      for (int64_t v = gtid; v < nv; v += gstride) {
        const uint4 u = __ldg(xv + v);
        amax = vec_amax_exact<DT>(u, amax);
        vec_store<DT, FMT, false>(q + v * VEC, u, m);
      }
    }
    done = nv * VEC;
  }
  for (int64_t i = done + gtid; i < n; i += gstride) {
    const float f = Dt<DT>::load1(x, i);
    amax = fmaxf(amax, finite_abs(f));
    q[i] = cvt1_exact<FMT>(__fmul_rn(f, m));
  }
  amax = block_max(amax, sh);
  uint32_t* counter = reinterpret_cast<uint32_t*>(ring + len + 1);
  if (threadIdx.x == 0) {
    atomicMax(&ws[0], __float_as_uint(amax));
    uint32_t prev;  // release: this CTA's maximum is in before the count; acquire for the last CTA
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
    is_last = prev == static_cast<uint32_t>(ncta - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __shared__ float a_sh;
  if (threadIdx.x == 0) a_sh = __uint_as_float(atomicExch(&ws[0], 0u));
  __syncthreads();
  const float a = a_sh;
  // the window: max of the history with this step's slot replaced by a
  float win;
  if (len <= kRingPrefetch) {  // from the history read at the start
    if (threadIdx.x != 0) return;
    win = a;
    for (int i = 0; i < len; ++i)
      if (i != idx) win = fmaxf(win, hist_sh[i]);
  } else {
    float w = (threadIdx.x == 0) ? a : 0.0f;
    for (int i = threadIdx.x; i < len; i += kThreads)
      if (i != idx) w = fmaxf(w, __ldcg(&ring[i]));
    win = block_max(w, sh);
    if (threadIdx.x != 0) return;
  }
  ring[idx] = a;
  if (win <= FLT_MAX && win > 0.0f) {
    const float next = ldexpf(__fdiv_rn(Fmt<FMT>::kMax, win), -margin);
    if (next <= FLT_MAX && next > 0.0f) ring[len] = next;
  }
  scales[0] = __fdiv_rn(1.0f, m);
  if (amax_out) amax_out[0] = a;
  atomicExch(counter, 0u);
}

template <int DT, int FMT, bool VECP>
__global__ void __launch_bounds__(kThreads) k_delayed(
    const void* __restrict__ x, int64_t n, uint8_t* __restrict__ q, float* __restrict__ ring,
    int len, int idx, int margin, uint32_t* __restrict__ ws, float* __restrict__ scales,
    float* __restrict__ amax_out) {
  pdl_wait();  // launched with programmatic stream serialization
  pdl_launch_dependents();
  delayed_body<DT, FMT, VECP>(x, n, q, ring, len, idx, margin, ws, scales, amax_out, blockIdx.x, gridDim.x);
}

// Batched delayed quantize: up to kBatchMax tensors of one dtype and format in
// one launch.  Tensor t owns CTAs [cta0[t], cta0[t + 1]); each tensor's CTAs
// run the single-tensor body with their own ring, workspace and counter.
constexpr int kBatchMax = 8;
struct DelayedBatch {
  int count;
  int cta0[kBatchMax + 1];
  const void* x[kBatchMax];
  int64_t n[kBatchMax];
  uint8_t* q[kBatchMax];
  float* scales[kBatchMax];
  float* amax_out[kBatchMax];
  float* ring[kBatchMax];
  int len[kBatchMax], idx[kBatchMax], margin[kBatchMax];
  uint32_t* ws[kBatchMax];
  int vec[kBatchMax];  // 1: 16-byte vector path
};

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads) k_delayed_batch(const __grid_constant__ DelayedBatch b) {
  pdl_wait();  // launched with programmatic stream serialization
  pdl_launch_dependents();
  int t = 0;
  while (t + 1 < b.count && static_cast<int>(blockIdx.x) >= b.cta0[t + 1]) ++t;
  const int64_t cta = static_cast<int64_t>(blockIdx.x) - b.cta0[t];
  const int64_t ncta = b.cta0[t + 1] - b.cta0[t];
  if (b.vec[t])
    delayed_body<DT, FMT, true>(b.x[t], b.n[t], b.q[t], b.ring[t], b.len[t], b.idx[t], b.margin[t], b.ws[t],
                                b.scales[t], b.amax_out[t], cta, ncta);
  else
    delayed_body<DT, FMT, false>(b.x[t], b.n[t], b.q[t], b.ring[t], b.len[t], b.idx[t], b.margin[t], b.ws[t],
                                 b.scales[t], b.amax_out[t], cta, ncta);
}

// ----------------------------------------- per-tensor with a transposed copy
// For the backward GEMMs (AstrAI ops.cu linear_backward_fp8: dX reads the
// weight codes transposed, dW reads the gradient and activation codes
// transposed) one pass writes the codes of x [R, C] row-major (optional) and
// transposed, qt [C, R].  A CTA walks 64 x 64 tiles: thread t quantizes the
// 16 consecutive elements at tile row t / 4, columns 16 (t % 4) .. + 15,
// stores them to q and to a shared tile; after a barrier it gathers the 16
// codes at tile column t / 4, rows 16 (t % 4) .. + 15, and stores them as one
// 16-byte piece of qt.  Every access of x, q and qt is a 16-byte vector.
// MODE 0: dynamic, the multiplier published by a k_tensor_amax pass in
// ws[2] (the last CTA returns ws[1..3] to zero); 1: delayed, the ring's
// multiplier, the last CTA steps the ring (as k_delayed); 2: a caller's
// multiplier, the ring-free static form (amax reported, nothing stepped).
constexpr int kQtTile = 64;
constexpr int kQtPitch = 68;  // bytes per shared tile row: conflict-light column gathers

template <int FMT>
__device__ __forceinline__ uint32_t codes4(const float* f, float m) {
  return cvt2_exact<FMT>(__fmul_rn(f[0], m), __fmul_rn(f[1], m)) |
         (cvt2_exact<FMT>(__fmul_rn(f[2], m), __fmul_rn(f[3], m)) << 16);
}

template <int DT, int FMT, int MODE>
__global__ void __launch_bounds__(kThreads) k_quant_transpose(
    const void* __restrict__ x, int64_t rows, int64_t cols, uint8_t* __restrict__ q, uint8_t* __restrict__ qt,
    const float* __restrict__ mult, float* __restrict__ ring, int len, int idx, int margin,
    uint32_t* __restrict__ ws, float* __restrict__ scales, float* __restrict__ amax_out) {
  constexpr int VEC = Dt<DT>::kVec;
  __shared__ __align__(16) uint8_t tile[kQtTile * kQtPitch];
  __shared__ float sh[kThreads / 32];
  __shared__ bool is_last;
  float m;
  if (MODE == 0) m = __uint_as_float(__ldcg(&ws[2]));
  else if (MODE == 1) m = __ldcg(&ring[len]);
  else m = __ldg(mult);
  const int64_t ntr = (rows + kQtTile - 1) / kQtTile;
  const int64_t ntc = (cols + kQtTile - 1) / kQtTile;
  const int t = threadIdx.x;
  const int lr = t >> 2, seg = (t & 3) * 16;  // quantize: tile row lr, columns seg .. seg + 15
  float amax = 0.0f;
  for (int64_t ti = blockIdx.x; ti < ntr * ntc; ti += gridDim.x) {
    const int64_t r0 = (ti / ntc) * kQtTile, c0 = (ti % ntc) * kQtTile;
    const int64_t r = r0 + lr, c = c0 + seg;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (r < rows && c < cols) {  // cols % 16 == 0: all 16 elements are inside
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + (r * cols + c) * Dt<DT>::kSize);
#pragma unroll
      for (int v = 0; v < 16 / VEC; ++v) {
        float f[VEC];
        Dt<DT>::unpack(ld_stream(src + v), f);
#pragma unroll
        for (int i = 0; i < VEC; ++i) amax = fmaxf(amax, finite_abs(f[i]));
#pragma unroll
        for (int k = 0; k < VEC / 4; ++k) w[v * (VEC / 4) + k] = codes4<FMT>(f + 4 * k, m);
      }
      if (q != nullptr) *reinterpret_cast<uint4*>(q + r * cols + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    uint32_t* trow = reinterpret_cast<uint32_t*>(tile + lr * kQtPitch + seg);
#pragma unroll
    for (int k = 0; k < 4; ++k) trow[k] = w[k];
    __syncthreads();
    const int jc = t >> 2, rs = (t & 3) * 16;  // gather: tile column jc, rows rs .. rs + 15
    const int64_t qr = c0 + jc, qc = r0 + rs;
    if (qr < cols && qc < rows) {  // rows % 16 == 0
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint8_t* col = tile + (rs + 4 * k) * kQtPitch + jc;
        o[k] = static_cast<uint32_t>(col[0]) | (static_cast<uint32_t>(col[kQtPitch]) << 8) |
               (static_cast<uint32_t>(col[2 * kQtPitch]) << 16) | (static_cast<uint32_t>(col[3 * kQtPitch]) << 24);
      }
      *reinterpret_cast<uint4*>(qt + qr * rows + qc) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
  }
  amax = block_max(amax, sh);
  if (MODE == 0) {  // m and the flag were read by every CTA: the last one clears them
    if (t == 0) is_last = atomicAdd(&ws[1], 1u) == gridDim.x - 1;
    __syncthreads();
    if (is_last && t == 0) {
      atomicExch(&ws[2], 0u);
      atomicExch(&ws[3], 0u);
      atomicExch(&ws[1], 0u);
    }
    return;
  }
  uint32_t* counter = (MODE == 1) ? reinterpret_cast<uint32_t*>(ring + len + 1) : &ws[1];
  if (t == 0) {
    atomicMax(&ws[0], __float_as_uint(amax));
    __threadfence();
    is_last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last || t != 0) return;
  __threadfence();
  const float a = __uint_as_float(atomicExch(&ws[0], 0u));
  if (MODE == 1) {
    ring[idx] = a;  // fold this step's amax into the history slot
    float win = 0.0f;
    for (int i = 0; i < len; ++i) win = fmaxf(win, __ldcg(&ring[i]));
    if (win <= FLT_MAX && win > 0.0f) {
      const float next = ldexpf(__fdiv_rn(Fmt<FMT>::kMax, win), -margin);
      if (next <= FLT_MAX && next > 0.0f) ring[len] = next;
    }
  }
  scales[0] = __fdiv_rn(1.0f, m);
  if (amax_out) amax_out[0] = a;
  atomicExch(counter, 0u);
}

// ---------------------------------------------------- stochastic E5M2
// Stochastic rounding to E5M2 (hip-quant README "Stochastic E5M2 Backward
// Gradients"): between the two adjacent E5M2 values, rounding up with
// probability proportional to the distance from the lower one, from a
// stateless hash of (seed, element index).  The hash is SplitMix64 used as a
// counter-based generator: element i draws the top half of the generator's
// output i + 1 from state `seed`.
__device__ __forceinline__ uint32_t sr_draw(uint64_t seed, uint64_t idx) {
  uint64_t z = seed + (idx + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return static_cast<uint32_t>(z >> 32);
}

// The E5M2 grid value y rounds to: with g the spacing at |y| and
// lo = floor(|y| / g) g, up to lo + g iff u < floor((|y| - lo) / g * 2^32).
// Zero, NaN, +-Inf and |y| >= 57344 come back unchanged (the saturating
// conversion then gives their codes); the sign is kept.
__device__ __forceinline__ float sr_e5m2(float y, uint32_t u) {
  const uint32_t b = __float_as_uint(y);
  const uint32_t a = b & 0x7FFFFFFFu, sgn = b & 0x80000000u;
  if (a == 0u || a >= 0x47600000u) return y;
  uint32_t r;
  if (a >= 0x38800000u) {  // |y| >= 2^-14: g is 2^21 units of the f32 last place
    const uint32_t d = a & 0x1FFFFFu;
    r = (a & ~0x1FFFFFu) + ((u < (d << 11)) ? 0x200000u : 0u);
  } else {  // below 2^-14: g = 2^-16
    const float t = __uint_as_float(a) * 65536.0f;  // exact
    float lo = floorf(t);
    const uint32_t thr = static_cast<uint32_t>((t - lo) * 4294967296.0f);  // exact, < 2^32
    lo += (u < thr) ? 1.0f : 0.0f;
    r = __float_as_uint(lo * 1.52587890625e-05f);  // * 2^-16, exact
  }
  return __uint_as_float(r | sgn);
}

template <int DT>
__device__ __forceinline__ void sr_store_vec(uint8_t* dst, const uint4& u, float m, uint64_t seed, uint64_t idx0) {
  float f[Dt<DT>::kVec];
  Dt<DT>::unpack(u, f);
  uint32_t w[Dt<DT>::kVec / 4];
#pragma unroll
  for (int k = 0; k < Dt<DT>::kVec / 4; ++k) {
    float g[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) g[i] = sr_e5m2(__fmul_rn(f[4 * k + i], m), sr_draw(seed, idx0 + 4 * k + i));
    w[k] = cvt2_exact<1>(g[0], g[1]) | (cvt2_exact<1>(g[2], g[3]) << 16);
  }
  if constexpr (Dt<DT>::kVec == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  else *reinterpret_cast<uint32_t*>(dst) = w[0];
}

// Per-tensor (GRAN 0, m in ws[2] from k_tensor_amax) or per-channel (GRAN 2,
// m[col] in ws_m from k_channel_amax): the stochastic cast of every element;
// the last CTA returns the workspace to zero.
template <int DT, int GRAN>
__global__ void __launch_bounds__(kThreads) k_sr_cast(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                      uint64_t seed, uint8_t* __restrict__ q,
                                                      uint32_t* __restrict__ header, float* __restrict__ ws_m) {
  constexpr int VEC = Dt<DT>::kVec;
  __shared__ bool is_last;
  const int64_t n = rows * cols;
  const int64_t nv = n / VEC;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * kThreads;
  const uint4* xv = static_cast<const uint4*>(x);
  const float mt = (GRAN == 0) ? __uint_as_float(__ldcg(&header[2])) : 0.0f;
  for (int64_t v = gtid; v < nv; v += gstride) {
    if (GRAN == 2) {  // cols % VEC == 0: the vector's columns are c0 .. c0 + VEC - 1
      float mm[VEC];
      const int64_t c0 = (v * VEC) % cols;
#pragma unroll
      for (int i = 0; i < VEC; ++i) mm[i] = __ldcg(&ws_m[c0 + i]);
      float f[VEC];
      Dt<DT>::unpack(ld_stream(xv + v), f);
      uint32_t w[VEC / 4];
#pragma unroll
      for (int k = 0; k < VEC / 4; ++k) {
        float g[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          g[i] = sr_e5m2(__fmul_rn(f[4 * k + i], mm[4 * k + i]), sr_draw(seed, v * VEC + 4 * k + i));
        w[k] = cvt2_exact<1>(g[0], g[1]) | (cvt2_exact<1>(g[2], g[3]) << 16);
      }
      if constexpr (VEC == 8) *reinterpret_cast<uint2*>(q + v * VEC) = make_uint2(w[0], w[1]);
      else *reinterpret_cast<uint32_t*>(q + v * VEC) = w[0];
    } else {
      sr_store_vec<DT>(q + v * VEC, ld_stream(xv + v), mt, seed, static_cast<uint64_t>(v * VEC));
    }
  }
  for (int64_t i = nv * VEC + gtid; i < n; i += gstride) {  // element tail
    const float m = (GRAN == 0) ? mt : __ldcg(&ws_m[i % cols]);
    q[i] = cvt1_exact<1>(sr_e5m2(__fmul_rn(Dt<DT>::load1(x, i), m), sr_draw(seed, static_cast<uint64_t>(i))));
  }
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&header[GRAN == 0 ? 1 : 0], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  if (GRAN == 0) {
    if (threadIdx.x == 0) {
      atomicExch(&header[2], 0u);
      atomicExch(&header[3], 0u);
      atomicExch(&header[1], 0u);
    }
  } else {
    for (int64_t c = threadIdx.x; c < cols; c += kThreads) ws_m[c] = 0.0f;
    __syncthreads();
    if (threadIdx.x == 0) {
      atomicExch(&header[1], 0u);
      atomicExch(&header[0], 0u);
    }
  }
}

// Per-token: one CTA per row; the row's finite amax, m = fmax / amax (as
// the RNE quantize), then the stochastic cast of the row.
template <int DT>
__global__ void __launch_bounds__(kThreads) k_sr_token(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                       uint64_t seed, uint8_t* __restrict__ q,
                                                       float* __restrict__ scales, float* __restrict__ amax_out) {
  __shared__ float sh[kThreads / 32];
  const int64_t r = blockIdx.x;
  const int64_t base = r * cols;
  float amax = 0.0f;
  for (int64_t c = threadIdx.x; c < cols; c += kThreads) amax = fmaxf(amax, finite_abs(Dt<DT>::load1(x, base + c)));
  amax = block_max(amax, sh);
  const float m = multiplier(amax, Fmt<1>::kMax);
  if (threadIdx.x == 0) {
    scales[r] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[r] = amax;
  }
  for (int64_t c = threadIdx.x; c < cols; c += kThreads)
    q[base + c] = cvt1_exact<1>(sr_e5m2(__fmul_rn(Dt<DT>::load1(x, base + c), m),
                                         sr_draw(seed, static_cast<uint64_t>(base + c))));
}

// ---------------------------------------------------------------- block-wise
// Block-wise FP8 (hip-quant README "Block-wise FP8 Scaling"): one f32 dequant
// scale per block of `block` consecutive elements along the last dimension,
// scales [rows, ceil(cols / block)] (the last block of a row may be short).
// One thread per block, consecutive threads on consecutive blocks: the block
// is read with 16-byte loads for its finite amax (raw bits, exact redo when
// a non-finite element shows), then again (from L1) for the cast, rounded
// to nearest even or, SR, stochastically (E5M2).  block % 16 == 0 and
// cols % 16 == 0.
template <int DT, int FMT, bool SR>
__global__ void __launch_bounds__(kThreads) k_block_quant(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                          int64_t block, uint64_t seed, uint8_t* __restrict__ q,
                                                          float* __restrict__ scales, float* __restrict__ amax_out) {
  constexpr int VEC = Dt<DT>::kVec;
  const int64_t nb = (cols + block - 1) / block;
  const int64_t total = rows * nb;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t r = t / nb, b = t - r * nb;
    const int64_t c0 = b * block;
    const int nvec = static_cast<int>((min(cols, c0 + block) - c0) / VEC);
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + (r * cols + c0) * Dt<DT>::kSize);
    uint32_t mraw = 0;
    for (int v = 0; v < nvec; ++v) mraw = Dt<DT>::lmax(mraw, vec_mag<DT>(__ldg(src + v)));
    float amax = 0.0f;
    if (!Dt<DT>::nonfinite(mraw)) {
      amax = Dt<DT>::value(mraw);
    } else {
      for (int v = 0; v < nvec; ++v) amax = vec_amax_exact<DT>(__ldg(src + v), amax);
    }
    const float m = multiplier(amax, Fmt<FMT>::kMax);
    scales[t] = __fdiv_rn(1.0f, m);
    if (amax_out) amax_out[t] = amax;
    uint8_t* dst = q + r * cols + c0;
    for (int v = 0; v < nvec; ++v) {
      const uint4 u = __ldg(src + v);
      if constexpr (SR) sr_store_vec<DT>(dst + v * VEC, u, m, seed, static_cast<uint64_t>(r * cols + c0 + v * VEC));
      else vec_store<DT, FMT, false>(dst + v * VEC, u, m);
    }
  }
}

// Block-wise quantize, warp-cooperative, for power-of-two blocks.  A warp
// takes chunks of UNR units of U = 32 * kVec * NV consecutive elements of one
// row; lane l holds vectors l, l + 32, ... of each unit, so every load
// instruction of the warp reads 512 contiguous bytes.  With NV == 1 a unit
// holds U / block whole blocks, each on block / kVec adjacent lanes (a power
// of two dividing 32) that reduce their raw magnitude by xor shuffles; with
// NV > 1 the unit is one block.  Index arithmetic is one division per chunk;
// within a row it is 32-bit, and the block index is a shift.  The codes equal
// k_block_quant's.
template <int DT, int FMT, bool SR, int NV>
__global__ void __launch_bounds__(kThreads) k_block_quant_warp(const void* __restrict__ x, int64_t rows, int cols,
                                                               int log2_block, uint64_t seed,
                                                               uint8_t* __restrict__ q, float* __restrict__ scales,
                                                               float* __restrict__ amax_out) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int U = 32 * VEC * NV;
  constexpr int UNR = NV == 1 ? 4 : (NV == 2 ? 2 : 1);
  constexpr int CH = U * UNR;
  const int lane = threadIdx.x & 31;
  const int cpr = (cols + CH - 1) / CH;  // chunks per row
  const int64_t chunks = rows * cpr;
  const int nb = ((cols - 1) >> log2_block) + 1;
  const int lpb = NV == 1 ? (1 << log2_block) / VEC : 32;
  const uint4* xv = static_cast<const uint4*>(x);
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const bool narrow = chunks <= 0xFFFFFFFFll;
  for (int64_t ch = warp0; ch < chunks; ch += nwarps) {
    int64_t r;
    int cc;
    if (narrow) {
      const uint32_t c32 = static_cast<uint32_t>(ch), rr = c32 / static_cast<uint32_t>(cpr);
      r = rr;
      cc = static_cast<int>(c32 - rr * static_cast<uint32_t>(cpr)) * CH;
    } else {
      r = ch / cpr;
      cc = static_cast<int>(ch - r * cpr) * CH;
    }
    const int64_t rbase = r * cols;
    uint4 v[UNR][NV];
#pragma unroll
    for (int j = 0; j < UNR; ++j)
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int c = cc + j * U + (k * 32 + lane) * VEC;
        v[j][k] = c < cols ? ld_stream(xv + (rbase + c) / VEC) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
    for (int j = 0; j < UNR; ++j) {
      const int cu = cc + j * U;
      if (cu >= cols) break;  // warp-uniform: the rest of the chunk is past the row
      uint32_t mr = 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) mr = Dt<DT>::lmax(mr, vec_mag<DT>(v[j][k]));
      for (int o = lpb >> 1; o > 0; o >>= 1) mr = Dt<DT>::lmax(mr, __shfl_xor_sync(0xFFFFFFFFu, mr, o));
      const bool special = __any_sync(0xFFFFFFFFu, Dt<DT>::nonfinite(mr));
      float amax;
      if (!special) {
        amax = Dt<DT>::value(mr);
      } else {  // warp-uniform: every lane takes the exact amax of its block
        amax = 0.0f;
#pragma unroll
        for (int k = 0; k < NV; ++k) amax = vec_amax_exact<DT>(v[j][k], amax);
        for (int o = lpb >> 1; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      }
      const float m = multiplier(amax, Fmt<FMT>::kMax);
      const int c0 = cu + lane * VEC;
      if ((lane & (lpb - 1)) == 0 && c0 < cols) {
        const int64_t t = r * nb + (c0 >> log2_block);
        scales[t] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[t] = amax;
      }
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int c = c0 + k * 32 * VEC;
        if (c >= cols) continue;
        if constexpr (SR) sr_store_vec<DT>(q + rbase + c, v[j][k], m, seed, static_cast<uint64_t>(rbase + c));
        else if (!special) vec_store<DT, FMT, true>(q + rbase + c, v[j][k], m);
        else vec_store<DT, FMT, false>(q + rbase + c, v[j][k], m);
      }
    }
  }
}

// Stage pipeline of the block-wise kernels (the per-token one): persistent
// CTAs; S stages of R whole rows, each filled by one 1-D bulk copy while the
// other stages are worked on.  work(stage, r0, nr) runs on every thread once
// rows [r0, r0 + nr) have landed in `stage`; a barrier separates it from the
// refill of that stage.  A stage that does not land within the time limit
// sets the error word and ends the kernel after the copies in flight drain.
template <class Work>
__device__ __forceinline__ void row_stage_pipeline(const void* __restrict__ x, int64_t rows, int64_t row_bytes, int R,
                                                   int S, unsigned* err, Work&& work) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kMaxStages];
  __shared__ int abort_flag;
  const int64_t stage_bytes = static_cast<int64_t>(R) * row_bytes;
  const int64_t ngroups = (rows + R - 1) / R;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) ptx::mbar_init(&full[s], 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  uint32_t pend_mask = 0, pend_parity = 0;  // thread 0: stages with a copy in flight
  auto issue = [&](int64_t g, int s, uint32_t parity) {
    const int64_t r0 = g * R;
    const int64_t nr = min(static_cast<int64_t>(R), rows - r0);
    const uint32_t bytes = static_cast<uint32_t>(nr * row_bytes);
    ptx::mbar_arrive_expect_tx(&full[s], bytes);
    ptx::bulk_load(stage_mem + s * stage_bytes, static_cast<const char*>(x) + r0 * row_bytes, bytes, &full[s]);
    pend_mask |= 1u << s;
    pend_parity = (pend_parity & ~(1u << s)) | (parity << s);
  };
  if (threadIdx.x == 0)
    for (int s = 0; s < S; ++s) {
      const int64_t g = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
      if (g < ngroups) issue(g, s, 0);
    }
  int64_t i = 0;
  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x, ++i) {
    const int s = static_cast<int>(i % S);
    const uint32_t parity = static_cast<uint32_t>((i / S) & 1);
    if (threadIdx.x == 0) {
      if (ptx::mbar_wait(&full[s], parity, &abort_flag, err, kDevErrTimeout)) pend_mask &= ~(1u << s);
    }
    __syncthreads();
    if (abort_flag) break;
    const int64_t r0 = g * R;
    work(stage_mem + s * stage_bytes, r0, static_cast<int>(min(static_cast<int64_t>(R), rows - r0)));
    __syncthreads();  // stage s fully read
    if (threadIdx.x == 0) {
      const int64_t g2 = g + static_cast<int64_t>(S) * gridDim.x;
      if (g2 < ngroups) {
        ptx::fence_proxy_async_smem();
        issue(g2, s, parity ^ 1u);
      }
    }
  }
  if (abort_flag && threadIdx.x == 0) {
    int dummy = 0;
    for (int s = 0; s < S; ++s)
      if (pend_mask & (1u << s))
        ptx::mbar_wait(&full[s], (pend_parity >> s) & 1u, &dummy, nullptr, 0, ptx::kDrainLimitNs);
  }
}

// Block-wise, staged, blocks of at least one warp-wide vector span (NV = block
// / (32 kVec) vectors per lane): a warp reduces one block per unit with xor
// shuffles over all 32 lanes.  A stage's units go to the warps round-robin.
template <int DT, int FMT, bool SR, int NV>
__global__ void __launch_bounds__(kThreads, 1) k_block_tma(
    const void* __restrict__ x, int64_t rows, int cols, int log2_block, int R, int S, uint64_t seed,
    uint8_t* __restrict__ q, float* __restrict__ scales, float* __restrict__ amax_out, unsigned* err) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int U = 32 * VEC * NV;
  constexpr int kWarps = kThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int upr = (cols + U - 1) / U;
  const int nb = ((cols - 1) >> log2_block) + 1;
  row_stage_pipeline(x, rows, static_cast<int64_t>(cols) * Dt<DT>::kSize, R, S, err,
                     [&](const uint8_t* stage, int64_t r0, int nr) {
    const uint4* st = reinterpret_cast<const uint4*>(stage);
    const int units = nr * upr;
    int rl = 0, uu = warp;  // this warp's unit: row rl of the stage, unit uu of the row
    while (uu >= upr) { uu -= upr; ++rl; }
    for (int u = warp; u < units; u += kWarps) {  // warp-uniform bounds
      const int cu = uu * U;
      uint4 v[NV];
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int c = cu + (k * 32 + lane) * VEC;
        v[k] = c < cols ? st[(rl * cols + c) / VEC] : make_uint4(0u, 0u, 0u, 0u);
      }
      uint32_t mr = 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) mr = Dt<DT>::lmax(mr, vec_mag<DT>(v[k]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mr = Dt<DT>::lmax(mr, __shfl_xor_sync(0xFFFFFFFFu, mr, o));
      const bool special = Dt<DT>::nonfinite(mr);  // uniform: mr is the whole block's
      float amax;
      if (!special) {
        amax = Dt<DT>::value(mr);
      } else {
        amax = 0.0f;
#pragma unroll
        for (int k = 0; k < NV; ++k) amax = vec_amax_exact<DT>(v[k], amax);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      }
      const float m = multiplier(amax, Fmt<FMT>::kMax);
      const int64_t row = r0 + rl;
      if (lane == 0) {
        const int64_t t = row * nb + (cu >> log2_block);
        scales[t] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[t] = amax;
      }
      const int64_t rbase = row * cols;
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int c = cu + (k * 32 + lane) * VEC;
        if (c >= cols) continue;
        if constexpr (SR) sr_store_vec<DT>(q + rbase + c, v[k], m, seed, static_cast<uint64_t>(rbase + c));
        else if (!special) vec_store<DT, FMT, true>(q + rbase + c, v[k], m);
        else vec_store<DT, FMT, false>(q + rbase + c, v[k], m);
      }
      uu += kWarps;
      while (uu >= upr) { uu -= upr; ++rl; }
    }
  });
}

// Block-wise, staged, blocks narrower than a warp-wide vector span (2 .. 16
// vectors of kVec elements).  A warp task is 32 consecutive blocks of a row:
// pass 1, lane l alone reduces block l (its vectors visited from a lane-
// rotated start, so that the strided shared-memory reads do not pile onto the
// same banks), takes the block's multiplier and dequant scale (one division
// each for 32 blocks at once) and writes the scales coalesced; pass 2 casts
// the task's vectors in coalesced order, each fetching its block's multiplier
// from the owning lane by a shuffle (negated when the block holds a
// non-finite element, which selects the exact cast).  The codes equal
// k_block_quant's.
template <int DT, int FMT, bool SR>
__global__ void __launch_bounds__(kThreads, 1) k_block_tma_narrow(
    const void* __restrict__ x, int64_t rows, int cols, int log2_block, int R, int S, uint64_t seed,
    uint8_t* __restrict__ q, float* __restrict__ scales, float* __restrict__ amax_out, unsigned* err) {
  constexpr int VEC = Dt<DT>::kVec;
  constexpr int kLog2Vec = VEC == 8 ? 3 : 2;
  constexpr int kWarps = kThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int log2_bpv = log2_block - kLog2Vec;  // vectors per block: 1 << log2_bpv
  const int bpv = 1 << log2_bpv;
  const int vpr = cols / VEC;                   // vectors per row (cols % 16 == 0)
  const int nb = ((cols - 1) >> log2_block) + 1;
  const int ntask = (nb + 31) >> 5;             // tasks per row
  row_stage_pipeline(x, rows, static_cast<int64_t>(cols) * Dt<DT>::kSize, R, S, err,
                     [&](const uint8_t* stage, int64_t r0, int nr) {
    const uint4* st = reinterpret_cast<const uint4*>(stage);
    const int tasks = nr * ntask;
    int rl = 0, tk = warp;
    while (tk >= ntask) { tk -= ntask; ++rl; }
    for (int t = warp; t < tasks; t += kWarps) {  // warp-uniform bounds
      const int64_t row = r0 + rl;
      const uint4* rs = st + rl * vpr;
      const int v0 = (tk * 32) << log2_bpv;      // the task's first vector in the row
      // pass 1: block b = tk * 32 + lane, vectors [vb, vb + bpv) of the row
      const int b = tk * 32 + lane;
      const int vb = v0 + (lane << log2_bpv);
      float ms = 1.0f;
      if (b < nb) {
        const int nvalid = min(bpv, vpr - vb);
        uint32_t mr = 0;
        for (int i = 0; i < bpv; ++i) {
          const int j = (i + lane) & (bpv - 1);
          if (j < nvalid) mr = Dt<DT>::lmax(mr, vec_mag<DT>(rs[vb + j]));
        }
        const bool special = Dt<DT>::nonfinite(mr);
        float amax;
        if (!special) {
          amax = Dt<DT>::value(mr);
        } else {
          amax = 0.0f;
          for (int j = 0; j < nvalid; ++j) amax = vec_amax_exact<DT>(rs[vb + j], amax);
        }
        const float m = multiplier(amax, Fmt<FMT>::kMax);
        const int64_t ti = row * nb + b;
        scales[ti] = __fdiv_rn(1.0f, m);
        if (amax_out) amax_out[ti] = amax;
        ms = special ? -m : m;
      }
      // pass 2: the task's vectors, lane-contiguous
      const int64_t rbase = row * cols;
      for (int i = 0; i < bpv; ++i) {
        const int vl = lane + 32 * i;            // vector within the task
        const float mv = __shfl_sync(0xFFFFFFFFu, ms, vl >> log2_bpv);
        const int v = v0 + vl;
        if (v < vpr) {
          const uint4 u = rs[v];
          uint8_t* dst = q + rbase + static_cast<int64_t>(v) * VEC;
          if constexpr (SR) sr_store_vec<DT>(dst, u, fabsf(mv), seed, static_cast<uint64_t>(rbase + v * VEC));
          else if (mv > 0.0f) vec_store<DT, FMT, true>(dst, u, mv);
          else vec_store<DT, FMT, false>(dst, u, -mv);
        }
      }
      tk += kWarps;
      while (tk >= ntask) { tk -= ntask; ++rl; }
    }
  });
}

// Block-wise dequantize: out = f32(dec(q) * block scale), or that rounded to
// bf16.  The codes decode exactly through cvt to f16 pairs.
template <int FMT, bool BF16_OUT>
__device__ __forceinline__ void dequant16(const uint4& u, float sc, void* __restrict__ out, int64_t e0) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float f[16];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const unsigned short pair = static_cast<unsigned short>(w[k] >> (16 * h));
      uint32_t hh;
      if (FMT == 0) asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"(pair));
      else asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(hh) : "h"(pair));
      f[4 * k + 2 * h] = __half2float(__ushort_as_half(static_cast<unsigned short>(hh & 0xFFFFu)));
      f[4 * k + 2 * h + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(hh >> 16)));
    }
#pragma unroll
  for (int i = 0; i < 16; ++i) f[i] = __fmul_rn(f[i], sc);
  if constexpr (BF16_OUT) {
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      o[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * i]))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * i + 1]))) << 16);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + e0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  } else {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
  }
}

// One thread per 16 codes (cols % 16 == 0 and block % 16 == 0: the 16 share a
// row and a block); kDequantUnroll groups are loaded before any is written.
constexpr int kDequantUnroll = 4;
template <int FMT, bool BF16_OUT>
__global__ void __launch_bounds__(kThreads) k_block_dequant(const uint8_t* __restrict__ q, int64_t rows, int64_t cols,
                                                            int64_t block, const float* __restrict__ scales,
                                                            void* __restrict__ out) {
  const int64_t nb = (cols + block - 1) / block;
  const int64_t n16 = rows * cols / 16;
  const int64_t gs = static_cast<int64_t>(gridDim.x) * kThreads;
  const uint4* qv = reinterpret_cast<const uint4*>(q);
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; t0 < n16;
       t0 += gs * kDequantUnroll) {
    uint4 u[kDequantUnroll];
    float sc[kDequantUnroll];
#pragma unroll
    for (int j = 0; j < kDequantUnroll; ++j) {
      const int64_t t = t0 + j * gs;
      if (t < n16) {
        const int64_t r = (t * 16) / cols, c = t * 16 - r * cols;
        u[j] = ld_stream(qv + t);
        sc[j] = __ldg(scales + r * nb + c / block);
      }
    }
#pragma unroll
    for (int j = 0; j < kDequantUnroll; ++j) {
      const int64_t t = t0 + j * gs;
      if (t < n16) dequant16<FMT, BF16_OUT>(u[j], sc[j], out, t * 16);
    }
  }
}

// ------------------------------------------------------------------- launch
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int flat_grid(int64_t nvec, int dev, int unroll) {
  const int64_t per_cta = static_cast<int64_t>(kThreads) * unroll;
  int64_t g = (nvec + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(device_sm_count(dev)) * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// Per-tensor in one cooperative launch: one CTA per SM, each holding up to
// kFusedHeldBytes of its range in shared memory.
constexpr int64_t kFusedHeldBytes = 208 * 1024;
constexpr int64_t kFusedMinBytes = 4 << 20;  // smaller tensors: the two-launch path

template <int DT, int FMT>
cudaError_t launch_tensor_fused(const QuantizeArgs& a, int dev, int64_t n, float fmax) {
  constexpr int VEC = Dt<DT>::kVec;
  static cudaError_t attr = cudaFuncSetAttribute(k_tensor_fused<DT, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kFusedHeldBytes));
  if (attr != cudaSuccess) return attr;
  const int grid = device_sm_count(dev);
  const int64_t nv = n / VEC;
  int64_t per = (nv + grid - 1) / grid;
  int64_t held_max = std::min<int64_t>(per, kFusedHeldBytes / 16);
  const size_t smem = static_cast<size_t>(held_max) * 16;
  const void* x = a.x;
  uint8_t* q = a.q;
  uint32_t* ws = static_cast<uint32_t*>(a.ws);
  float* scales = a.scales;
  float* amax_out = a.amax_out;
  unsigned* err = device_error_word();
  return launch_pdl(k_tensor_fused<DT, FMT>, dim3(grid), dim3(kFusedThreads), smem, a.stream, true, x, n, per,
                    held_max, q, ws, fmax, scales, amax_out, err);
}

// Per-token rows of up to 1024 vectors: the register-resident kernel on a
// persistent grid of as many resident CTAs as its registers allow.
template <int DT, int FMT, int VPL, int RPW>
cudaError_t launch_token_reg(const QuantizeArgs& a, int dev, int64_t nv) {
  static int per_sm = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_token_reg<DT, FMT, VPL, RPW>, kRegThreads, 0) !=
        cudaSuccess) {
      cudaGetLastError();
      per_sm = 0;
    }
  });
  const int64_t warps_needed = (a.rows + RPW - 1) / RPW;
  const int64_t ctas_needed = (warps_needed + kRegThreads / 32 - 1) / (kRegThreads / 32);
  int64_t grid = static_cast<int64_t>(device_sm_count(dev)) * std::max(per_sm, 1);
  if (grid > ctas_needed) grid = ctas_needed;
  if (grid < 1) grid = 1;
  return launch_pdl(k_token_reg<DT, FMT, VPL, RPW>, dim3(static_cast<unsigned>(grid)), dim3(kRegThreads), 0,
                    a.stream, false, a.x, a.rows, nv, a.q, a.scales, a.amax_out);
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
    const int grid = flat_grid(flat_vec ? n / VEC : n, dev, kUnroll);
    if (flat_vec)
      return launch_pdl(k_delayed<DT, FMT, true>, dim3(grid), dim3(kThreads), 0, a.stream, false, a.x, n, a.q, a.ring,
                        a.ring_len, a.ring_idx, a.ring_margin, ws, a.scales, a.amax_out);
    return launch_pdl(k_delayed<DT, FMT, false>, dim3(grid), dim3(kThreads), 0, a.stream, false, a.x, n, a.q, a.ring,
                      a.ring_len, a.ring_idx, a.ring_margin, ws, a.scales, a.amax_out);
  }

  if (a.gran == 1) {  // per-token
    if (row_vec && a.cols > 0 && a.cols / VEC <= 32 * 32) {
      const int64_t nv = a.cols / VEC;
      if (nv <= 32) return launch_token_reg<DT, FMT, 1, 16>(a, dev, nv);
      if (nv <= 64) return launch_token_reg<DT, FMT, 2, 8>(a, dev, nv);
      if (nv <= 128) return launch_token_reg<DT, FMT, 4, 4>(a, dev, nv);
      if (nv <= 256) return launch_token_reg<DT, FMT, 8, 2>(a, dev, nv);
      if (nv <= 512) return launch_token_reg<DT, FMT, 16, 1>(a, dev, nv);
      return launch_token_reg<DT, FMT, 32, 1>(a, dev, nv);
    }
    if (row_vec && a.cols > 0) {
      // Stages of at least 32 KB (whole rows), two per CTA, as many CTAs per
      // SM as shared memory and registers allow (a sweep over stage size,
      // depth and CTAs per SM on the workload shapes picked this rule).
      const int64_t row_bytes = a.cols * Dt<DT>::kSize;
      int R = 1;
      while (R < 8 && R * row_bytes < 32768) R *= 2;
      const int64_t stage_bytes = R * row_bytes;
      const int S = 2;
      if (S * stage_bytes <= 220 * 1024) {
        const int smem = static_cast<int>(S * stage_bytes);
        static cudaError_t attr = cudaFuncSetAttribute(k_token_tma<DT, FMT>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
        if (attr != cudaSuccess) return attr;
        const int64_t ngroups = (a.rows + R - 1) / R;
        int per_sm = static_cast<int>(std::min<int64_t>(4, (227 * 1024) / (smem + 1024)));
        if (per_sm < 1) per_sm = 1;
        int64_t grid = static_cast<int64_t>(device_sm_count(dev)) * per_sm;
        if (grid > ngroups) grid = ngroups;
        k_token_tma<DT, FMT><<<static_cast<unsigned>(grid), kThreads, smem, a.stream>>>(
            a.x, a.rows, a.cols, R, S, a.q, a.scales, a.amax_out, device_error_word());
        return cudaGetLastError();
      }
    }
    k_token_generic<DT, FMT><<<static_cast<unsigned>(a.rows), kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q,
                                                                                        a.scales, a.amax_out);
    return cudaGetLastError();
  }

  if (a.gran == 0 && flat_vec && n * Dt<DT>::kSize >= kFusedMinBytes && device_error_word() != nullptr)
    return launch_tensor_fused<DT, FMT>(a, dev, n, fmax);
  if (a.gran == 0) {  // per-tensor, two phases
    uint32_t* ws = static_cast<uint32_t*>(a.ws);
    const int grid = flat_grid(flat_vec ? n / VEC : n, dev, kUnrollFlat);
    if (flat_vec)
      k_tensor_amax<DT, true><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, fmax, a.scales, a.amax_out);
    else
      k_tensor_amax<DT, false><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, fmax, a.scales, a.amax_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (n == 0)  // nothing to cast: clear the published multiplier and flag
      return cudaMemsetAsync(ws + 2, 0, 2 * sizeof(uint32_t), a.stream);
    if (flat_vec)
      k_tensor_cast<DT, FMT, true><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, a.q);
    else
      k_tensor_cast<DT, FMT, false><<<grid, kThreads, 0, a.stream>>>(a.x, n, ws, a.q);
    return cudaGetLastError();
  }

  if (row_vec && n * Dt<DT>::kSize >= kFusedMinBytes && device_error_word() != nullptr) {
    const int sms = device_sm_count(dev);
    const int64_t nvc = a.cols / VEC;
    const int64_t strips = (nvc + kStripVecs - 1) / kStripVecs;
    if (strips <= sms) {
      static cudaError_t attr = cudaFuncSetAttribute(k_channel_fused<DT, FMT>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(kFusedHeldBytes));
      if (attr != cudaSuccess) return attr;
      int64_t bands = std::max<int64_t>(1, std::min<int64_t>(sms / strips, a.rows));
      int64_t band = (a.rows + bands - 1) / bands;
      bands = (a.rows + band - 1) / band;
      const int64_t fixed = static_cast<int64_t>(kRowLanes) * kStripVecs * VEC * 4;
      const int64_t strip_bytes = std::min<int64_t>(nvc, kStripVecs) * 16;
      int64_t held = std::min<int64_t>({band, (kFusedHeldBytes - fixed) / strip_bytes, kMaxHeldRows});
      const size_t smem = static_cast<size_t>(fixed + held * strip_bytes);
      uint32_t* header = static_cast<uint32_t*>(a.ws);
      uint32_t* ws_amax = header + 4;
      const void* x = a.x;
      int64_t rows = a.rows, cols = a.cols;
      int nstrips = static_cast<int>(strips);
      uint8_t* q = a.q;
      float f = fmax;
      float* scales = a.scales;
      float* amax_out = a.amax_out;
      unsigned* err = device_error_word();
      return launch_pdl(k_channel_fused<DT, FMT>, dim3(static_cast<unsigned>(strips * bands)), dim3(kFusedThreads),
                        smem, a.stream, true, x, rows, cols, nstrips, band, held, q, header, ws_amax, f, scales,
                        amax_out, err);
    }
  }

  // per-channel, two phases
  const int vec = row_vec ? VEC : 1;
  const int64_t nvc = a.cols / vec;
  const int64_t strips = (nvc + 31) / 32;
  const int64_t target = static_cast<int64_t>(device_sm_count(dev)) * 8;
  int64_t bands = (target + strips - 1) / strips;
  if (bands > a.rows) bands = a.rows;
  if (bands < 1) bands = 1;
  if (bands > 65535) bands = 65535;
  const int64_t band_rows = a.rows > 0 ? (a.rows + bands - 1) / bands : 1;
  bands = a.rows > 0 ? (a.rows + band_rows - 1) / band_rows : 1;
  if (strips > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(bands));
  uint32_t* header = static_cast<uint32_t*>(a.ws);
  uint32_t* ws_amax = header + 4;
  float* ws_m = reinterpret_cast<float*>(ws_amax + ((a.cols + 3) / 4) * 4);
  if (row_vec)
    k_channel_amax<DT, true><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, header, ws_amax,
                                                              ws_m, fmax, a.scales, a.amax_out);
  else
    k_channel_amax<DT, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, header, ws_amax,
                                                               ws_m, fmax, a.scales, a.amax_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (n == 0) {  // nothing to cast: clear the published multipliers and flag
    e = cudaMemsetAsync(header + 1, 0, sizeof(uint32_t), a.stream);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(ws_m, 0, static_cast<size_t>(a.cols) * sizeof(float), a.stream);
  }
  if (row_vec)
    k_channel_cast<DT, FMT, true><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, header, ws_m,
                                                                   a.q);
  else
    k_channel_cast<DT, FMT, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, header, ws_m,
                                                                    a.q);
  return cudaGetLastError();
}

template <int DT, int FMT>
cudaError_t launch_transpose_typed(const QuantizeArgs& a) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t n = a.rows * a.cols;
  const float fmax = Fmt<FMT>::kMax;
  uint32_t* ws = static_cast<uint32_t*>(a.ws);
  const int64_t tiles = ((a.rows + kQtTile - 1) / kQtTile) * ((a.cols + kQtTile - 1) / kQtTile);
  int64_t grid = std::min<int64_t>(tiles, static_cast<int64_t>(device_sm_count(dev)) * 8);
  if (grid < 1) grid = 1;
  const unsigned g = static_cast<unsigned>(grid);
  if (a.ring) {
    k_quant_transpose<DT, FMT, 1><<<g, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q, a.qt, nullptr, a.ring,
                                                                 a.ring_len, a.ring_idx, a.ring_margin, ws, a.scales,
                                                                 a.amax_out);
    return cudaGetLastError();
  }
  if (a.mult) {
    k_quant_transpose<DT, FMT, 2><<<g, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q, a.qt, a.mult, nullptr, 0,
                                                                 0, 0, ws, a.scales, a.amax_out);
    return cudaGetLastError();
  }
  // dynamic: the per-tensor amax pass publishes m, then the transposing cast
  const int agrid = flat_grid(n / Dt<DT>::kVec, dev, kUnrollFlat);
  k_tensor_amax<DT, true><<<agrid, kThreads, 0, a.stream>>>(a.x, n, ws, fmax, a.scales, a.amax_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (n == 0) return cudaMemsetAsync(ws + 2, 0, 2 * sizeof(uint32_t), a.stream);
  k_quant_transpose<DT, FMT, 0><<<g, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.q, a.qt, nullptr, nullptr, 0, 0,
                                                               0, ws, a.scales, a.amax_out);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_sr_typed(const QuantizeArgs& a) {
  constexpr int VEC = Dt<DT>::kVec;
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t n = a.rows * a.cols;
  const float fmax = Fmt<1>::kMax;
  if (a.gran == 1) {
    if (a.rows == 0) return cudaSuccess;
    k_sr_token<DT><<<static_cast<unsigned>(a.rows), kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.seed, a.q,
                                                                             a.scales, a.amax_out);
    return cudaGetLastError();
  }
  const int grid = flat_grid(n / VEC, dev, 1);
  if (a.gran == 0) {
    uint32_t* ws = static_cast<uint32_t*>(a.ws);
    k_tensor_amax<DT, true><<<flat_grid(n / VEC, dev, kUnrollFlat), kThreads, 0, a.stream>>>(a.x, n, ws, fmax,
                                                                                           a.scales, a.amax_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (n == 0) return cudaMemsetAsync(ws + 2, 0, 2 * sizeof(uint32_t), a.stream);
    k_sr_cast<DT, 0><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.seed, a.q, ws, nullptr);
    return cudaGetLastError();
  }
  // per-channel: the two-launch column amax, then the stochastic cast
  const int64_t nvc = a.cols / VEC;
  const int64_t strips = (nvc + 31) / 32;
  const int64_t target = static_cast<int64_t>(device_sm_count(dev)) * 8;
  int64_t bands = std::max<int64_t>(1, std::min<int64_t>({(target + strips - 1) / std::max<int64_t>(strips, 1),
                                                          a.rows, 65535}));
  const int64_t band_rows = a.rows > 0 ? (a.rows + bands - 1) / bands : 1;
  bands = a.rows > 0 ? (a.rows + band_rows - 1) / band_rows : 1;
  uint32_t* header = static_cast<uint32_t*>(a.ws);
  uint32_t* ws_amax = header + 4;
  float* ws_m = reinterpret_cast<float*>(ws_amax + ((a.cols + 3) / 4) * 4);
  const dim3 cgrid(static_cast<unsigned>(std::max<int64_t>(strips, 1)), static_cast<unsigned>(bands));
  k_channel_amax<DT, true><<<cgrid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, band_rows, header, ws_amax, ws_m,
                                                              fmax, a.scales, a.amax_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (n == 0) {
    e = cudaMemsetAsync(header + 1, 0, sizeof(uint32_t), a.stream);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(ws_m, 0, static_cast<size_t>(a.cols) * sizeof(float), a.stream);
  }
  k_sr_cast<DT, 2><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, a.seed, a.q, header, ws_m);
  return cudaGetLastError();
}

// Staged block-wise launch: two stages of R whole rows, R doubled (up to 8)
// until a stage holds at least 32 KB and four warp tasks, while the stage
// pair stays within kBlockStageMax; as many CTAs per SM as shared memory
// allows (at most 3).  A sweep over the rule on [8192|16384, 8192] and
// [4096, 28672] bf16 with blocks of 16 .. 128 picked it: asking for a task per
// warp doubles the stage at blocks of 128, leaving one CTA per SM and 20-35 %
// less bandwidth.  Returns cudaErrorNotSupported when one row pair does
// not fit.  NV = 0 selects the narrow-block kernel.
constexpr int64_t kBlockStageMax = 200 * 1024;
template <int DT, int NV>
cudaError_t launch_block_tma(const QuantizeArgs& a, int log2_block, bool sr, int dev) {
  constexpr int VEC = Dt<DT>::kVec;
  const int64_t row_bytes = a.cols * Dt<DT>::kSize;
  const int S = 2;
  unsigned* err = device_error_word();
  if (S * row_bytes > kBlockStageMax || err == nullptr) return cudaErrorNotSupported;
  const int64_t nb = (a.cols + (int64_t{1} << log2_block) - 1) >> log2_block;
  const int64_t tasks_per_row = NV == 0 ? (nb + 31) / 32 : (a.cols + 32 * VEC * NV - 1) / (32 * VEC * NV);
  int R = 1;
  while (R < 8 && (R * row_bytes < 32768 || R * tasks_per_row < 4) &&
         S * 2 * R * row_bytes <= kBlockStageMax)
    R *= 2;
  const int smem = static_cast<int>(S * R * row_bytes);
  void (*kern)(const void*, int64_t, int, int, int, int, uint64_t, uint8_t*, float*, float*, unsigned*);
  if constexpr (NV == 0)
    kern = sr ? k_block_tma_narrow<DT, 1, true>
              : (a.fmt == 0 ? k_block_tma_narrow<DT, 0, false> : k_block_tma_narrow<DT, 1, false>);
  else
    kern = sr ? k_block_tma<DT, 1, true, NV>
              : (a.fmt == 0 ? k_block_tma<DT, 0, false, NV> : k_block_tma<DT, 1, false, NV>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kBlockStageMax));
  if (e != cudaSuccess) return e;
  const int64_t ngroups = (a.rows + R - 1) / R;
  int per_sm = static_cast<int>(std::min<int64_t>(3, (227 * 1024) / (smem + 1024)));
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(device_sm_count(dev)) * per_sm;
  if (grid > ngroups) grid = ngroups;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, a.stream>>>(a.x, a.rows, static_cast<int>(a.cols), log2_block,
                                                                   R, S, sr ? a.seed : 0, a.q, a.scales, a.amax_out,
                                                                   err);
  return cudaGetLastError();
}

template <int DT, int NV>
cudaError_t launch_block_warp(const QuantizeArgs& a, int64_t block, bool sr, int dev) {
  constexpr int64_t CH = 32 * Dt<DT>::kVec * NV * (NV == 1 ? 4 : (NV == 2 ? 2 : 1));
  const int64_t warps = a.rows * ((a.cols + CH - 1) / CH);  // one chunk per warp and pass
  const int64_t g = (warps + kThreads / 32 - 1) / (kThreads / 32);
  int log2_block = 0;
  while ((int64_t{1} << log2_block) < block) ++log2_block;
  auto kern = sr ? k_block_quant_warp<DT, 1, true, NV>
                 : (a.fmt == 0 ? k_block_quant_warp<DT, 0, false, NV> : k_block_quant_warp<DT, 1, false, NV>);
  // one resident wave: the warps stride over the units
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0);
  if (e != cudaSuccess) return e;
  const int64_t cap = static_cast<int64_t>(device_sm_count(dev)) * (per_sm > 0 ? per_sm : 1);
  const int grid = static_cast<int>(g < 1 ? 1 : (g > cap ? cap : g));
  kern<<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, static_cast<int>(a.cols), log2_block, sr ? a.seed : 0, a.q,
                                        a.scales, a.amax_out);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_block_typed(const QuantizeArgs& a, int64_t block, bool sr) {
  int dev = 0;
  cudaGetDevice(&dev);
  // Power-of-two blocks of up to four warp-wide vector spans (W elements)
  // take the staged kernels when a stage pair of rows fits; otherwise, and
  // for eight spans, the unstaged warp-cooperative kernel; any other block
  // (a multiple of 16) one thread per block.
  constexpr int64_t W = 32 * Dt<DT>::kVec;
  const bool pow2 = (block & (block - 1)) == 0;
  int log2_block = 0;
  while ((int64_t{1} << log2_block) < block) ++log2_block;
  // rows that fit a stage pair go through the bulk-copy pipeline
  if (pow2 && block <= 4 * W && a.rows > 0) {
    cudaError_t e = block < W        ? launch_block_tma<DT, 0>(a, log2_block, sr, dev)
                    : block == W     ? launch_block_tma<DT, 1>(a, log2_block, sr, dev)
                    : block == 2 * W ? launch_block_tma<DT, 2>(a, log2_block, sr, dev)
                                     : launch_block_tma<DT, 4>(a, log2_block, sr, dev);
    if (e != cudaErrorNotSupported) return e;
  }
  if (pow2 && block <= W) return launch_block_warp<DT, 1>(a, block, sr, dev);
  if (pow2 && block == 2 * W) return launch_block_warp<DT, 2>(a, block, sr, dev);
  if (pow2 && block == 4 * W) return launch_block_warp<DT, 4>(a, block, sr, dev);
  if (pow2 && block == 8 * W) return launch_block_warp<DT, 8>(a, block, sr, dev);
  const int64_t nb = (a.cols + block - 1) / block;
  const int grid = flat_grid(a.rows * nb, dev, 1);
  if (sr)
    k_block_quant<DT, 1, true><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, block, a.seed, a.q, a.scales,
                                                                 a.amax_out);
  else if (a.fmt == 0)
    k_block_quant<DT, 0, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, block, 0, a.q, a.scales,
                                                                  a.amax_out);
  else
    k_block_quant<DT, 1, false><<<grid, kThreads, 0, a.stream>>>(a.x, a.rows, a.cols, block, 0, a.q, a.scales,
                                                                  a.amax_out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_blockwise(const QuantizeArgs& a, int64_t block, bool stochastic) {
  switch (a.xt) {
    case 0: return launch_block_typed<0>(a, block, stochastic);
    case 1: return launch_block_typed<1>(a, block, stochastic);
    case 2: return launch_block_typed<2>(a, block, stochastic);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dequantize_blockwise(const uint8_t* q, int fmt, int64_t rows, int64_t cols, int64_t block,
                                        const float* scales, bool bf16_out, void* out, cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int grid = flat_grid(rows * cols / 16, dev, kDequantUnroll);
  if (fmt == 0 && bf16_out) k_block_dequant<0, true><<<grid, kThreads, 0, stream>>>(q, rows, cols, block, scales, out);
  else if (fmt == 0) k_block_dequant<0, false><<<grid, kThreads, 0, stream>>>(q, rows, cols, block, scales, out);
  else if (bf16_out) k_block_dequant<1, true><<<grid, kThreads, 0, stream>>>(q, rows, cols, block, scales, out);
  else k_block_dequant<1, false><<<grid, kThreads, 0, stream>>>(q, rows, cols, block, scales, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_sr(const QuantizeArgs& a) {
  switch (a.xt) {
    case 0: return launch_sr_typed<0>(a);
    case 1: return launch_sr_typed<1>(a);
    case 2: return launch_sr_typed<2>(a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_transpose(const QuantizeArgs& a) {
  const int key = a.xt * 2 + a.fmt;
  switch (key) {
    case 0: return launch_transpose_typed<0, 0>(a);
    case 1: return launch_transpose_typed<0, 1>(a);
    case 2: return launch_transpose_typed<1, 0>(a);
    case 3: return launch_transpose_typed<1, 1>(a);
    case 4: return launch_transpose_typed<2, 0>(a);
    case 5: return launch_transpose_typed<2, 1>(a);
    default: return cudaErrorInvalidValue;
  }
}

size_t quantize_workspace_bytes(int gran, int64_t rows, int64_t cols, int delayed) {
  (void)rows;
  if (delayed) return 256;
  if (gran == 0) return 256;
  if (gran == 1) return 0;
  // header (16 bytes), amax bits[cols] padded to 16 bytes, m[cols]
  const size_t c4 = static_cast<size_t>((cols + 3) / 4) * 4;
  size_t b = 16 + c4 * 4 + static_cast<size_t>(cols) * 4;
  return (b + 255) / 256 * 256;
}

template <int DT, int FMT>
cudaError_t launch_delayed_batch_typed(const DelayedTensorArgs* t, int count, cudaStream_t stream) {
  constexpr int VEC = Dt<DT>::kVec;
  int dev = 0;
  cudaGetDevice(&dev);
  DelayedBatch b;
  memset(&b, 0, sizeof(b));
  b.count = count;
  int total = 0;
  for (int i = 0; i < count; ++i) {
    const bool vec = aligned(t[i].x, 16) && aligned(t[i].q, VEC);
    b.cta0[i] = total;
    total += flat_grid(vec ? t[i].n / VEC : t[i].n, dev, kUnroll);
    b.x[i] = t[i].x;
    b.n[i] = t[i].n;
    b.q[i] = t[i].q;
    b.scales[i] = t[i].scale;
    b.amax_out[i] = t[i].amax_out;
    b.ring[i] = t[i].ring;
    b.len[i] = t[i].ring_len;
    b.idx[i] = t[i].ring_idx;
    b.margin[i] = t[i].ring_margin;
    b.ws[i] = static_cast<uint32_t*>(t[i].ws);
    b.vec[i] = vec ? 1 : 0;
  }
  b.cta0[count] = total;
  return launch_pdl(k_delayed_batch<DT, FMT>, dim3(static_cast<unsigned>(total)), dim3(kThreads), 0, stream, false, b);
}

cudaError_t launch_quantize_delayed_batch(int xt, int fmt, const DelayedTensorArgs* t, int count,
                                          cudaStream_t stream) {
  if (count < 1 || count > kBatchMax) return cudaErrorInvalidValue;
  switch (xt * 2 + fmt) {
    case 0: return launch_delayed_batch_typed<0, 0>(t, count, stream);
    case 1: return launch_delayed_batch_typed<0, 1>(t, count, stream);
    case 2: return launch_delayed_batch_typed<1, 0>(t, count, stream);
    case 3: return launch_delayed_batch_typed<1, 1>(t, count, stream);
    case 4: return launch_delayed_batch_typed<2, 0>(t, count, stream);
    case 5: return launch_delayed_batch_typed<2, 1>(t, count, stream);
    default: return cudaErrorInvalidValue;
  }
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
