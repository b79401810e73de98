// fp8_cvt.cuh -- the saturating round-to-nearest-even FP8 conversion shared by
// the quantize kernels and the GEMM's FP8-output epilogue (hip-quant README
// "FP8 Formats": E4M3 max 448, E5M2 max 57344, RNE).  sm_100a only.
#pragma once

#include <cfloat>
#include <cstdint>

namespace hq {
namespace {

// Two f32 values -> two FP8 codes (lo in the low byte), saturating RNE; a
// NaN input gives the canonical code 0x7F.  FMT: 0 E4M3, 1 E5M2.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2_exact(float lo, float hi) {
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

// The same for inputs known not to be NaN: the conversion alone.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2_fast(float lo, float hi) {
  unsigned short r;
  if (FMT == 0)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int FMT>
__device__ __forceinline__ uint8_t cvt1_exact(float y) {
  return static_cast<uint8_t>(cvt2_exact<FMT>(y, 0.0f) & 0xFFu);
}

// |v| if finite, else 0 (NaN and +-Inf do not take part in amax).
__device__ __forceinline__ float finite_abs(float v) {
  const float a = fabsf(v);
  return (a <= FLT_MAX) ? a : 0.0f;
}

}  // namespace
}  // namespace hq
