/*
 * hq_oracle.c -- plain, slow, single-threaded CPU oracle for dynamic FP8
 * quantization (amax -> scale -> saturating RNE cast) and the scaled FP8
 * GEMM it feeds.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this
 * file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load it.  It shares no code, header, table or constant with the
 * CUDA library; every number below is derived here from the format
 * definitions.
 *
 * Sources (web pages this restates; no code is copied from them):
 *  [HQ]  hip-quant 0.6.0 README, "FP8 Formats" table (E4M3: 1s.4e.3m, bias 7,
 *        max +-448, NaN only; E5M2: 1s.5e.2m, bias 15, max +-57344, +-Inf and
 *        NaN) and the sentence after it (OCP round-to-nearest-even);
 *        "Training-path numerical guards" (quant scales are pre-quant
 *        multipliers, the reciprocal is the dequant scale; non-finite amax
 *        samples are ignored); "Scale / amax tracking" (history_len = 16).
 *  [AS]  AstrAI csrc/kernels/fp8/ops.cu: commit "finalize fp8 scale rings
 *        inside quantize kernels" (last-block epilogue folds amax into
 *        hist[idx], reduces the window, publishes the next scale; ring
 *        packs [hist | scale | counter]), pack_quantize_params (len =
 *        numel-2, idx = caller's slot, margin from the recipe), mm_fp8
 *        (out = a @ b^T * (sa*sb), FP32 accumulate), linear_backward_fp8
 *        (the bias gradient is the sum of g over its rows, cast back to
 *        g's dtype).
 *  [QS]  fuel-ir 0.22.4 src/quant_scale.rs: ScaleGranularity (PerTensor
 *        f32[1], PerToken f32[n_rows], PerChannel f32[n_cols]) and
 *        scale_count.
 *  [PR]  ROCm/aiter PR 6437, "Technical Details": out[M,N] bf16 from XQ[M,K],
 *        WQ[N,K], x_scale[M], w_scale[N].
 *  [GG]  megablocks-hip _dev/TODO-gg.md: per-expert Y_e = X_e . W_e^T, the
 *        output is overwritten, never accumulated.
 *
 * Readings where the pages are silent:
 *  R1  NaN input encodes to the canonical code 0x7F in both formats.
 *  R2  The cast saturates: |y| >= fmax (including +-Inf) -> sign | max code.
 *  R3  amax skips NaN and +-Inf elements.
 *  R4  amax == 0, or fmax/amax not finite -> multiplier m = 1.
 *  R5  The exported per-row/column/tensor scale is the dequant scale d = 1/m.
 *  R6  Delayed ring: after the cast, hist[idx] = amax; win = max(hist);
 *      if win is finite and > 0 the scale slot becomes ldexp(fmax/win,
 *      -margin), else it keeps its value; the counter slot is 0 on exit.
 *  R7  Per-channel reduces over rows (one scale per column), as [QS] says.
 *
 * Floating point: f32 steps are single f32 operations (compile with
 * -ffp-contract=off, no fast-math); everything else is exact integer
 * arithmetic or fp64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define HQO_E4M3 0
#define HQO_E5M2 1
#define HQO_F32 0
#define HQO_BF16 1
#define HQO_F16 2
#define HQO_PER_TENSOR 0
#define HQO_PER_TOKEN 1
#define HQO_PER_CHANNEL 2

/* ---------------------------------------------------------------- formats */

/* Format parameters straight from the [HQ] "FP8 Formats" table. */
typedef struct {
  int ebits, mbits, bias;
  double fmax;    /* largest finite magnitude */
  uint8_t maxcode; /* code of +fmax */
} fmt_info;

static fmt_info get_fmt(int fmt) {
  fmt_info f;
  if (fmt == HQO_E4M3) {
    /* 4 exponent bits, 3 mantissa bits, bias 7.  The all-ones exponent is
       still finite except for mantissa 111 (NaN), so the top finite value is
       exponent field 15, mantissa 110: (1 + 6/8) * 2^(15-7) = 448. */
    f.ebits = 4; f.mbits = 3; f.bias = 7;
    f.fmax = ldexp(1.0 + 6.0 / 8.0, 15 - 7);
    f.maxcode = (uint8_t)((15 << 3) | 6);
  } else {
    /* 5 exponent bits, 2 mantissa bits, bias 15; exponent field 31 is
       Inf/NaN, so the top finite value is (1 + 3/4) * 2^(30-15) = 57344. */
    f.ebits = 5; f.mbits = 2; f.bias = 15;
    f.fmax = ldexp(1.0 + 3.0 / 4.0, 30 - 15);
    f.maxcode = (uint8_t)((30 << 2) | 3);
  }
  return f;
}

double hqo_fmax(int fmt) { return get_fmt(fmt).fmax; }

/* Decode one code by its bit fields ([HQ] "FP8 Formats"). */
double hqo_decode(uint8_t c, int fmt) {
  fmt_info f = get_fmt(fmt);
  int s = (c >> 7) & 1;
  int e = (c >> f.mbits) & ((1 << f.ebits) - 1);
  int m = c & ((1 << f.mbits) - 1);
  double v;
  int emin = 1 - f.bias;
  if (fmt == HQO_E4M3 && (c & 0x7F) == 0x7F) return NAN;
  if (fmt == HQO_E5M2 && e == 31) {
    if (m != 0) return NAN;
    return s ? -INFINITY : INFINITY;
  }
  if (e == 0)
    v = ldexp((double)m, emin - f.mbits); /* subnormal: m * 2^(emin-mbits) */
  else
    v = ldexp(1.0 + ldexp((double)m, -f.mbits), e - f.bias);
  return s ? -v : v;
}

/* Saturating round-to-nearest-even encode of an f32 value (R1, R2, [HQ]).
   |y| as a double is exact; scaling by a power of two and nearbyint (the
   default rounding mode is to-nearest-even) rounds exactly once. */
uint8_t hqo_encode_sat(float y, int fmt) {
  fmt_info f = get_fmt(fmt);
  int emin = 1 - f.bias;
  uint8_t sign;
  double a, quantum, r;
  int e;
  if (isnan(y)) return 0x7F;
  sign = signbit(y) ? 0x80 : 0x00;
  a = fabs((double)y);
  if (a >= f.fmax) return (uint8_t)(sign | f.maxcode);
  if (a < ldexp(1.0, emin)) {
    quantum = ldexp(1.0, emin - f.mbits);
  } else {
    frexp(a, &e); /* a = g * 2^e, g in [0.5, 1): binade exponent is e-1 */
    quantum = ldexp(1.0, (e - 1) - f.mbits);
  }
  r = nearbyint(a / quantum) * quantum;
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, emin)) {
    /* subnormal: exponent field 0, mantissa = r / 2^(emin-mbits) */
    return (uint8_t)(sign | (int)(r / ldexp(1.0, emin - f.mbits)));
  }
  frexp(r, &e);
  {
    int efield = (e - 1) + f.bias;
    int mfield = (int)((ldexp(r, -(e - 1)) - 1.0) * (double)(1 << f.mbits));
    return (uint8_t)(sign | (efield << f.mbits) | mfield);
  }
}

/* ------------------------------------------------------------ bf16 / f16 */

float hqo_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

float hqo_f16_to_f32(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -24);
  else v = ldexp(1.0 + m / 1024.0, e - 15);
  return (float)(s ? -v : v);
}

/* Round a double to the nearest bf16 (ties to even), once. */
uint16_t hqo_double_to_bf16(double v) {
  double a, q, r;
  int e;
  float rf;
  uint32_t u;
  if (isnan(v)) return 0x7FC0;
  a = fabs(v);
  if (a == 0.0 || isinf(v)) {
    rf = (float)v;
    memcpy(&u, &rf, 4);
    return (uint16_t)(u >> 16);
  }
  if (a < ldexp(1.0, -126)) {
    q = ldexp(1.0, -133); /* bf16 subnormal step: 2^(-126-7) */
  } else {
    frexp(a, &e);
    q = ldexp(1.0, (e - 1) - 7);
  }
  r = nearbyint(a / q) * q;
  if (r >= ldexp(1.0, 128)) r = INFINITY;
  rf = (float)(v < 0 ? -r : r); /* exact: r is on the bf16 grid */
  memcpy(&u, &rf, 4);
  return (uint16_t)(u >> 16);
}

/* Correct bf16 rounding of an unevaluated sum hi + lo with |lo| <= ulp(hi)/2:
   only an exact bf16 midpoint in hi can be moved by lo. */
static uint16_t dd_to_bf16(double hi, double lo) {
  uint16_t r = hqo_double_to_bf16(hi);
  if (lo != 0.0 && isfinite(hi) && hi != 0.0) {
    double a = fabs(hi), q, t;
    int e;
    if (a < ldexp(1.0, -126)) q = ldexp(1.0, -133);
    else { frexp(a, &e); q = ldexp(1.0, (e - 1) - 7); }
    t = a / q;
    if (t - floor(t) == 0.5) {
      /* hi is a tie; the true value lies on lo's side of it */
      double nudged = hi + (lo > 0 ? 1.0 : -1.0) * q * 0.25;
      r = hqo_double_to_bf16(nudged);
    }
  }
  return r;
}

/* ------------------------------------------------------------------ amax */

static float load_elem(const void* x, int dtype, int64_t i) {
  if (dtype == HQO_F32) return ((const float*)x)[i];
  if (dtype == HQO_BF16) return hqo_bf16_to_f32(((const uint16_t*)x)[i]);
  return hqo_f16_to_f32(((const uint16_t*)x)[i]);
}

/* Multiplier m = fl32(fmax / amax) with reading R4. */
float hqo_multiplier(float amax, int fmt) {
  float fmax = (float)get_fmt(fmt).fmax;
  float m;
  if (!(amax > 0.0f)) return 1.0f;
  m = fmax / amax; /* one correctly rounded f32 division */
  if (!isfinite(m)) return 1.0f;
  return m;
}

/* scale_count per [QS] ScaleGranularity::scale_count. */
int64_t hqo_scale_count(int gran, int64_t rows, int64_t cols) {
  if (gran == HQO_PER_TENSOR) return 1;
  if (gran == HQO_PER_TOKEN) return rows;
  if (gran == HQO_PER_CHANNEL) return cols;
  return -1;
}

/* amax over the elements that share one scale (R3, R7).  out has
   scale_count(gran, rows, cols) entries. */
void hqo_amax(const void* x, int dtype, int64_t rows, int64_t cols, int gran,
              float* out) {
  int64_t n = hqo_scale_count(gran, rows, cols), r, c;
  for (r = 0; r < n; ++r) out[r] = 0.0f;
  for (r = 0; r < rows; ++r) {
    for (c = 0; c < cols; ++c) {
      float v = load_elem(x, dtype, r * cols + c);
      float a;
      int64_t slot;
      if (!isfinite(v)) continue;
      a = fabsf(v);
      slot = (gran == HQO_PER_TENSOR) ? 0 : (gran == HQO_PER_TOKEN ? r : c);
      if (a > out[slot]) out[slot] = a;
    }
  }
}

/* ---------------------------------------------------------------- quantize */

/* Delayed-scaling ring step (R6; AstrAI ops.cu ring commit): fold this
   step's amax into hist[idx], reduce the window, publish the next multiplier
   fmax / max(hist) / 2^margin when that window is finite and > 0, and leave
   the counter slot at 0. */
void hqo_ring_update(float amax, int fmt, float* ring, int ring_len, int ring_idx,
                     int ring_margin) {
  float win = 0.0f;
  int i;
  ring[ring_idx] = amax;
  for (i = 0; i < ring_len; ++i)
    if (ring[i] > win) win = ring[i];
  if (isfinite(win) && win > 0.0f) {
    float fmax = (float)get_fmt(fmt).fmax;
    float next = ldexpf(fmax / win, -ring_margin);
    if (isfinite(next) && next > 0.0f) ring[ring_len] = next;
  }
  ring[ring_len + 1] = 0.0f; /* counter slot, 0 on exit */
}

/* Dynamic quantize (ring == NULL) or delayed per-tensor quantize (ring !=
   NULL, R6).  q: rows*cols codes; scales: dequant scales d = 1/m (R5);
   amax_out (nullable): the amax array of the input at this granularity.
   Returns 0, or -1 on an invalid argument. */
int hqo_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int fmt,
                 int gran, uint8_t* q, float* scales, float* amax_out,
                 float* ring, int ring_len, int ring_idx, int ring_margin) {
  int64_t n = hqo_scale_count(gran, rows, cols), r, c;
  float* amax;
  float* mult;
  if (n < 0) return -1;
  if (ring && (gran != HQO_PER_TENSOR || ring_len < 1 || ring_idx < 0 ||
               ring_idx >= ring_len))
    return -1;
  amax = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  mult = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  hqo_amax(x, dtype, rows, cols, gran, amax);
  if (ring) {
    mult[0] = ring[ring_len]; /* the scale slot published by the last step */
  } else {
    for (r = 0; r < n; ++r) mult[r] = hqo_multiplier(amax[r], fmt);
  }
  for (r = 0; r < n; ++r) scales[r] = 1.0f / mult[r];
  for (r = 0; r < rows; ++r) {
    for (c = 0; c < cols; ++c) {
      int64_t slot = (gran == HQO_PER_TENSOR) ? 0 : (gran == HQO_PER_TOKEN ? r : c);
      float y = load_elem(x, dtype, r * cols + c) * mult[slot]; /* one f32 mul */
      q[r * cols + c] = hqo_encode_sat(y, fmt);
    }
  }
  if (amax_out)
    for (r = 0; r < n; ++r) amax_out[r] = amax[r];
  if (ring) hqo_ring_update(amax[0], fmt, ring, ring_len, ring_idx, ring_margin);
  free(amax);
  free(mult);
  return 0;
}

/* ---------------------------------------------------- stochastic E5M2 */

/* SplitMix64 (Steele, Lea and Flood 2014, with the constants of Vigna's
   reference implementation) as a counter-based generator: the draw for
   element index i under seed s is the (i+1)-th output of the generator
   started at state s; its top 32 bits are returned.  hqo_splitmix64_next
   steps one generator (used to pin the definition against its published
   outputs). */
static uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t hqo_splitmix64_next(uint64_t* state) {
  *state += 0x9E3779B97F4A7C15ull;
  return splitmix64_mix(*state);
}

uint32_t hqo_sr_bits(uint64_t seed, uint64_t idx) {
  return (uint32_t)(splitmix64_mix(seed + (idx + 1) * 0x9E3779B97F4A7C15ull) >> 32);
}

/* Stochastic rounding of an f32 to E5M2 ([HQ] "Stochastic E5M2 Backward
   Gradients": between the two adjacent E5M2 values, with probability
   proportional to the distance from the other one).  With g the E5M2 spacing
   at |y| (2^(e-2) for |y| in [2^e, 2^(e+1)) with e >= -14, else 2^-16),
   lo = floor(|y| / g) g and frac32 = floor((|y| - lo) / g * 2^32), |y|
   rounds up to lo + g iff the draw u < frac32, so P(up) = frac32 / 2^32.
   NaN gives 0x7F; |y| >= 57344 and +-Inf saturate; the sign is kept (a
   negative value rounded to zero is -0, code 0x80). */
uint8_t hqo_encode_e5m2_sr(float y, uint32_t u) {
  double a, g, t, q, fr, v;
  uint64_t frac32;
  int e;
  if (isnan(y)) return 0x7F;
  a = fabs((double)y);
  if (a >= 57344.0 || a == 0.0) return hqo_encode_sat(y, HQO_E5M2);
  frexp(a, &e); /* a = f * 2^e with f in [0.5, 1): |y| in [2^(e-1), 2^e) */
  e -= 1;
  g = ldexp(1.0, (e < -14 ? -14 : e) - 2);
  t = a / g; /* exact: g is a power of two */
  q = floor(t);
  fr = t - q; /* exact */
  frac32 = (uint64_t)floor(ldexp(fr, 32));
  v = (q + ((uint64_t)u < frac32 ? 1.0 : 0.0)) * g; /* on the E5M2 grid, <= 57344 */
  return hqo_encode_sat((float)(signbit(y) ? -v : v), HQO_E5M2);
}

/* Dynamic quantize to E5M2 with stochastic rounding: amax and the multiplier
   per granularity exactly as hqo_quantize (no ring), the cast of
   y = f32(x) * m by hqo_encode_e5m2_sr with the draw of the element's flat
   index r * cols + c under `seed`. */
int hqo_quantize_e5m2_sr(const void* x, int dtype, int64_t rows, int64_t cols,
                         int gran, uint64_t seed, uint8_t* q, float* scales,
                         float* amax_out) {
  int64_t n = hqo_scale_count(gran, rows, cols), r, c;
  float* amax;
  float* mult;
  if (n < 0) return -1;
  amax = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  mult = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  hqo_amax(x, dtype, rows, cols, gran, amax);
  for (r = 0; r < n; ++r) mult[r] = hqo_multiplier(amax[r], HQO_E5M2);
  for (r = 0; r < n; ++r) scales[r] = 1.0f / mult[r];
  for (r = 0; r < rows; ++r)
    for (c = 0; c < cols; ++c) {
      int64_t slot = (gran == HQO_PER_TENSOR) ? 0 : (gran == HQO_PER_TOKEN ? r : c);
      float y = load_elem(x, dtype, r * cols + c) * mult[slot]; /* one f32 mul */
      q[r * cols + c] = hqo_encode_e5m2_sr(y, hqo_sr_bits(seed, (uint64_t)(r * cols + c)));
    }
  if (amax_out)
    for (r = 0; r < n; ++r) amax_out[r] = amax[r];
  free(amax);
  free(mult);
  return 0;
}

/* ------------------------------------------------------------ block-wise */

/* Block-wise quantize ([HQ] "Block-wise FP8 Scaling"): one f32 dequant scale
   per block of `block` consecutive elements along the last dimension, scales
   [rows, ceil(cols / block)] (the last block of a row may be shorter).  Per
   block: amax over the finite |x|, m = fmax / amax (1 when amax is 0 or the
   quotient is not finite), scale = 1 / m, codes of f32(x) * m, rounded to
   nearest even or, with stochastic != 0 (E5M2 only), by hqo_encode_e5m2_sr
   with the draw of the element's flat index under `seed`. */
int hqo_quantize_blockwise(const void* x, int dtype, int64_t rows, int64_t cols,
                           int fmt, int64_t block, int stochastic, uint64_t seed,
                           uint8_t* q, float* scales, float* amax_out) {
  int64_t nb, r, b, c;
  if (block < 1 || rows < 0 || cols < 0 || (stochastic && fmt != HQO_E5M2)) return -1;
  nb = (cols + block - 1) / block;
  for (r = 0; r < rows; ++r)
    for (b = 0; b < nb; ++b) {
      int64_t c0 = b * block, c1 = c0 + block < cols ? c0 + block : cols;
      float amax = 0.0f, m;
      for (c = c0; c < c1; ++c) {
        float v = fabsf(load_elem(x, dtype, r * cols + c));
        if (isfinite(v) && v > amax) amax = v;
      }
      m = hqo_multiplier(amax, fmt);
      scales[r * nb + b] = 1.0f / m;
      if (amax_out) amax_out[r * nb + b] = amax;
      for (c = c0; c < c1; ++c) {
        float y = load_elem(x, dtype, r * cols + c) * m; /* one f32 mul */
        q[r * cols + c] = stochastic ? hqo_encode_e5m2_sr(y, hqo_sr_bits(seed, (uint64_t)(r * cols + c)))
                                     : hqo_encode_sat(y, fmt);
      }
    }
  return 0;
}

/* Block-wise dequantize: out = f32(dec(q) * scale) of the element's block
   (real ~= fp8 * block scale), one f32 multiply; bf16_out rounds that to
   bf16 (nearest even). */
int hqo_dequantize_blockwise(const uint8_t* q, int fmt, int64_t rows, int64_t cols,
                             int64_t block, const float* scales, int bf16_out,
                             void* out) {
  int64_t nb, r, c;
  if (block < 1 || rows < 0 || cols < 0) return -1;
  nb = (cols + block - 1) / block;
  for (r = 0; r < rows; ++r)
    for (c = 0; c < cols; ++c) {
      float v = (float)hqo_decode(q[r * cols + c], fmt) * scales[r * nb + c / block];
      if (bf16_out) ((uint16_t*)out)[r * cols + c] = hqo_double_to_bf16((double)v);
      else ((float*)out)[r * cols + c] = v;
    }
  return 0;
}

/* --------------------------------------------------------------------- GEMM */

/* Integer numerator of a finite code: value = n * 2^-frac, frac = 9 (E4M3)
   or 16 (E5M2).  The 256 numerators of each format are taken once from
   hqo_decode and cached; finite[] marks the codes that have one. */
static int64_t num_tbl[2][256];
static int finite_tbl[2][256];
static int tbl_ready[2];

static void build_tbl(int fmt) {
  int c;
  for (c = 0; c < 256; ++c) {
    double v = hqo_decode((uint8_t)c, fmt);
    finite_tbl[fmt][c] = isfinite(v) ? 1 : 0;
    num_tbl[fmt][c] = isfinite(v) ? (int64_t)ldexp(v, fmt == HQO_E4M3 ? 9 : 16) : 0; /* exact */
  }
  tbl_ready[fmt] = 1;
}

/* Exact dot product S = sum_k dec(a[k]) * dec(b[k]) as a double (exact for
   E4M3, one rounding of an exact integer for E5M2); non-finite operands fall
   back to IEEE double arithmetic. */
static double exact_dot(const uint8_t* a, const uint8_t* b, int64_t K, int fmt) {
  int frac = (fmt == HQO_E4M3) ? 9 : 16;
  const int64_t* nt;
  const int* ft;
  int64_t k;
  if (!tbl_ready[fmt]) build_tbl(fmt);
  nt = num_tbl[fmt];
  ft = finite_tbl[fmt];
  if (fmt == HQO_E4M3) {
    /* |n| <= 448 * 2^9 < 2^18: products < 2^36, K < 2^27 terms fit int64 */
    int64_t acc = 0;
    for (k = 0; k < K; ++k) {
      if (!ft[a[k]] || !ft[b[k]]) goto nonfinite;
      acc += nt[a[k]] * nt[b[k]];
    }
    return ldexp((double)acc, -2 * frac);
  } else {
    __int128 acc = 0;
    for (k = 0; k < K; ++k) {
      if (!ft[a[k]] || !ft[b[k]]) goto nonfinite;
      acc += (__int128)nt[a[k]] * (__int128)nt[b[k]];
    }
    return ldexp((double)acc, -2 * frac);
  }
nonfinite:
  {
    double s = 0.0;
    for (k = 0; k < K; ++k) s += hqo_decode(a[k], fmt) * hqo_decode(b[k], fmt);
    return s;
  }
}

static uint16_t gemm_entry(const uint8_t* xq, const uint8_t* wq, int fmt,
                           const float* xs, int64_t xs_len, const float* ws,
                           int64_t ws_len, int64_t K, int64_t m, int64_t n,
                           double* ref) {
  double s = exact_dot(xq + m * K, wq + n * K, K, fmt);
  double sx = (double)xs[xs_len == 1 ? 0 : m];
  double sw = (double)ws[ws_len == 1 ? 0 : n];
  double v = sx * sw * s;
  if (ref) *ref = v;
  return hqo_double_to_bf16(v);
}

/* out[m,n] = bf16(x_scale[m'] * w_scale[n'] * sum_k dec(XQ[m,k]) dec(WQ[n,k]))
   ([PR] Technical Details; [AS] mm_fp8 NT layout).  x_scale has M or 1
   entries, w_scale N or 1.  ref_out (nullable) receives the unrounded fp64
   value. */
void hqo_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, int fmt,
                   const float* xs, int64_t xs_len, const float* ws,
                   int64_t ws_len, int64_t M, int64_t N, int64_t K,
                   uint16_t* out, double* ref_out) {
  int64_t m, n;
  for (m = 0; m < M; ++m)
    for (n = 0; n < N; ++n)
      out[m * N + n] = gemm_entry(xq, wq, fmt, xs, xs_len, ws, ws_len, K, m, n,
                                  ref_out ? &ref_out[m * N + n] : NULL);
}

/* out[m,n] = bf16(x_scale[m'] * w_scale[n'] * sum_k dec(XQ) dec(WQ) + bias[n])
   with bias a bf16 vector of N entries ([AS] linear_forward_fp8: the bias is
   added in the GEMM epilogue, before the output rounding).  The sum and the
   scaling are exact or fp64 as in hqo_gemm_a8w8; the bias is added in fp64
   and the result rounded once to bf16. */
void hqo_gemm_a8w8_bias(const uint8_t* xq, const uint8_t* wq, int fmt,
                        const float* xs, int64_t xs_len, const float* ws,
                        int64_t ws_len, const uint16_t* bias, int64_t M,
                        int64_t N, int64_t K, uint16_t* out) {
  int64_t m, n;
  for (m = 0; m < M; ++m)
    for (n = 0; n < N; ++n) {
      double v;
      gemm_entry(xq, wq, fmt, xs, xs_len, ws, ws_len, K, m, n, &v);
      out[m * N + n] = hqo_double_to_bf16(v + (double)hqo_bf16_to_f32(bias[n]));
    }
}

/* Block-scaled GEMM ([HQ] "Block-scaled Linear and Adafactor Kernel Helpers":
   the pre-quantized linear consumes the FP8 bytes and FP32 per-block scales of
   both operands; [HQ] "Block-wise FP8 Scaling" fixes the layout: one dequant
   scale per block of `block` consecutive elements along K, xs [M, nb],
   ws [N, nb], nb = ceil(K / block), the last block the short remainder).
     out[m,n] = bf16( sum_b xs[m,b] * ws[n,b] * S_b[m,n]  (+ bias[n]) )
   with S_b the exact dot product of the codes over block b.  Each block's
   term is sx * sw * S_b in fp64 (sx * sw exact), the terms and the bias are
   summed in fp64 in block order, and the result is rounded once.  bias
   (bf16, N entries) is nullable. */
static double blockscaled_entry(const uint8_t* xq, const uint8_t* wq, int fmt,
                                const float* xs, const float* ws, int64_t block,
                                int64_t K, int64_t m, int64_t n) {
  int64_t nb = (K + block - 1) / block, b;
  double v = 0.0;
  for (b = 0; b < nb; ++b) {
    int64_t k0 = b * block, len = (K - k0 < block) ? K - k0 : block;
    double s = exact_dot(xq + m * K + k0, wq + n * K + k0, len, fmt);
    v += (double)xs[m * nb + b] * (double)ws[n * nb + b] * s;
  }
  return v;
}

void hqo_gemm_blockscaled(const uint8_t* xq, const uint8_t* wq, int fmt,
                          const float* xs, const float* ws, int64_t block,
                          const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                          uint16_t* out, double* ref_out) {
  int64_t m, n;
  for (m = 0; m < M; ++m)
    for (n = 0; n < N; ++n) {
      double v = blockscaled_entry(xq, wq, fmt, xs, ws, block, K, m, n);
      if (bias) v += (double)hqo_bf16_to_f32(bias[n]);
      if (ref_out) ref_out[m * N + n] = v;
      out[m * N + n] = hqo_double_to_bf16(v);
    }
}

/* The same at sampled (m, n) positions. */
void hqo_gemm_blockscaled_entries(const uint8_t* xq, const uint8_t* wq, int fmt,
                                  const float* xs, const float* ws, int64_t block,
                                  const uint16_t* bias, int64_t K,
                                  const int64_t* ms, const int64_t* ns,
                                  int64_t count, uint16_t* out) {
  int64_t i;
  for (i = 0; i < count; ++i) {
    double v = blockscaled_entry(xq, wq, fmt, xs, ws, block, K, ms[i], ns[i]);
    if (bias) v += (double)hqo_bf16_to_f32(bias[ns[i]]);
    out[i] = hqo_double_to_bf16(v);
  }
}

/* The same entries at sampled (m, n) positions only. */
void hqo_gemm_a8w8_entries(const uint8_t* xq, const uint8_t* wq, int fmt,
                           const float* xs, int64_t xs_len, const float* ws,
                           int64_t ws_len, int64_t K, const int64_t* ms,
                           const int64_t* ns, int64_t count, uint16_t* out) {
  int64_t i;
  for (i = 0; i < count; ++i)
    out[i] = gemm_entry(xq, wq, fmt, xs, xs_len, ws, ws_len, K, ms[i], ns[i], NULL);
}

/* Grouped a8w8 GEMM ([GG]): for expert e, rows [off[e], off[e+1]) of XQ times
   WQ[e]^T with x_scale[row] and w_scale[e, n].  Rows outside every expert's
   range are not written.  Returns -1 on malformed offsets. */
int hqo_grouped_gemm_a8w8(const uint8_t* xq, const uint8_t* wq, int fmt,
                          const float* xs, const float* ws,
                          const int32_t* off, int32_t E, int64_t M_total,
                          int64_t N, int64_t K, uint16_t* out) {
  int32_t e;
  int64_t m, n;
  if (off[0] != 0 || off[E] != M_total) return -1;
  for (e = 0; e < E; ++e) {
    if (off[e + 1] < off[e]) return -1;
    for (m = off[e]; m < off[e + 1]; ++m)
      for (n = 0; n < N; ++n) {
        double s = exact_dot(xq + m * K, wq + ((int64_t)e * N + n) * K, K, fmt);
        double v = (double)xs[m] * (double)ws[(int64_t)e * N + n] * s;
        out[m * N + n] = hqo_double_to_bf16(v);
      }
  }
  return 0;
}

/* Grouped bf16 GEMM with a wide accumulator: out = bf16(sum_k a*b).  Each
   bf16*bf16 product is exact in fp64 (8-bit significands); the sum is carried
   as an unevaluated double-double (Knuth's TwoSum), then rounded once. */
int hqo_grouped_gemm_bf16(const uint16_t* x, const uint16_t* w,
                          const int32_t* off, int32_t E, int64_t M_total,
                          int64_t N, int64_t K, uint16_t* out) {
  int32_t e;
  int64_t m, n, k;
  if (off[0] != 0 || off[E] != M_total) return -1;
  for (e = 0; e < E; ++e) {
    if (off[e + 1] < off[e]) return -1;
    for (m = off[e]; m < off[e + 1]; ++m)
      for (n = 0; n < N; ++n) {
        const uint16_t* a = x + m * K;
        const uint16_t* b = w + ((int64_t)e * N + n) * K;
        double hi = 0.0, lo = 0.0;
        for (k = 0; k < K; ++k) {
          double p = (double)hqo_bf16_to_f32(a[k]) * (double)hqo_bf16_to_f32(b[k]);
          double s = hi + p;
          double bb = s - hi;
          double err = (hi - (s - bb)) + (p - bb);
          hi = s;
          lo += err;
        }
        {
          double s = hi + lo; /* renormalise */
          double err = lo - (s - hi);
          out[m * N + n] = dd_to_bf16(s, err);
        }
      }
  }
  return 0;
}

/* Batch forms of the scalar encode/decode above (same arithmetic). */
void hqo_encode_sat_array(const float* y, int64_t n, int fmt, uint8_t* out) {
  int64_t i;
  for (i = 0; i < n; ++i) out[i] = hqo_encode_sat(y[i], fmt);
}

void hqo_decode_array(const uint8_t* c, int64_t n, int fmt, double* out) {
  int64_t i;
  for (i = 0; i < n; ++i) out[i] = hqo_decode(c[i], fmt);
}

/* ---------------------------------------------------------- bias gradient */

/* Round a double to the nearest f16 (ties to even), once: 10 fraction bits,
   exponent bias 15, subnormal step 2^-24, values from 65520 up to Inf. */
uint16_t hqo_double_to_f16(double v) {
  double a, q, r;
  int e;
  uint16_t sign = (v < 0 || (v == 0.0 && signbit(v))) ? 0x8000 : 0;
  if (isnan(v)) return 0x7E00;
  a = fabs(v);
  if (isinf(v)) return (uint16_t)(sign | 0x7C00);
  if (a == 0.0) return sign;
  if (a < ldexp(1.0, -14)) {
    q = ldexp(1.0, -24);
  } else {
    frexp(a, &e);
    q = ldexp(1.0, (e - 1) - 10);
  }
  r = nearbyint(a / q) * q;
  if (r > 65504.0) return (uint16_t)(sign | 0x7C00);
  if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
  frexp(r, &e); /* r = f * 2^e, f in [0.5, 1): leading bit 2^(e-1) */
  return (uint16_t)(sign | (uint16_t)((e - 1 + 15) << 10) |
                    (uint16_t)(r / ldexp(1.0, e - 1) * 1024.0 - 1024.0));
}

/* Bias gradient ([AS] linear_backward_fp8: the sum of g over dim 0, cast
   to g's dtype): sum[c] = sum over r of g[r, c] in fp64, rows in order,
   then rounded once to g's dtype (bf16 or f16 ties-to-even, or f32).
   out holds dtype elements [cols]; ref (optional) the fp64 sums. */
void hqo_grad_bias(const void* g, int dtype, int64_t rows, int64_t cols, void* out, double* ref) {
  int64_t r, c;
  double* s = (double*)calloc((size_t)(cols > 0 ? cols : 1), sizeof(double));
  if (!s) return;
  for (r = 0; r < rows; ++r) /* row by row: each column's terms still added in row order */
    for (c = 0; c < cols; ++c) s[c] += (double)load_elem(g, dtype, r * cols + c);
  for (c = 0; c < cols; ++c) {
    if (ref) ref[c] = s[c];
    if (dtype == 0) ((float*)out)[c] = (float)s[c];
    else if (dtype == 1) ((uint16_t*)out)[c] = hqo_double_to_bf16(s[c]);
    else ((uint16_t*)out)[c] = hqo_double_to_f16(s[c]);
  }
  free(s);
}
