// gemm.cu -- scaled FP8 (and bf16) GEMM on sm_100a tensor cores.
//
// out[m, n] = bf16_rn( acc[m, n] * x_scale[m'] * w_scale[n'] ),
// acc = sum_k A[m, k] * B[n, k] accumulated in FP32 on tcgen05 tensor cores.
// (ROCm/aiter PR 6437 "Technical Details": XQ[M,K], WQ[N,K], x_scale[M],
// w_scale[N], caller-owned bf16 out; AstrAI ops.cu mm_fp8: NT layout, FP32
// accumulate; megablocks-hip TODO-gg.md: the grouped per-expert form, output
// overwritten.)
//
// Design (persistent CTAs or CTA pairs, one per SM, 320 threads, 10 warps):
//   warp 0      TMA producer: one elected thread streams 128-byte-wide K
//               slices of A (128 rows) and B (BN rows) into a ring of shared
//               memory stages (128B swizzle), signalling mbarriers.
//   warp 1      allocates TMEM (two FP32 accumulators of up to 256 columns)
//               and issues tcgen05.mma (kind::f8f6f4 for FP8, kind::f16 for
//               bf16) from one thread; tcgen05.commit frees a stage /
//               publishes an accumulator (CTA pairs: cta_group::2).
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (two warps per
//               32-lane TMEM quadrant), scale, bias, round to bf16 (or FP8),
//               TMA or 16-byte stores.  Two accumulators let the epilogue of
//               tile i overlap the main loop of tile i+1.
// Every wait is bounded: on a stalled barrier the CTA records an error in a
// device word, drains what it has in flight and exits instead of hanging.
#include "fp8_cvt.cuh"
#include "hq_internal.cuh"
#include "launch.cuh"
#include "ptx.cuh"
#include "tc.cuh"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

namespace hq {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kBM = 128;            // tile rows (MMA M)
constexpr int kBKBytes = 128;       // K bytes per stage = one 128B swizzle row
constexpr int kGemmThreads = 320;   // CTA-pair kernel: TMA, MMA, 8 epilogue warps
constexpr int kGemm1Threads = 320;  // 1-CTA kernel: TMA, MMA, 8 epilogue warps
constexpr int kMaxExperts = 1024;
constexpr unsigned long long kDrainLimitNs = ptx::kDrainLimitNs;

struct Params {
  int M, N, K;          // M: rows of A (M_total for grouped), K in elements
  int nkb;              // number of K blocks
  int n_tiles, m_tiles; // m_tiles: dense only
  int group_m;          // rasterisation group (dense)
  int E;                // experts (1 for dense)
  const int32_t* offsets;
  const float* xs;
  int xs_bcast;
  const float* ws;
  int ws_bcast;
  uint16_t* out;
  uint32_t idesc;
  int prefetch;         // 1: L2-prefetch operands ahead of the TMA loads
  // fused epilogues (dense only): bias added before the bf16 rounding; FP8
  // output = the delayed per-tensor quantize of the bf16 result
  const uint16_t* bias;  // bf16 [N] or null
  uint8_t* qout;         // FP8 codes [M, N] or null (then out holds bf16)
  int qfmt;
  float* qscale;
  float* qamax;
  float* ring;
  int ring_len, ring_idx, ring_margin;
  uint32_t* qws;         // amax accumulator word
  // block-wise FP8 output instead of the ring: each row's 32-column blocks
  // quantized on their own, dequant scales [M, N / 32]
  float* qbs;
};

// ------------------------------------------------------------ PTX wrappers
using ptx::smem_u32;
using ptx::mbar_init;
using ptx::mbar_arrive_expect_tx;
using ptx::mbar_arrive;

// Bounded wait; a timeout is recorded in the device error word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit = ptx::kWaitLimitNs) {
  return ptx::mbar_wait(bar, parity, abort_flag, &g_device_error, kDevErrTimeout, limit);
}

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Two columns at once with packed f32x2 arithmetic: (a0, a1) * (x * s0,
// x * s1), each product rounded once (the same operations, in the same
// order, as the scalar form), plus the bias pair (b0, b1) by one fused
// multiply-add each when with_bias.
__device__ __forceinline__ void scale2(float a0, float a1, float s0, float s1, float x, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, s, xx;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 s, {%4, %5};\n\t"
      "mov.b64 xx, {%6, %6};\n\t"
      "mul.rn.f32x2 s, s, xx;\n\t"
      "mul.rn.f32x2 a, a, s;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(s0), "f"(s1), "f"(x));
}
__device__ __forceinline__ void scale2_bias(float a0, float a1, float s0, float s1, float x, float b0, float b1,
                                            float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, s, xx, b;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 s, {%4, %5};\n\t"
      "mov.b64 xx, {%6, %6};\n\t"
      "mov.b64 b, {%7, %8};\n\t"
      "mul.rn.f32x2 s, s, xx;\n\t"
      "fma.rn.f32x2 a, a, s, b;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(s0), "f"(s1), "f"(x), "f"(b0), "f"(b1));
}

// One chunk's 32 scaled values of a lane's row, plus the bias (bias != null),
// rounded to bf16 pairs: w[j] holds columns n0 + 2j (low half) and n0 + 2j + 1.
// has_acc == false (K == 0) reads the accumulator as zero.
__device__ __forceinline__ void chunk_to_bf16(const uint32_t (&v)[32], bool has_acc, float xsv, const float* sc,
                                              const uint16_t* bias, int n0, int N, uint32_t (&w)[16]) {
  if (bias == nullptr) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a0 = has_acc ? __uint_as_float(v[2 * j]) : 0.0f;
      const float a1 = has_acc ? __uint_as_float(v[2 * j + 1]) : 0.0f;
      float r0, r1;
      scale2(a0, a1, sc[2 * j], sc[2 * j + 1], xsv, r0, r1);
      w[j] = pack_bf16x2(r0, r1);
    }
  } else {
    const uint32_t* bp = reinterpret_cast<const uint32_t*>(bias) + (n0 >> 1);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a0 = has_acc ? __uint_as_float(v[2 * j]) : 0.0f;
      const float a1 = has_acc ? __uint_as_float(v[2 * j + 1]) : 0.0f;
      const uint32_t bb = (n0 + 2 * j < N) ? __ldg(bp + j) : 0u;
      float r0, r1;
      scale2_bias(a0, a1, sc[2 * j], sc[2 * j + 1], xsv, __uint_as_float(bb << 16), __uint_as_float(bb & 0xFFFF0000u),
                  r0, r1);
      w[j] = pack_bf16x2(r0, r1);
    }
  }
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// FP8 output of one chunk: codes of f32(bf16 value) * m, saturating RNE (NaN
// -> 0x7F), into c4 (the lane's 32 codes, column n0 in the low byte of
// c4[0]); the lane's finite-only amax over its valid columns is kept as the
// raw bits of the largest bf16 magnitude in qraw (for non-negative bf16
// values the unsigned order of the bits is the numeric order), or in qam on
// the exact path.  Columns past N hold zero (their scales are zero), so only
// rows past the tile's valid rows (vrow false) need excluding.  A chunk
// without an Inf or NaN takes one max.u16x2 per pair and the plain
// conversion; otherwise each element is checked.
// Block-wise FP8 output: the multiplier of one 32-column block of a row
// (this lane's chunk of bf16 results), as the block-wise quantize derives it:
// amax over the finite |h|, m = fmax / amax, 1 when amax is 0 or the quotient
// is not finite.
__device__ __forceinline__ float chunk_block_multiplier(const uint32_t (&w)[16], int qfmt) {
  uint32_t mx = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
    if (lo < 0x7F80u) mx = max(mx, lo);  // bf16 magnitudes below Inf: bit order = value order
    if (hi < 0x7F80u) mx = max(mx, hi);
  }
  const float a = __uint_as_float(mx << 16);
  if (!(a > 0.0f)) return 1.0f;
  const float m = __fdiv_rn(qfmt == 0 ? kFmaxE4M3 : kFmaxE5M2, a);
  return (m <= FLT_MAX) ? m : 1.0f;
}

__device__ __forceinline__ void chunk_to_fp8(const uint32_t (&w)[16], int qfmt, float qm, bool vrow, int n0, int N,
                                             uint32_t& qraw, float& qam, uint32_t (&c4)[8]) {
  uint32_t mx = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) mx = max_u16x2(mx, w[j] & 0x7FFF7FFFu);
  const uint32_t mmax = max(mx & 0xFFFFu, mx >> 16);
  if (mmax < 0x7F80u) {  // no Inf or NaN in this lane's chunk
    if (vrow) qraw = max(qraw, mmax);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float lo = __uint_as_float(w[j] << 16);
      const float hi = __uint_as_float(w[j] & 0xFFFF0000u);
      const uint32_t c2 = (qfmt == 0) ? cvt2_fast<0>(__fmul_rn(lo, qm), __fmul_rn(hi, qm))
                                      : cvt2_fast<1>(__fmul_rn(lo, qm), __fmul_rn(hi, qm));
      c4[j >> 1] = (j & 1) ? (c4[j >> 1] | (c2 << 16)) : c2;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float lo = __uint_as_float(w[j] << 16);
      const float hi = __uint_as_float(w[j] & 0xFFFF0000u);
      if (vrow && n0 + 2 * j < N) qam = fmaxf(qam, fmaxf(finite_abs(lo), finite_abs(hi)));
      const uint32_t c2 = (qfmt == 0) ? cvt2_exact<0>(__fmul_rn(lo, qm), __fmul_rn(hi, qm))
                                      : cvt2_exact<1>(__fmul_rn(lo, qm), __fmul_rn(hi, qm));
      c4[j >> 1] = (j & 1) ? (c4[j >> 1] | (c2 << 16)) : c2;
    }
  }
}

// End of a kernel with an FP8 output: the CTA's amax joins the workspace
// word; the last CTA (threadfence + the ring's counter word) folds it into
// the ring and publishes the next multiplier, as the delayed quantize does.
template <int NWARPS>
__device__ __forceinline__ void finalize_fp8_out(const Params& p, float qam) {
  __shared__ float red[NWARPS];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) qam = fmaxf(qam, __shfl_xor_sync(0xFFFFFFFFu, qam, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = qam;
  __syncthreads();
  if (threadIdx.x != 0) return;
  float a = 0.0f;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) a = fmaxf(a, red[w]);
  atomicMax(p.qws, __float_as_uint(a));  // non-negative: bit order = value order
  __threadfence();
  uint32_t* counter = reinterpret_cast<uint32_t*>(p.ring + p.ring_len + 1);
  if (atomicAdd(counter, 1u) != gridDim.x - 1) return;
  __threadfence();
  const float am = __uint_as_float(atomicExch(p.qws, 0u));
  const float m = __ldcg(p.ring + p.ring_len);  // the multiplier every CTA used
  p.ring[p.ring_idx] = am;
  float win = 0.0f;
  for (int i = 0; i < p.ring_len; ++i) win = fmaxf(win, __ldcg(p.ring + i));
  if (win <= FLT_MAX && win > 0.0f) {
    const float next = ldexpf(__fdiv_rn(p.qfmt == 0 ? kFmaxE4M3 : kFmaxE5M2, win), -p.ring_margin);
    if (next <= FLT_MAX && next > 0.0f) p.ring[p.ring_len] = next;
  }
  p.qscale[0] = __fdiv_rn(1.0f, m);
  if (p.qamax) p.qamax[0] = am;
  atomicExch(counter, 0u);
}

// L2 prefetch of a TMA tile (no shared-memory destination, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(c0), "r"(c1)
               : "memory");
}

// TMA tile store shared -> global (clipped at the tensor's bounds), and its
// bulk-group bookkeeping.
// The output tile store carries an L2 evict_first policy: nothing reads the
// output again in this kernel, and letting L2 write it back early (while the
// main loop leaves DRAM mostly idle) keeps dirty lines from piling up for the
// next kernel to flush.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1, uint64_t pol) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
                   map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed group has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_le0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// ------------------------------------------------------------ epilogue
// One epilogue warp's share of a tile: chunks half, half + 2, ... of 32
// columns (chunk j's scales at wsh + 32 j), read from TMEM at tacc (the
// warp's lane quadrant and the accumulator's first column).  Per chunk the
// warp scales (+ bias) and rounds to bf16, then writes either the FP8 codes,
// or the 32 x 32 chunk through its staging tile with one TMA store (rows
// inside the tile's valid rows, a whole chunk inside the tile), or masked
// 16-byte stores.
template <int KIND, int kChunks>
__device__ __forceinline__ void epilogue_chunks(uint32_t tacc, int half, int lane, int col0, int col_end, int tile_end,
                                                int row0, bool vrow, bool tma_ok, bool has_acc, float xsv,
                                                const float* wsh, const Params& p, const uint16_t* bias, uint16_t* orow,
                                                uint8_t* qrow, float* qsrow, float qm, uint32_t& qraw, float& qam,
                                                uint8_t* sb, const CUtensorMap* tm_out, uint64_t out_pol) {
  auto process = [&](const uint32_t (&v)[32], int j) {
    const int n0 = col0 + (half + 2 * j) * 32;
    if (n0 >= col_end) return;
    uint32_t w[16];
    chunk_to_bf16(v, has_acc, xsv, wsh + j * 32, bias, n0, p.N, w);
    if (KIND == 0 && qrow != nullptr) {
      uint32_t c4[8];
      float qmc = qm;
      if (p.qbs != nullptr) {  // block-wise: this chunk is one whole block of the row (N % 32 == 0)
        qmc = chunk_block_multiplier(w, p.qfmt);
        if (vrow) qsrow[n0 >> 5] = __fdiv_rn(1.0f, qmc);
      }
      chunk_to_fp8(w, p.qfmt, qmc, vrow, n0, p.N, qraw, qam, c4);
      if (tma_ok && n0 + 32 <= tile_end) {
        // the 32 x 32 codes through the staging tile, 32-byte rows with the
        // 32-byte swizzle: 16-byte half h of row r sits at h ^ ((r >> 2) & 1)
        if (lane == 0) bulk_wait_read_le0();
        __syncwarp();
        const uint32_t flip = (static_cast<uint32_t>(lane) >> 2) & 1u;
        st_shared_v4(sb + lane * 32 + (flip << 4), c4[0], c4[1], c4[2], c4[3]);
        st_shared_v4(sb + lane * 32 + ((flip ^ 1u) << 4), c4[4], c4[5], c4[6], c4[7]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tm_out, sb, n0, row0, out_pol);
          bulk_commit_group();
        }
      } else if (vrow) {  // N % 16 == 0 and n0 % 32 == 0: 16 or 32 codes of this chunk lie inside the row
        st_global_v4(qrow + n0, c4[0], c4[1], c4[2], c4[3]);
        if (n0 + 32 <= p.N) st_global_v4(qrow + n0 + 16, c4[4], c4[5], c4[6], c4[7]);
      }
      return;
    }
    // the tensor map clips at M and N; a 16-column tail chunk inside N is masked
    if (tma_ok && n0 + 32 <= tile_end) {
      if (lane == 0) bulk_wait_read_le0();  // the previous chunk's store has read the staging tile
      __syncwarp();
      // the staging tile is the 64-byte-swizzled image of the 32 x 32 box:
      // 16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3), which
      // spreads each quarter-warp's stores over all banks
#pragma unroll
      for (int k = 0; k < 4; ++k)
        st_shared_v4(sb + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4), w[4 * k], w[4 * k + 1], w[4 * k + 2],
                     w[4 * k + 3]);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tm_out, sb, n0, row0, out_pol);
        bulk_commit_group();
      }
    } else if (vrow) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (n0 + 8 * k < col_end) st_global_v4(orow + n0 + 8 * k, w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
  };
#pragma unroll 1
  for (int j = 0; half + 2 * j < kChunks; ++j) {
    uint32_t v[32];
    tmem_ld32(tacc + static_cast<uint32_t>((half + 2 * j) * 32), v);
    process(v, j);
  }
}

// ------------------------------------------------------------ tile schedule
struct Tile {
  int a_row;   // first A row loaded (global)
  int b_row;   // first B row loaded (global, in the [E*N, K] view)
  int row_lo;  // rows [row_lo, row_hi) are written
  int row_hi;
  int col0;    // first output column
  int expert;
};

// Tile t of the persistent loop -> rows, columns and expert.  Dense: TM-row
// tiles rasterised in groups of group_m M-tiles.  Grouped: the per-expert
// tile prefix (built by build_tile_prefix) is searched for t's expert.
template <int TM, int BN>
__device__ __forceinline__ Tile decode_tile(int t, const Params& p, const int* prefix, const int* starts) {
  Tile T;
  if (p.offsets == nullptr) {
    const int per_group = p.group_m * p.n_tiles;
    const int g = t / per_group;
    const int within = t - g * per_group;
    const int gm = min(p.group_m, p.m_tiles - g * p.group_m);
    const int mt = g * p.group_m + within % gm;
    const int nt = within / gm;
    T.row_lo = mt * TM;
    T.row_hi = min(p.M, T.row_lo + TM);
    T.a_row = T.row_lo;
    T.col0 = nt * BN;
    T.b_row = T.col0;
    T.expert = 0;
  } else {
    int lo = 0, hi = p.E;  // find e with prefix[e] <= t < prefix[e+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int local = t - prefix[e];
    const int mt = local / p.n_tiles;
    const int nt = local - mt * p.n_tiles;
    T.row_lo = starts[e] + mt * TM;
    T.row_hi = min(starts[e + 1], T.row_lo + TM);
    T.a_row = T.row_lo;
    T.col0 = nt * BN;
    T.b_row = e * p.N + T.col0;
    T.expert = e;
  }
  return T;
}

// One thread: clamp the device offsets into [prev, M], record each expert's
// first row and the prefix of its TM-row x BN tiles.  Malformed offsets are
// flagged in the device error word (once per launch).
template <int TM>
__device__ void build_tile_prefix(const Params& p, int* prefix, int* starts) {
  bool bad = false;
  int prev = 0;
  int acc = 0;
  for (int e = 0; e <= p.E; ++e) {
    int o = p.offsets[e];
    if ((e == 0 && o != 0) || (e == p.E && o != p.M) || o < prev || o > p.M) bad = true;
    o = min(max(o, prev), p.M);
    if (e == 0) o = 0;
    starts[e] = o;
    if (e > 0) {
      const int cnt = o - prev;
      prefix[e - 1] = acc;
      acc += ((cnt + TM - 1) / TM) * p.n_tiles;
    }
    prev = o;
  }
  prefix[p.E] = acc;
  if (bad && blockIdx.x == 0) atomicOr(&g_device_error, kDevErrBadOffsets);
}

// ------------------------------------------------------------------ kernel
// AROWS: rows of A loaded per K block.  128 normally; for small M (decode)
// only the first AROWS >= M rows are loaded, packed at AROWS-row stride, which
// leaves room for more of B.  The MMA still reads 128 rows of A from the
// block start; rows past AROWS then come from the following blocks and only
// produce accumulator rows >= M, which are never stored.
// KPS: consecutive K blocks per pipeline stage.  With KPS > 1 each stage asks
// DRAM for KPS * 128 contiguous bytes of every weight row at once instead of
// one 128-byte piece per row, so more of each opened DRAM page is used.
template <int KIND, int BN, int STAGES, int AROWS = kBM, int KPS = 1>
__global__ void __launch_bounds__(kGemm1Threads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_out, const Params p) {
  static_assert((STAGES * KPS - 1) * AROWS * kBKBytes + kBM * kBKBytes <= STAGES * KPS * (AROWS + BN) * kBKBytes,
                "the MMA's 128-row read of the last A block must stay inside shared memory");
  static_assert(AROWS % 8 == 0 && (AROWS * kBKBytes) % 1024 == 0, "A blocks keep the 1024-byte swizzle atom");
  static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "MMA N (M = 128): a multiple of 16 in [64, 256]");
  constexpr int kChunks = (BN + 31) / 32;      // 32-column epilogue chunks (the last may hold 16)
  constexpr int kMyChunks = (kChunks + 1) / 2;  // per epilogue warp (two warps per quadrant)
  constexpr int kABytes = AROWS * kBKBytes;  // one K block of A
  constexpr int kBBytes = BN * kBKBytes;     // one K block of B
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr int kKElems = (KIND == 0) ? 128 : 64;  // K elements per stage
  constexpr uint32_t kTmemCols = (2 * BN <= 256) ? 256u : 512u;
  constexpr uint32_t kAccStride = (2 * BN <= 256) ? BN : 256u;  // TMEM columns between the two accumulators
  constexpr int kPrefetch = 2 * STAGES;  // L2 prefetch distance, in K blocks

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t final_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int tile_prefix[kMaxExperts + 1];
  __shared__ int row_start[kMaxExperts + 1];

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-byte aligned stages
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * KPS * kABytes;
  // epilogue: one 32 x 32 bf16 staging tile (2 KB) per warp for TMA stores,
  // and each warp's BN/2 column scales
  uint8_t* sOut = smem + STAGES * KPS * kStageBytes;
  float* sWs = reinterpret_cast<float*>(sOut + 8 * 2048);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);  // one arrive per epilogue warp
    }
    mbar_init(&final_bar, 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  pdl_wait();  // launched with programmatic stream serialization: global memory only after this
  pdl_launch_dependents();
  if (threadIdx.x == 32 && p.offsets != nullptr) build_tile_prefix<kBM>(p, tile_prefix, row_start);
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_a) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_b) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_out) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total = (p.offsets != nullptr) ? tile_prefix[p.E] : p.m_tiles * p.n_tiles;
  float qam = 0.0f;    // FP8 output: this thread's finite-only amax of the bf16 result (exact path)
  uint32_t qraw = 0;   // the same as the raw bits of the largest bf16 magnitude (fast path)

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_parity[STAGES];
      bool armed[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) { armed[s] = false; armed_parity[s] = 0; }
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const Tile T = decode_tile<kBM, BN>(t, p, tile_prefix, row_start);
        for (int kb = 0; kb < p.nkb; kb += KPS) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { stop = true; break; }
          const int nsub = min(KPS, p.nkb - kb);
          mbar_arrive_expect_tx(&full_bar[stage], nsub * kStageBytes);
          for (int u = 0; u < nsub; ++u) {
            tma_load_2d(sA + (stage * KPS + u) * kABytes, &tm_a, &full_bar[stage], (kb + u) * kKElems, T.a_row);
            tma_load_2d(sB + (stage * KPS + u) * kBBytes, &tm_b, &full_bar[stage], (kb + u) * kKElems, T.b_row);
          }
          // L2 prefetch of both operands kPrefetch blocks ahead: the ring
          // alone cannot cover DRAM latency at this tile's byte rate
          if (p.prefetch && kb + kPrefetch < p.nkb) {
            tma_prefetch_2d(&tm_a, (kb + kPrefetch) * kKElems, T.a_row);
            tma_prefetch_2d(&tm_b, (kb + kPrefetch) * kKElems, T.b_row);
          }
#pragma unroll
          for (int s = 0; s < STAGES; ++s)
            if (s == stage) { armed[s] = true; armed_parity[s] = phase; }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (abort_flag) {
        // drain: every armed stage's last transfer must land before exit
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
          int dummy = 0;
          if (armed[s]) mbar_wait(&full_bar[s], armed_parity[s], &dummy, kDrainLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    bool issued = false;
    bool stop = false;
    int i = 0;
    for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++i) {
      const int acc = i & 1;
      const uint32_t acc_phase = (i >> 1) & 1;
      // the warp agrees on giving up a wait, so that no lane is left at a
      // warp-wide step after another has left
      if (__any_sync(0xFFFFFFFFu, !mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &abort_flag))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * kAccStride;
      for (int kb = 0; kb < p.nkb; kb += KPS) {
        if (__any_sync(0xFFFFFFFFu, !mbar_wait(&full_bar[stage], phase, &abort_flag))) { stop = true; break; }
        tc_fence_after();
        if (lane == 0) {
          const int nsub = min(KPS, p.nkb - kb);
          for (int u = 0; u < nsub; ++u) {
            const uint64_t ad = smem_desc(smem_u32(sA + (stage * KPS + u) * kABytes));
            const uint64_t bd = smem_desc(smem_u32(sB + (stage * KPS + u) * kBBytes));
#pragma unroll
            for (int k = 0; k < kBKBytes / 32; ++k)  // 32 bytes of K per instruction
              mma_issue<KIND>(d_tmem, ad + 2u * k, bd + 2u * k, p.idesc, (kb + u > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty_bar[stage]);
          issued = true;
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (stop) break;
      if (lane == 0) tc_commit(&tfull_bar[acc]);
      __syncwarp();
    }
    if (abort_flag && lane == 0 && issued) {
      int dummy = 0;
      tc_commit(&final_bar);
      mbar_wait(&final_bar, 0, &dummy, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- epilogue
    // Eight warps: warp w reads TMEM lane quadrant w % 4 (32 rows); the two
    // warps of a quadrant take alternate 32-column chunks of the BN columns.
    // Per chunk a warp scales, rounds to bf16 and, when its 32 rows lie
    // inside the tile's valid rows (the tensor map clips at M and N), writes
    // the chunk through a staging tile with one TMA store; a 32-row group
    // that straddles an expert boundary uses masked 16-byte stores instead.
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;
    uint8_t* sb = sOut + ew * 2048;
    float* wsh = sWs + ew * kMyChunks * 32;
    const uint64_t out_pol = l2_evict_first_policy();
    const float qm = (p.qout != nullptr && p.qbs == nullptr) ? __ldcg(p.ring + p.ring_len) : 0.0f;  // the delayed multiplier
    const bool has_acc = p.nkb > 0;
    const uint16_t* bias = (KIND == 0) ? p.bias : nullptr;
    int i = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      const int acc = i & 1;
      const uint32_t acc_phase = (i >> 1) & 1;
      // The tile's row and column scales do not depend on the accumulator:
      // they are loaded before the wait, so their latency overlaps the
      // tile's main loop instead of adding to the epilogue.
      const Tile T = decode_tile<kBM, BN>(t, p, tile_prefix, row_start);
      const int row0 = T.row_lo + quad * 32;
      const int row = row0 + lane;
      const bool vrow = row < T.row_hi;
      // rows past M are clipped by the tensor map; rows of another expert are not
      const bool tma_ok = row0 < T.row_hi && (p.offsets == nullptr || row0 + 32 <= T.row_hi);
      const int ncap = min(p.N, T.col0 + BN);  // end of this tile's columns
      float xsv = 0.0f;
      if (vrow) xsv = (KIND == 0) ? __ldg(p.xs + (p.xs_bcast ? 0 : row)) : 1.0f;
      float wpre[kMyChunks];
      {
        const float* wsp = p.ws + (p.ws_bcast ? 0 : static_cast<int64_t>(T.expert) * p.N);
#pragma unroll
        for (int j = 0; j < kMyChunks; ++j) {
          const int ch = half + 2 * j;
          const int n = T.col0 + ch * 32 + lane;
          wpre[j] = (KIND != 0) ? 1.0f
                                : ((ch < kChunks && n < p.N) ? __ldg(wsp + (p.ws_bcast ? 0 : n)) : 0.0f);
        }
      }
      // the warp agrees on giving up: the TMEM loads below are warp-wide
      if (__any_sync(0xFFFFFFFFu, !mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < kMyChunks; ++j) wsh[j * 32 + lane] = wpre[j];
      __syncwarp();
      uint16_t* orow = p.out + static_cast<int64_t>(vrow ? row : 0) * p.N;
      uint8_t* qrow = (KIND == 0 && p.qout != nullptr) ? p.qout + static_cast<int64_t>(vrow ? row : 0) * p.N : nullptr;
      float* qsrow = (KIND == 0 && p.qbs != nullptr) ? p.qbs + static_cast<int64_t>(vrow ? row : 0) * (p.N >> 5) : nullptr;
      epilogue_chunks<KIND, kChunks>(
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc) * kAccStride, half, lane,
          T.col0, ncap, T.col0 + BN, row0, vrow, tma_ok, has_acc, xsv, wsh, p, bias, orow, qrow, qsrow, qm, qraw, qam, sb, &tm_out,
          out_pol);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
    }
    if (lane == 0) bulk_wait_all();  // stores complete before the CTA's shared memory goes
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (KIND == 0 && p.qout != nullptr && p.qbs == nullptr)
    finalize_fp8_out<kGemm1Threads / 32>(p, fmaxf(qam, __uint_as_float(qraw << 16)));
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// --------------------------------------------------------------- host side
// bf16 out[M, N] for TMA stores: 32 x 32 boxes (64-byte rows) with the
// 64-byte swizzle, so that the epilogue's staging stores avoid bank
// conflicts.
bool make_out_map(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols, std::string* msg) {
  auto encode = get_encode_fn();
  if (!encode) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[128];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (%d) for the output", static_cast<int>(r));
    *msg = buf;
    return false;
  }
  return true;
}

// FP8 codes out[M, N] (N % 16 == 0) for TMA stores: 32 x 32 boxes (32-byte
// rows) with the 32-byte swizzle.
bool make_codes_map(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols, std::string* msg) {
  auto encode = get_encode_fn();
  if (!encode) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[128];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (%d) for the FP8 output", static_cast<int>(r));
    *msg = buf;
    return false;
  }
  return true;
}

// The output's tensor map: the bf16 out, or the FP8 codes with an FP8 output.
bool make_result_map(CUtensorMap* map, const GemmArgs& a, std::string* msg) {
  if (a.q_out != nullptr)
    return make_codes_map(map, a.q_out, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.N), msg);
  return make_out_map(map, a.out, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.N), msg);
}

void set_fused_epilogue(const GemmArgs& a, Params& p) {
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.qout = a.q_out;
  p.qfmt = a.q_fmt;
  p.qscale = a.q_scale;
  p.qamax = a.q_amax;
  p.ring = a.ring;
  p.ring_len = a.ring_len;
  p.ring_idx = a.ring_idx;
  p.ring_margin = a.ring_margin;
  p.qws = a.q_ws;
  p.qbs = a.q_bscales;
}

template <int KIND, int BN, int STAGES, int AROWS = kBM, int KPS = 1>
cudaError_t run(const GemmArgs& a, std::string* msg) {
  constexpr int kElem = (KIND == 0) ? 1 : 2;
  constexpr int kSmem = STAGES * KPS * (AROWS + BN) * kBKBytes + 8 * 2048 + 8 * (((BN + 31) / 32 + 1) / 2) * 32 * 4 + 1024;
  static_assert(kSmem + 8352 <= 232448, "shared memory over the 227 KB per-CTA limit");
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err =
        cudaFuncSetAttribute(k_gemm<KIND, BN, STAGES, AROWS, KPS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  });
  if (attr_err != cudaSuccess) {
    *msg = "cudaFuncSetAttribute failed";
    return attr_err;
  }
  CUtensorMap ta, tb;
  memset(&ta, 0, sizeof(ta));
  memset(&tb, 0, sizeof(tb));
  if (a.K > 0) {  // K == 0: no loads are issued and the maps are never read
    if (!make_map(&ta, a.a, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), kElem, AROWS, msg) ||
        !make_map(&tb, a.b, static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K),
                  kElem, BN, msg))
      return cudaErrorInvalidValue;
  }
  CUtensorMap to;
  if (!make_result_map(&to, a, msg)) return cudaErrorInvalidValue;

  Params p;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.nkb = static_cast<int>((a.K + (kBKBytes / kElem) - 1) / (kBKBytes / kElem));
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.m_tiles = static_cast<int>((a.M + kBM - 1) / kBM);
  p.group_m = 16;
  p.E = a.E;
  p.offsets = a.offsets;
  p.xs = a.x_scale;
  p.xs_bcast = (a.x_scale_len == 1) ? 1 : 0;
  p.ws = a.w_scale;
  p.ws_bcast = (a.w_scale_len == 1) ? 1 : 0;
  p.out = static_cast<uint16_t*>(a.out);
  // Grouped tiles re-read A and B from L2 at a high byte rate and gain from
  // the prefetch; the small-M dense stream reads W once and loses by it.
  p.prefetch = (a.offsets != nullptr) ? 1 : 0;
  set_fused_epilogue(a, p);
  const uint32_t ab_fmt = (KIND == 0) ? static_cast<uint32_t>(a.fmt) : 1u;  // E4M3/E5M2, or BF16
  p.idesc = (1u << 4)                                   // D: FP32
            | (ab_fmt << 7) | (ab_fmt << 10)            // A and B element types
            | (static_cast<uint32_t>(BN >> 3) << 17)     // N / 8
            | (static_cast<uint32_t>(kBM >> 4) << 24);   // M / 16 (A and B K-major)

  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = device_sm_count(dev);
  int64_t tiles_bound;
  if (a.offsets == nullptr)
    tiles_bound = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  else
    tiles_bound = (static_cast<int64_t>(p.m_tiles) + a.E) * p.n_tiles;
  int grid = static_cast<int>(tiles_bound < sms ? tiles_bound : sms);
  if (grid < 1) grid = 1;
  return launch_pdl(k_gemm<KIND, BN, STAGES, AROWS, KPS>, dim3(grid), dim3(kGemm1Threads), kSmem, a.stream, false,
                    ta, tb, to, p);
}

// ====================================================== 2-CTA pair kernel
// Dense GEMM on CTA pairs (a cluster of 2, tcgen05 cta_group::2): the pair
// computes a 256 x BN tile.  CTA rank r loads A rows [m0 + 128 r, +128) and
// B rows [n0 + BN/2 r, +BN/2) into its own shared memory; the leader (rank 0)
// issues one M=256 MMA that reads both CTAs' stages, and each CTA's TMEM
// holds its own 128 accumulator rows.  Per SM this halves the B bytes per
// MMA cycle of the 1-CTA 128 x BN tile, which lets six stages fit.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory, completing on an mbarrier that
// may live in the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster_addr, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
      : "memory");
}
// Commit this thread's MMAs to the same barrier offset in both CTAs.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
template <int KIND>
__device__ __forceinline__ void mma_issue_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  }
}

// BN = SUBN * NSUB columns per pair tile; one MMA per sub-tile per K step
// (M = 256 across the pair, N = SUBN), each CTA holding SUBN/2 rows of every
// sub-tile of B.  When two BN-column accumulators fit in TMEM (BN <= 256),
// tile i's epilogue overlaps tile i+1's main loop.  NSUB = 2: each K step issues two
// MMAs against the same A stage (fewer operand bytes per flop) into one
// accumulator of up to 512 columns; the epilogue then does not overlap.
template <int KIND, int SUBN, int NSUB, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    k_gemm2(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
            const __grid_constant__ CUtensorMap tm_out, const Params p) {
  constexpr int BN = SUBN * NSUB;
  static_assert(SUBN % 16 == 0 && SUBN >= 32 && SUBN <= 256, "MMA N (M = 256 across the pair): 16 .. 256, step 16");
  static_assert((SUBN / 2) % 8 == 0, "each CTA's half of a sub-tile keeps whole 1024-byte swizzle atoms");
  static_assert(BN % 32 == 0 && BN <= 512, "32-column epilogue chunks; at most the 512 TMEM columns");
  constexpr int kABytes = 128 * kBKBytes;           // this CTA's 128 rows of A
  constexpr int kBSub = (SUBN / 2) * kBKBytes;      // this CTA's SUBN/2 rows of one sub-tile of B
  constexpr int kBBytes = NSUB * kBSub;
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr int kKElems = (KIND == 0) ? 128 : 64;
  constexpr int kAccs = (2 * BN <= 512) ? 2 : 1;  // accumulators in TMEM
  constexpr uint32_t kTmemCols = 512u;
  constexpr uint32_t kAccStride = 256u;
  constexpr int kPrefetch = 2 * STAGES;           // L2 prefetch distance for B, in K blocks
  constexpr int kChunks = BN / 32;                // 32-column epilogue chunks
  constexpr int kMyChunks = (kChunks + 1) / 2;    // per epilogue warp (two warps per quadrant)

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[kAccs];
  __shared__ __align__(8) uint64_t tempty_bar[kAccs];
  __shared__ __align__(8) uint64_t final_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int tile_prefix[kMaxExperts + 1];
  __shared__ int row_start[kMaxExperts + 1];

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  // epilogue: one 32 x 32 bf16 staging tile (2 KB) per warp for TMA stores,
  // and each warp's column scales
  uint8_t* sOut = smem + STAGES * kStageBytes;
  float* sWs = reinterpret_cast<float*>(sOut + 8 * 2048);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);   // leader: its producer's arrive + both CTAs' bytes
      mbar_init(&empty_bar[s], 1);  // one multicast commit per use
    }
    for (int a = 0; a < kAccs; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 16);  // leader: 8 epilogue warps x 2 CTAs
    }
    mbar_init(&final_bar, 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  // each CTA of the pair builds the same tile prefix from the device offsets
  pdl_wait();  // launched with programmatic stream serialization: global memory only after this
  // No early pdl_launch_dependents() here: this grid runs for milliseconds,
  // and the next kernel's CTAs parked beside it for that long cost the
  // power-capped large GEMM 1-3 % (measured); the next launch waits for
  // this grid's CTAs to exit, as without the trigger.
  if (threadIdx.x == 32 && p.offsets != nullptr) build_tile_prefix<256>(p, tile_prefix, row_start);
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_a) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_b) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_out) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int total = (p.offsets != nullptr) ? tile_prefix[p.E] : p.m_tiles * p.n_tiles;  // tiles of 256 x BN
  float qam = 0.0f;    // FP8 output: this thread's finite-only amax of the bf16 result (exact path)
  uint32_t qraw = 0;   // the same as the raw bits of the largest bf16 magnitude (fast path)

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pend_mask = 0, pend_parity = 0;
      bool stop = false;
      for (int t = cluster; t < total && !stop; t += nclusters) {
        const Tile T = decode_tile<256, BN>(t, p, tile_prefix, row_start);
        // rows past the tile's own (another expert's, or past M) only reach
        // accumulator rows that are never stored
        const int a_row = T.a_row + static_cast<int>(rank) * 128;
        const int b_row = T.b_row + static_cast<int>(rank) * (SUBN / 2);  // + SUBN per sub-tile
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { stop = true; break; }
          const uint32_t full_leader = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * kStageBytes);
          tma_load_2d_pair(sA + stage * kABytes, &tm_a, full_leader, kb * kKElems, a_row);
#pragma unroll
          for (int s = 0; s < NSUB; ++s)
            tma_load_2d_pair(sB + stage * kBBytes + s * kBSub, &tm_b, full_leader, kb * kKElems, b_row + SUBN * s);
          // The clusters that share this B tile run in step, so its DRAM
          // latency would stall all of them at once: ask L2 for the B tile
          // kPrefetch blocks ahead.
          if (kb + kPrefetch < p.nkb) {
#pragma unroll
            for (int s = 0; s < NSUB; ++s) tma_prefetch_2d(&tm_b, (kb + kPrefetch) * kKElems, b_row + SUBN * s);
          }
          pend_mask |= 1u << stage;
          pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (abort_flag && leader) {
        // the leader's full barriers also count the peer's bytes: drain them
        int dummy = 0;
        for (int s = 0; s < STAGES; ++s)
          if (pend_mask & (1u << s)) mbar_wait(&full_bar[s], (pend_parity >> s) & 1u, &dummy, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool issued = false;
      bool stop = false;
      int i = 0;
      for (int t = cluster; t < total && !stop; t += nclusters, ++i) {
        const int acc = i % kAccs;
        const uint32_t acc_phase = (i / kAccs) & 1;
        // the warp agrees on giving up a wait, so that no lane is left at a
        // warp-wide step after another has left
        if (__any_sync(0xFFFFFFFFu, !mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &abort_flag))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * kAccStride;
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (__any_sync(0xFFFFFFFFu, !mbar_wait(&full_bar[stage], phase, &abort_flag))) { stop = true; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint64_t ad = smem_desc(smem_u32(sA + stage * kABytes));
#pragma unroll
            for (int k = 0; k < kBKBytes / 32; ++k)
#pragma unroll
              for (int s = 0; s < NSUB; ++s) {
                const uint64_t bd = smem_desc(smem_u32(sB + stage * kBBytes + s * kBSub));
                mma_issue_pair<KIND>(d_tmem + static_cast<uint32_t>(SUBN * s), ad + 2u * k, bd + 2u * k, p.idesc,
                                     (kb > 0 || k > 0) ? 1u : 0u);
              }
            tc_commit_pair(&empty_bar[stage]);
            issued = true;
          }
          __syncwarp();
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (stop) break;
        if (lane == 0) tc_commit_pair(&tfull_bar[acc]);
        __syncwarp();
      }
      if (abort_flag && lane == 0 && issued) {
        int dummy = 0;
        tc_commit(&final_bar);
        mbar_wait(&final_bar, 0, &dummy, kDrainLimitNs);
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------------------- epilogue
    // Eight warps: warp w reads TMEM lane quadrant w % 4 (32 rows of this
    // CTA's half of the tile); the two warps of a quadrant take alternate
    // 32-column chunks.  Per chunk a warp scales, rounds to bf16 and stores
    // through a staging tile with one TMA store (clipped at M and N); a
    // 32-row group that straddles an expert boundary uses masked 16-byte
    // stores.
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;
    uint8_t* sb = sOut + ew * 2048;
    float* wsh = sWs + ew * kMyChunks * 32;
    const uint64_t out_pol = l2_evict_first_policy();
    const float qm = (p.qout != nullptr && p.qbs == nullptr) ? __ldcg(p.ring + p.ring_len) : 0.0f;  // the delayed multiplier
    const bool has_acc = p.nkb > 0;
    const uint16_t* bias = (KIND == 0) ? p.bias : nullptr;
    uint32_t tempty_leader[kAccs];
#pragma unroll
    for (int a = 0; a < kAccs; ++a) tempty_leader[a] = mapa_shared(smem_u32(&tempty_bar[a]), 0);
    int i = 0;
    for (int t = cluster; t < total; t += nclusters, ++i) {
      const int acc = i % kAccs;
      const uint32_t acc_phase = (i / kAccs) & 1;
      // The tile's row and column scales do not depend on the accumulator:
      // they are loaded before the wait, so their latency overlaps the
      // tile's main loop instead of adding to the epilogue (with one
      // 512-column accumulator the epilogue does not overlap the next tile).
      const Tile T = decode_tile<256, BN>(t, p, tile_prefix, row_start);
      const int row0 = T.row_lo + static_cast<int>(rank) * 128 + quad * 32;  // this warp's first row
      const int row = row0 + lane;
      const bool vrow = row < T.row_hi;
      // rows past M are clipped by the tensor map; rows of another expert are not
      const bool tma_ok = row0 < T.row_hi && (p.offsets == nullptr || row0 + 32 <= T.row_hi);
      float xsv = 0.0f;
      if (vrow) xsv = (KIND == 0) ? __ldg(p.xs + (p.xs_bcast ? 0 : row)) : 1.0f;
      float wpre[kMyChunks];
      {
        const float* wsp = p.ws + (p.ws_bcast ? 0 : static_cast<int64_t>(T.expert) * p.N);
#pragma unroll
        for (int j = 0; j < kMyChunks; ++j) {
          const int ch = half + 2 * j;
          const int n = T.col0 + ch * 32 + lane;
          wpre[j] = (KIND != 0) ? 1.0f
                                : ((ch < kChunks && n < p.N) ? __ldg(wsp + (p.ws_bcast ? 0 : n)) : 0.0f);
        }
      }
      // the warp agrees on giving up: the TMEM loads below are warp-wide
      if (__any_sync(0xFFFFFFFFu, !mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < kMyChunks; ++j) wsh[j * 32 + lane] = wpre[j];
      __syncwarp();
      uint16_t* orow = p.out + static_cast<int64_t>(vrow ? row : 0) * p.N;
      uint8_t* qrow = (KIND == 0 && p.qout != nullptr) ? p.qout + static_cast<int64_t>(vrow ? row : 0) * p.N : nullptr;
      float* qsrow = (KIND == 0 && p.qbs != nullptr) ? p.qbs + static_cast<int64_t>(vrow ? row : 0) * (p.N >> 5) : nullptr;
      epilogue_chunks<KIND, kChunks>(
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc) * kAccStride, half, lane,
          T.col0, p.N, T.col0 + BN, row0, vrow, tma_ok, has_acc, xsv, wsh, p, bias, orow, qrow, qsrow, qm, qraw, qam, sb, &tm_out,
          out_pol);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
    }
    if (lane == 0) bulk_wait_all();  // stores complete before the CTA's shared memory goes
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (KIND == 0 && p.qout != nullptr && p.qbs == nullptr)
    finalize_fp8_out<kGemmThreads / 32>(p, fmaxf(qam, __uint_as_float(qraw << 16)));
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

template <int KIND, int SUBN, int NSUB, int STAGES>
cudaError_t run2(const GemmArgs& a, std::string* msg) {
  constexpr int BN = SUBN * NSUB;
  constexpr int kElem = (KIND == 0) ? 1 : 2;
  constexpr int kSmem =
      STAGES * (128 + BN / 2) * kBKBytes + 8 * 2048 + 8 * ((BN / 32 + 1) / 2) * 32 * 4 + 1024;
  static_assert(kSmem + 8400 <= 232448, "shared memory over the 227 KB per-CTA limit");
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [] {
    attr_err =
        cudaFuncSetAttribute(k_gemm2<KIND, SUBN, NSUB, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(148, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, k_gemm2<KIND, SUBN, NSUB, STAGES>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      max_clusters = 0;
    }
  });
  if (attr_err != cudaSuccess) {
    *msg = "cudaFuncSetAttribute failed";
    return attr_err;
  }
  CUtensorMap ta, tb;
  memset(&ta, 0, sizeof(ta));
  memset(&tb, 0, sizeof(tb));
  if (a.K > 0) {
    if (!make_map(&ta, a.a, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), kElem, 128, msg) ||
        !make_map(&tb, a.b, static_cast<uint64_t>(a.E) * static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K),
                  kElem, SUBN / 2, msg))
      return cudaErrorInvalidValue;
  }
  CUtensorMap to;
  if (!make_result_map(&to, a, msg)) return cudaErrorInvalidValue;
  Params p;
  memset(&p, 0, sizeof(p));
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.nkb = static_cast<int>((a.K + (kBKBytes / kElem) - 1) / (kBKBytes / kElem));
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.m_tiles = static_cast<int>((a.M + 255) / 256);
  // Groups of 16 M-tiles (4096 rows): the group's A rows (32 MB at K = 8192)
  // stay in L2 while B streams past, so B is read once per 4096 rows.  At
  // M = 8192, N = 28672, K = 8192: DRAM 1371 MB per launch against 1780 MB
  // with groups of 8 and 2075 MB with groups of 32 (whose 64 MB of A no
  // longer stays), and 1-2 % faster.
  p.group_m = 16;
  p.E = a.E;
  p.offsets = a.offsets;
  p.xs = a.x_scale;
  p.xs_bcast = (a.x_scale_len == 1) ? 1 : 0;
  p.ws = a.w_scale;
  p.ws_bcast = (a.w_scale_len == 1) ? 1 : 0;
  p.out = static_cast<uint16_t*>(a.out);
  set_fused_epilogue(a, p);
  const uint32_t ab_fmt = (KIND == 0) ? static_cast<uint32_t>(a.fmt) : 1u;
  p.idesc = (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | (static_cast<uint32_t>(SUBN >> 3) << 17) |
            (static_cast<uint32_t>(256 >> 4) << 24);  // one MMA: M = 256 across the pair, N = SUBN
  int dev = 0;
  cudaGetDevice(&dev);
  int clusters = device_sm_count(dev) / 2;
  if (max_clusters > 0 && max_clusters < clusters) clusters = max_clusters;
  // grouped: the tile count lives on the device; a bound suffices
  const int64_t tiles = static_cast<int64_t>(p.m_tiles + (a.offsets != nullptr ? a.E : 0)) * p.n_tiles;
  if (tiles < clusters) clusters = static_cast<int>(tiles);
  if (clusters < 1) clusters = 1;
  return launch_pdl(k_gemm2<KIND, SUBN, NSUB, STAGES>, dim3(2 * clusters), dim3(kGemmThreads), kSmem, a.stream,
                    false, ta, tb, to, p);
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& a, std::string* msg) {
  // Wide tiles when there is enough work to fill the machine with them.
  // 256-wide tiles halve the A bytes per MMA cycle; worth a ragged last N
  // tile once N is large enough
  const bool wide = ((a.N % 256 == 0) && a.N >= 2048 && a.M >= 256) || (a.offsets != nullptr && a.N >= 1024);
  // Large dense GEMMs run on CTA pairs (256 x 256 tiles).  Below M = 4096
  // only with much work: for M = 1024 .. 3072 at K = 1024 .. 4096 the 1-CTA
  // 128 x 256 tiles measured 2-7 % faster (the pair's set-up and coarser
  // last round weigh more in a 15-40 us GEMM); at M = 2048, N = 28672,
  // K = 8192 the pair was 3 % faster.
  const bool pair = a.offsets == nullptr && a.kind == 0 && (a.N % 256 == 0) && a.N >= 2048 &&
                    (a.M >= 4096 || (a.M >= 512 && static_cast<double>(a.M) * a.N * a.K >= 137438953472.0));  // 2^37
  // 256 x 512 pair tiles read a quarter fewer operand bytes per flop; with
  // enough M their coarser last round costs little
  if (pair && a.N % 512 == 0 && a.M >= 8192) return run2<0, 256, 2, 4>(a, msg);
  if (pair) return run2<0, 256, 1, 6>(a, msg);
  // Grouped GEMMs with wide experts run on CTA pairs too: 256-row tiles per
  // expert, one third fewer operand bytes per flop than 128 x 256 tiles.
  if (a.offsets != nullptr && a.N >= 1024 && a.M >= 512) {
    if (a.kind == 0) return run2<0, 256, 1, 6>(a, msg);
    return run2<1, 256, 1, 6>(a, msg);
  }
  // Small M (decode): the weight stream from HBM is the bound, and each SM
  // streams at a roughly fixed rate, so the tile width is the narrowest that
  // keeps the most SMs busy in one round: 64 when N/64 tiles fit on the SMs,
  // else 128, else 208 (N <= 208 * SMs), else 256.  Only AROWS rows of A are
  // loaded per K block, which leaves shared memory for several K blocks of W
  // per stage (longer runs of each weight row per request).
  if (a.offsets == nullptr && a.kind == 0 && a.M <= 128) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int64_t sms = device_sm_count(dev);
    // (a block-wise FP8 output needs tiles that start on its 32-column
    // blocks: 256 instead of 208)
    const int bn = ((a.N + 63) / 64 <= sms)                              ? 64
                   : ((a.N + 127) / 128 <= sms)                          ? 128
                   : ((a.N + 207) / 208 <= sms && a.q_bscales == nullptr) ? 208
                                                                          : 256;
    if (a.M <= 16) {
      if (bn == 64) return run<0, 64, 2, 16, 8>(a, msg);
      if (bn == 128) return run<0, 128, 3, 16, 3>(a, msg);
      if (bn == 208) return run<0, 208, 3, 16, 2>(a, msg);
      return run<0, 256, 2, 16, 2>(a, msg);
    }
    if (a.M <= 64) {
      if (bn == 64) return run<0, 64, 3, 64, 4>(a, msg);
      if (bn == 128) return run<0, 128, 2, 64, 4>(a, msg);
      if (bn == 208) return run<0, 208, 2, 64, 2>(a, msg);
      return run<0, 256, 2, 64, 2>(a, msg);
    }
    if (bn == 64) return run<0, 64, 2, 128, 4>(a, msg);
    if (bn == 128) return run<0, 128, 3, 128, 2>(a, msg);
    if (bn == 208) return run<0, 208, 4, 128, 1>(a, msg);
    return run<0, 256, 4>(a, msg);
  }
  if (a.kind == 0) {
    if (wide) return run<0, 256, 4>(a, msg);
    return run<0, 128, 6>(a, msg);
  }
  if (wide) return run<1, 256, 4>(a, msg);
  return run<1, 128, 6>(a, msg);
}

unsigned* device_error_word() {
  static std::mutex mu;
  static unsigned* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) ptrs[dev] = static_cast<unsigned*>(p);
    else cudaGetLastError();
  }
  return ptrs[dev];
}

cudaError_t read_and_clear_device_error(unsigned* word) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  unsigned w = 0;
  e = cudaMemcpyFromSymbol(&w, g_device_error, sizeof(w));
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  *word = w;
  return e;
}

}  // namespace hq
