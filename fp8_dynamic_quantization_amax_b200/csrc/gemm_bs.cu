// gemm_bs.cu -- block-scaled FP8 GEMM on sm_100a tensor cores.
//
// out[m, n] = bf16_rn( sum_b xs[m, b] * ws[n, b] * S_b[m, n]  (+ bias[n]) ),
// S_b[m, n] = sum over the K block b of A[m, k] * B[n, k]
// (hip-quant README "Block-scaled Linear and Adafactor Kernel Helpers": the
// pre-quantized block-scaled linear consumes the FP8 bytes and FP32 per-block
// scales of both operands; "Block-wise FP8 Scaling": one dequant scale per
// block of block_size consecutive elements along the last dimension, scales
// [..., ceil(K / block_size)], the last block the short remainder).
//
// The block scales are arbitrary f32 values.  The tensor cores' block-scaled
// MMA applies power-of-two scale factors only, so the per-block sums are
// promoted in software, out of tensor memory.  Tiles are 128 x BN, BN = 256
// (128 for N <= 128):
//   warp 0      TMA producer: 128-byte K slices of A (128 rows) and B (BN
//               rows) into a ring of shared-memory stages (128B swizzle).
//   warp 1      allocates all 512 TMEM columns: 512 / BN FP32 accumulators of
//               BN columns, in slots of one block (BN = 256) or two (BN =
//               128).  One thread issues tcgen05.mma kind::f8f6f4, 32 K per
//               instruction, a stage's four back to back when blocks are
//               whole stages; all products of one scale block go to one
//               accumulator (the first overwrites it); a slot's blocks are
//               committed together, so the epilogue hands back a slot while
//               the other fills.  Blocks need not align with the 128-wide
//               stages.
//   promotion   BN / 16 warps (warps 2 ..), each owning 64 columns of one
//               TMEM lane quadrant: per slot, tcgen05.ld of each block's
//               partial sums, then acc += partial * (ws[n,b] * xs[m,b]) in
//               registers with packed f32x2 multiplies and fmas, and the
//               slot is handed back; after the last block, + bias, round to
//               bf16, 16-byte stores.
//   last warp   block-scale loader: per tile and chunk of 4 blocks, the
//               tile's 128 xs rows and BN ws rows (one 16-byte load per row
//               when nb % 4 == 0), written transposed ([block][row]) into a
//               ring of shared-memory slots.  The scales of a row are strided
//               by nb in memory, so a warp-wide load of one block's scales
//               touches 32 cache lines; loading 4 blocks per row once per CTA
//               (instead of per promotion warp and block) keeps the L1 load
//               pipe, which the per-warp loads saturated, out of the way.
// Consecutive MMAs into different TMEM accumulators do not overlap, and each
// scale block needs its own accumulator, so the wider tile does twice the
// MMA work per accumulator switch.
// Persistent CTAs, one per SM, tiles in groups of 8 M tiles.  Every wait is
// bounded: on a stalled barrier the CTA sets the device error word, drains
// what it has in flight, frees TMEM and exits.
#include "hq_internal.cuh"
#include "ptx.cuh"
#include "tc.cuh"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

namespace hq {
namespace {

constexpr int kBsM = 128;                            // tile rows (MMA M)
constexpr int kBsChunk = 4;                          // scale blocks per loader slot
constexpr int kBsScSlots = 4;                        // loader slots in flight
constexpr int kBsGroupM = 8;
constexpr uint32_t kBsTmemCols = 512;

// Tile width BN (MMA N) 128 or 256.  Every promotion warp owns 64 columns of
// one lane quadrant, so BN / 16 warps; the TMEM holds 512 / BN accumulators
// of BN columns, in slots of kGroup scale blocks.
template <int BN>
struct BsCfg {
  static constexpr int kEpiWarps = BN / 16;
  static constexpr int kLoaderWarp = 2 + kEpiWarps;
  static constexpr int kThreads = 32 * (kLoaderWarp + 1);       // TMA, MMA, promotion warps, scale loader
  static constexpr int kAcc = static_cast<int>(kBsTmemCols) / BN;
  static constexpr int kGroup = (kAcc >= 4) ? 2 : 1;
  static constexpr int kSlots = kAcc / kGroup;
  static constexpr int kStages = (BN == 128) ? 6 : 4;
  static constexpr int kLd = (BN == 128) ? 64 : 16;            // TMEM columns per load
  static constexpr int kABytes = kBsM * 128;                    // one 128-row x 128-byte K slice of A
  static constexpr int kBBytes = BN * 128;                      // one BN-row K slice of B
  static constexpr int kScFloats = kBsChunk * (kBsM + BN);      // a loader slot: xs [chunk][128], ws [chunk][BN]
  static constexpr int kSmem = kStages * (kABytes + kBBytes) + kBsScSlots * kScFloats * 4 + 1024;
  static_assert(BN == 128 || BN == 256, "tile widths 128 and 256");
  static_assert(kSmem + 1024 <= 232448, "shared memory over the per-CTA limit");
};

struct BsParams {
  int M, N, K;
  int nkb;               // 128-wide K stages
  int nks;               // 32-wide MMA K steps
  int spb;               // K steps per scale block
  int nb;                // scale blocks: ceil(K / block)
  int m_tiles, n_tiles;
  const float* xs;       // [M, nb]
  const float* ws;       // [N, nb]
  int sc_vec;            // 1: nb % 4 == 0 and both scale arrays 16-byte aligned (16-byte scale loads)
  const uint16_t* bias;  // bf16 [N] or null
  uint16_t* out;         // bf16 [M, N]
  uint32_t idesc;
  unsigned* err;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, unsigned* err,
                                         unsigned long long limit = ptx::kWaitLimitNs) {
  return ptx::mbar_wait(bar, parity, abort_flag, err, kDevErrTimeout, limit);
}

// (a0, a1) += (p0, p1) * ((w0, w1) * (x, x)): one packed multiply and one
// packed fma (FMUL2 / FFMA2), each IEEE round-to-nearest per lane.
__device__ __forceinline__ void promote2(float& a0, float& a1, uint32_t p0, uint32_t p1, float w0, float w1,
                                         float x) {
  const float2 r = __ffma2_rn(make_float2(__uint_as_float(p0), __uint_as_float(p1)),
                              __fmul2_rn(make_float2(w0, w1), make_float2(x, x)), make_float2(a0, a1));
  a0 = r.x;
  a1 = r.y;
}

// 32 TMEM lanes x N columns (16 or 64) of 32-bit in one load and its wait.
// No memory clobber: TMEM is not memory the compiler sees, so shared-memory
// loads may move across it; the volatile asm keeps its order against the
// tcgen05 fences, which are volatile asm too.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
               "tcgen05.wait::ld.sync.aligned;"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, uint32_t (&v)[64]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
               "tcgen05.wait::ld.sync.aligned;"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]), "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]), "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]), "=r"(v[48]), "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]), "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]), "=r"(v[63])
               : "r"(taddr));
}

template <int BN>
__device__ __forceinline__ void tile_coords(int t, const BsParams& p, int& m0, int& n0) {
  const int per_group = kBsGroupM * p.n_tiles;
  const int g = t / per_group;
  const int first_m = g * kBsGroupM;
  const int gsize = min(kBsGroupM, p.m_tiles - first_m);
  const int r = t - g * per_group;
  m0 = (first_m + r % gsize) * kBsM;
  n0 = (r / gsize) * BN;
}

template <int BN>
__global__ void __launch_bounds__(BsCfg<BN>::kThreads, 1)
    k_gemm_bs(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, const BsParams p) {
  using C = BsCfg<BN>;
  constexpr int kBsStages = C::kStages;
  constexpr int kBsSlots = C::kSlots;
  constexpr int kBsGroupBlocks = C::kGroup;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kBsStages];
  __shared__ __align__(8) uint64_t empty_bar[kBsStages];
  __shared__ __align__(8) uint64_t afull_bar[kBsSlots];
  __shared__ __align__(8) uint64_t aempty_bar[kBsSlots];
  __shared__ __align__(8) uint64_t sfull_bar[kBsScSlots];
  __shared__ __align__(8) uint64_t sempty_bar[kBsScSlots];
  __shared__ __align__(8) uint64_t final_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-byte aligned stages
  uint8_t* sA = smem;
  uint8_t* sB = smem + kBsStages * C::kABytes;
  // scale slots: [slot][xs: block of the chunk][128 rows], then [ws: block][BN columns]
  float* sSc = reinterpret_cast<float*>(smem + kBsStages * (C::kABytes + C::kBBytes));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBsStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < kBsSlots; ++a) {
      ptx::mbar_init(&afull_bar[a], 1);
      ptx::mbar_init(&aempty_bar[a], C::kEpiWarps);  // one arrive per promotion warp
    }
    for (int a = 0; a < kBsScSlots; ++a) {
      ptx::mbar_init(&sfull_bar[a], 1);   // the loader's lane 0
      ptx::mbar_init(&sempty_bar[a], C::kEpiWarps);  // one arrive per promotion warp
    }
    ptx::mbar_init(&final_bar, 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0 && p.nkb > 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_a) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_b) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kBsTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total = p.m_tiles * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_parity[kBsStages];
      bool armed[kBsStages];
#pragma unroll
      for (int s = 0; s < kBsStages; ++s) { armed[s] = false; armed_parity[s] = 0; }
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        int m0, n0;
        tile_coords<BN>(t, p, m0, n0);
        for (int kb = 0; kb < p.nkb; ++kb) {
          if (!wait_bar(&empty_bar[stage], phase ^ 1u, &abort_flag, p.err)) { stop = true; break; }
          ptx::mbar_arrive_expect_tx(&full_bar[stage], C::kABytes + C::kBBytes);
          tma_load_2d(sA + stage * C::kABytes, &tm_a, &full_bar[stage], kb * 128, m0);
          tma_load_2d(sB + stage * C::kBBytes, &tm_b, &full_bar[stage], kb * 128, n0);
#pragma unroll
          for (int s = 0; s < kBsStages; ++s)
            if (s == stage) { armed[s] = true; armed_parity[s] = phase; }
          if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (abort_flag) {  // every armed stage's last transfer lands before exit
#pragma unroll
        for (int s = 0; s < kBsStages; ++s) {
          int dummy = 0;
          if (armed[s]) wait_bar(&full_bar[s], armed_parity[s], &dummy, nullptr, ptx::kDrainLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    // Scale blocks go in groups of kBsGroupBlocks, each block into its own
    // accumulator of the group's slot.  Blocks of whole stages (block % 128
    // == 0): the warp waits per stage and one thread issues the stage's four
    // MMAs back to back, as the plain GEMM does; issuing them one K step at a
    // time with the bookkeeping in between measured 1.4-1.8x slower.
    if (p.spb % 4 == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t jg = 0;  // groups issued so far (the slot ring position)
      bool issued = false, stop = false;
      const int spbs = p.spb / 4;  // stages per block
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        int kb = 0;
        for (int b0 = 0; b0 < p.nb && !stop; b0 += kBsGroupBlocks, ++jg) {
          const uint32_t sl = jg % kBsSlots;
          const uint32_t sph = (jg / kBsSlots) & 1u;
          // the warp agrees on giving up, so that no lane is left at a warp-wide step
          if (__any_sync(0xFFFFFFFFu, !wait_bar(&aempty_bar[sl], sph ^ 1u, &abort_flag, p.err))) {
            stop = true;
            break;
          }
          tc_fence_after();
          for (int i = 0; i < kBsGroupBlocks && b0 + i < p.nb && !stop; ++i) {
            const uint32_t d_tmem = tmem_base + (sl * kBsGroupBlocks + i) * BN;
            const int kb_first = kb;
            const int kb_end = min(p.nkb, (b0 + i + 1) * spbs);
            for (; kb < kb_end; ++kb) {
              if (__any_sync(0xFFFFFFFFu, !wait_bar(&full_bar[stage], phase, &abort_flag, p.err))) {
                stop = true;
                break;
              }
              tc_fence_after();
              if (lane == 0) {
                const uint64_t ad = smem_desc(smem_u32(sA + stage * C::kABytes));
                const uint64_t bd = smem_desc(smem_u32(sB + stage * C::kBBytes));
                // K steps past K in the last stage read the zero fill
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_issue<0>(d_tmem, ad + 2u * k, bd + 2u * k, p.idesc, (kb > kb_first || k > 0) ? 1u : 0u);
                tc_commit(&empty_bar[stage]);
                issued = true;
              }
              __syncwarp();
              if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
            }
          }
          if (stop) break;
          if (lane == 0) tc_commit(&afull_bar[sl]);
          __syncwarp();
        }
      }
      if (abort_flag && lane == 0 && issued) {
        int dummy = 0;
        tc_commit(&final_bar);
        wait_bar(&final_bar, 0, &dummy, nullptr, ptx::kDrainLimitNs);
      }
    } else if ((p.spb == 1 || p.spb == 2) && lane == 0) {
      // Blocks of 32 or 64: a group of two blocks is 2 or 4 K steps inside
      // one stage; one thread issues them back to back.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t jg = 0;
      bool issued = false, stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        int ks = 0;
        for (int b0 = 0; b0 < p.nb && !stop; b0 += kBsGroupBlocks, ++jg) {
          const uint32_t sl = jg % kBsSlots;
          const uint32_t sph = (jg / kBsSlots) & 1u;
          if (!wait_bar(&aempty_bar[sl], sph ^ 1u, &abort_flag, p.err)) { stop = true; break; }
          tc_fence_after();
          if ((ks & 3) == 0) {  // the group opens a stage
            if (!wait_bar(&full_bar[stage], phase, &abort_flag, p.err)) { stop = true; break; }
            tc_fence_after();
          }
          const int nsteps = min(p.nks, (b0 + kBsGroupBlocks) * p.spb) - ks;  // 1 .. 4, one stage
          const uint64_t ad = smem_desc(smem_u32(sA + stage * C::kABytes));
          const uint64_t bd = smem_desc(smem_u32(sB + stage * C::kBBytes));
          const uint32_t d0 = tmem_base + sl * kBsGroupBlocks * BN;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q < nsteps) {
              const int kk = ks + q;
              const uint32_t blk = static_cast<uint32_t>(kk / p.spb - b0);  // 0 or 1 within the group
              mma_issue<0>(d0 + blk * BN, ad + 2u * (kk & 3), bd + 2u * (kk & 3), p.idesc,
                     (kk % p.spb != 0) ? 1u : 0u);
            }
          }
          issued = true;
          ks += nsteps;
          if ((ks & 3) == 0 || ks == p.nks) {  // the stage's last K step: hand the stage back
            tc_commit(&empty_bar[stage]);
            if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
          }
          tc_commit(&afull_bar[sl]);
        }
      }
      if (abort_flag && issued) {
        int dummy = 0;
        tc_commit(&final_bar);
        wait_bar(&final_bar, 0, &dummy, nullptr, ptx::kDrainLimitNs);
      }
    } else if (lane == 0) {
      // Blocks that split a stage: one thread walks the 32-wide K steps.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t jg = 0;  // groups issued so far (the slot ring position)
      bool issued = false, stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        int ks = 0;
        for (int b0 = 0; b0 < p.nb && !stop; b0 += kBsGroupBlocks, ++jg) {
          const uint32_t sl = jg % kBsSlots;
          const uint32_t sph = (jg / kBsSlots) & 1u;
          if (!wait_bar(&aempty_bar[sl], sph ^ 1u, &abort_flag, p.err)) { stop = true; break; }
          tc_fence_after();
          for (int i = 0; i < kBsGroupBlocks && b0 + i < p.nb && !stop; ++i) {
            const uint32_t d_tmem = tmem_base + (sl * kBsGroupBlocks + i) * BN;
            const int kfirst = ks;
            const int kend = min(p.nks, (b0 + i + 1) * p.spb);
            for (; ks < kend; ++ks) {
              const int sub = ks & 3;
              if (sub == 0) {
                if (!wait_bar(&full_bar[stage], phase, &abort_flag, p.err)) { stop = true; break; }
                tc_fence_after();
              }
              const uint64_t ad = smem_desc(smem_u32(sA + stage * C::kABytes));
              const uint64_t bd = smem_desc(smem_u32(sB + stage * C::kBBytes));
              mma_issue<0>(d_tmem, ad + 2u * sub, bd + 2u * sub, p.idesc, ks > kfirst ? 1u : 0u);
              issued = true;
              if (sub == 3 || ks == p.nks - 1) {  // the stage's last K step: hand the stage back
                tc_commit(&empty_bar[stage]);
                if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
              }
            }
          }
          if (stop) break;
          tc_commit(&afull_bar[sl]);
        }
      }
      if (abort_flag && issued) {
        int dummy = 0;
        tc_commit(&final_bar);
        wait_bar(&final_bar, 0, &dummy, nullptr, ptx::kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp < C::kLoaderWarp) {
    // -------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;
    uint32_t jg = 0;
    uint32_t cs = 0, cph = 0;  // scale slot ring position
    bool stop = false;
    for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
      int m0, n0;
      tile_coords<BN>(t, p, m0, n0);
      const int row = m0 + quad * 32 + lane;
      const bool vrow = row < p.M;
      const int c0 = n0 + half * 64;  // this warp's first column
      float acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
      const float* sc = sSc;  // the current chunk's slot
      for (int b0 = 0; b0 < p.nb && !stop; b0 += kBsGroupBlocks, ++jg) {
        const uint32_t sl = jg % kBsSlots;
        const uint32_t sph = (jg / kBsSlots) & 1u;
        // the warp agrees on giving up: the TMEM loads below are warp-wide
        if (__any_sync(0xFFFFFFFFu, !wait_bar(&afull_bar[sl], sph, &abort_flag, p.err))) {
          stop = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < kBsGroupBlocks; ++i) {
          const int b = b0 + i;
          if (b >= p.nb) break;
          const int bi = b % kBsChunk;
          if (bi == 0) {  // a chunk opens: its scales are in slot cs
            if (__any_sync(0xFFFFFFFFu, !wait_bar(&sfull_bar[cs], cph, &abort_flag, p.err))) {
              stop = true;
              break;
            }
            sc = sSc + cs * C::kScFloats;
          }
          const float xb = sc[bi * kBsM + quad * 32 + lane];
          const float* wrow = sc + kBsChunk * kBsM + bi * BN + half * 64;
          const uint32_t tcol = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                (sl * kBsGroupBlocks + i) * BN + static_cast<uint32_t>(half * 64);
          // the 64 columns in TMEM loads of kLd columns (fewer registers in
          // flight where the CTA has more warps and so fewer registers each)
#pragma unroll
          for (int e0 = 0; e0 < 64; e0 += C::kLd) {
            uint32_t v[C::kLd];
            tmem_ld_cols(tcol + static_cast<uint32_t>(e0), v);
#pragma unroll
            for (int e = 0; e < C::kLd; e += 4) {
              const float4 w = *reinterpret_cast<const float4*>(wrow + e0 + e);
              promote2(acc[e0 + e], acc[e0 + e + 1], v[e], v[e + 1], w.x, w.y, xb);
              promote2(acc[e0 + e + 2], acc[e0 + e + 3], v[e + 2], v[e + 3], w.z, w.w, xb);
            }
          }
          if (bi == kBsChunk - 1 || b == p.nb - 1) {  // the chunk's last block: hand its slot back
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sempty_bar[cs]);
            if (++cs == kBsScSlots) { cs = 0; cph ^= 1u; }
          }
        }
        if (stop) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&aempty_bar[sl]);
      }
      if (stop) break;
      if (vrow) {
        uint16_t* orow = p.out + static_cast<int64_t>(row) * p.N;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int n = c0 + g * 8;
          if (n >= p.N) break;  // N % 8 == 0: a group of 8 is inside or outside
          float o[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) o[k] = acc[g * 8 + k];
          if (p.bias) {
            const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
            const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              o[2 * k] = __fadd_rn(o[2 * k], __uint_as_float(bw[k] << 16));
              o[2 * k + 1] = __fadd_rn(o[2 * k + 1], __uint_as_float(bw[k] & 0xFFFF0000u));
            }
          }
          const uint4 st = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                      pack_bf16x2(o[6], o[7]));
          *reinterpret_cast<uint4*>(orow + n) = st;
        }
      }
    }
  } else {
    // ------------------------------------------------------ scale loader
    // Lane l fills rows l, l + 32, l + 64, l + 96 of the tile: xs of those
    // rows and ws of those columns, kBsChunk blocks each; rows past M or N
    // and blocks past nb read as zero.
    uint32_t cs = 0, cph = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
      int m0, n0;
      tile_coords<BN>(t, p, m0, n0);
      for (int b0 = 0; b0 < p.nb; b0 += kBsChunk) {
        if (__any_sync(0xFFFFFFFFu, !wait_bar(&sempty_bar[cs], cph ^ 1u, &abort_flag, p.err))) {
          stop = true;
          break;
        }
        float* sx = sSc + cs * C::kScFloats;
        float* sw = sx + kBsChunk * kBsM;
        // kBsChunk scales of one row of xs (rows = M) or ws (rows = N), transposed
        // into dst[block][r]; rows past the matrix and blocks past nb read as zero
        auto stage_row = [&](const float* base, int row, int rows, float* dst, int stride, int r) {
          float v[kBsChunk];
          const bool in = row < rows;
          const float* src = base + static_cast<int64_t>(in ? row : 0) * p.nb + b0;
          if (p.sc_vec) {  // b0 + 4 <= nb
            const float4 f4 = __ldg(reinterpret_cast<const float4*>(src));
            v[0] = f4.x; v[1] = f4.y; v[2] = f4.z; v[3] = f4.w;
          } else {
#pragma unroll
            for (int i = 0; i < kBsChunk; ++i) v[i] = (b0 + i < p.nb) ? __ldg(src + i) : 0.0f;
          }
#pragma unroll
          for (int i = 0; i < kBsChunk; ++i) dst[i * stride + r] = in ? v[i] : 0.0f;
        };
#pragma unroll
        for (int j = 0; j < kBsM / 32; ++j) stage_row(p.xs, m0 + lane + 32 * j, p.M, sx, kBsM, lane + 32 * j);
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) stage_row(p.ws, n0 + lane + 32 * j, p.N, sw, BN, lane + 32 * j);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sfull_bar[cs]);  // releases the lanes' stores to the epilogue
        if (++cs == kBsScSlots) { cs = 0; cph ^= 1u; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kBsTmemCols)
                 : "memory");
  }
}

// --------------------------------------------------------------- host side
template <int BN>
cudaError_t run_bs(const BlockScaledGemmArgs& a, std::string* msg) {
  using C = BsCfg<BN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_gemm_bs<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (attr_err != cudaSuccess) {
    *msg = "cudaFuncSetAttribute failed";
    return attr_err;
  }
  unsigned* err = device_error_word();
  if (err == nullptr) {
    *msg = "the device error word is not available";
    return cudaErrorUnknown;
  }
  CUtensorMap ta, tb;
  memset(&ta, 0, sizeof(ta));
  memset(&tb, 0, sizeof(tb));
  if (a.K > 0) {  // K == 0: no loads are issued and the maps are never read
    if (!make_map(&ta, a.a, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), 1, kBsM, msg) ||
        !make_map(&tb, a.b, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K), 1, BN, msg))
      return cudaErrorInvalidValue;
  }
  BsParams p;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.nkb = static_cast<int>((a.K + 127) / 128);
  p.nks = static_cast<int>((a.K + 31) / 32);
  p.spb = static_cast<int>(a.block / 32);
  p.nb = static_cast<int>((a.K + a.block - 1) / a.block);
  p.m_tiles = static_cast<int>((a.M + kBsM - 1) / kBsM);
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.xs = a.x_scales;
  p.ws = a.w_scales;
  p.sc_vec = (p.nb % 4 == 0 && reinterpret_cast<uintptr_t>(a.x_scales) % 16 == 0 &&
              reinterpret_cast<uintptr_t>(a.w_scales) % 16 == 0)
                 ? 1
                 : 0;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out);
  p.idesc = (1u << 4)                                         // D: FP32
            | (static_cast<uint32_t>(a.fmt) << 7) | (static_cast<uint32_t>(a.fmt) << 10)  // E4M3 / E5M2
            | (static_cast<uint32_t>(BN >> 3) << 17)            // N / 8
            | (static_cast<uint32_t>(kBsM >> 4) << 24);         // M / 16
  p.err = err;
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  const int sms = device_sm_count(dev);
  const int grid = static_cast<int>(tiles < sms ? (tiles < 1 ? 1 : tiles) : sms);
  k_gemm_bs<BN><<<grid, C::kThreads, C::kSmem, a.stream>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_blockscaled(const BlockScaledGemmArgs& a, std::string* msg) {
  // 128 x 256 tiles do twice the MMA work per accumulator switch of 128 x
  // 128 tiles (the large layer: 1233 against 888 TF/s at blocks of 128, 575
  // against 475 at 64, equal at 32); the narrow form serves N <= 128
  return (a.N <= 128) ? run_bs<128>(a, msg) : run_bs<256>(a, msg);
}

}  // namespace hq
