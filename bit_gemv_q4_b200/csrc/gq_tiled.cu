// gq_tiled.cu -- tiled storage of packed weights and the batch-1 GEMV that
// streams it.
//
// Operation: the matrix multiply that consumes decoded blocks ("GGUF 量化内幕
// 第4章" 4.3: w = d * (code - 8); "GGUF K-quants" 套娃, step 5: s~_j = S * q_j),
// y[m] = sum_k W_hat[m][k] * x[k], in the decode setting where the weight
// stream sets the speed (TurboQuant W4A8 post, section 2.3).
//
// Tiled storage (layout in include/gq.h) is a byte permutation of the
// canonical rows, made once (gq_repack_*): every tile of 16 rows x 64 Q4_0
// blocks (16 rows x 8 super-blocks) is contiguous and ordered by the lanes
// that multiply it, so that
//   * one bulk copy moves a whole pipeline stage.  On B200 the copy engine
//     spends about 55 ns on each small copy: the canonical layout needs one
//     copy per row and stage (sixteen 1.15 KB copies), which holds a single
//     launch near 1.7 TB/s, while one 18 KB copy per stage streams at the
//     HBM rate;
//   * each lane reads its code words as 16-byte aligned, bank-conflict-free
//     shared loads, with no byte permutes, and its row's scales as one word.
//
// Launch shape.  In a chain of GEMVs joined by programmatic dependent launch,
// launch i+1 may stream its weights early but may read x only once launch i
// has finished, so its arithmetic sits on the critical path after that
// point.  The kernel keeps its footprint to half an SM (one CTA per SM, at
// most 113 KB of shared memory, 544 threads x 56 registers) so that the next
// launch's CTA is resident while this one computes, and while its grid
// dependency is pending it stages its share on chip: the producer warp fills
// a 4-stage shared-memory ring, and the consumer warps move the first stages
// out of the ring into tensor memory (64 columns per warp, 6 stages, as the
// 32-bit words each lane uses) so that the ring can take later stages.
// Shared plus tensor memory hold 10 stages, about 180 KB per CTA.
//
// Arithmetic.  Codes enter a warp MMA m16n8k16 as fp16 subnormals: a 4-bit
// code c in the low bits of a half is exactly c * 2^-24, one at bits 4-7 is
// c * 2^-20 (the binary16 subnormal encoding), so a nibble mask is the whole
// decode.  The low nibbles of a block (weights 0-15) and the high nibbles
// (16-31) go to two MMAs with zero accumulators, and
// s = C_lo + C_hi / 16 - 8 * 2^-24 * sum(x over the block)
//   = 2^-24 * sum_k (c_k - 8) x_k.
// Products are exact; the MMA's fp32 accumulation and the fp32 sums round.
// The block scale multiplies s in fp32 (d for Q4_0; q_j, then S, for
// super-blocks) and the row sum is scaled by 2^24 at the end (exact).  Each
// warp keeps its share of a row in registers and leaves it in a shared
// table; the shares of a batch of row groups are added at one barrier.
//
// Grouped form (gq_gemv_*_tiled_grouped).  Many tiled matrices that share K
// and x go into one launch: their row groups are numbered back to back and a
// table passed by value maps a group to its matrix.  A group's arithmetic
// does not depend on the CTA that takes it, so each output equals the
// single-matrix call's bit for bit.  This launch puts two CTAs on each SM
// and always stages the first tiles in tensor memory, which measured fastest
// on long grouped streams.
//
// Every wait is bounded (kWaitBudget cycles); on expiry the kernel ORs
// GQ_DEV_TIMEOUT into the status word, lets its copies land, releases its
// tensor memory and exits.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_host.h"
#include "gq_tc.cuh"

namespace gq {
namespace {

#ifndef GQ_TILED_CONS
#define GQ_TILED_CONS 16
#endif

constexpr int kRows = 16;
constexpr int kCons = GQ_TILED_CONS;           // consumer warps (warps 1..kCons)
constexpr int kThreads = 32 * (1 + kCons);
constexpr int kRing = 4;                       // shared-memory stages
static_assert((kRing & (kRing - 1)) == 0, "ring slots are taken as j & (kRing - 1)");
constexpr int kStageBytes = 18432;             // a full Q4_0 tile; a ksb tile is 17664
constexpr int kStageWords = 160 / kCons;       // words per lane, warp and stage (10 or 20)
constexpr int kWordsA = kStageWords >= 16 ? 16 : 8;   // stash words of a stage in column block A
constexpr int kWordsB = kStageWords - kWordsA;        // ... and in column block B
constexpr int kStashMax = 6;                   // stashed stages per warp
constexpr int kColsA = kStashMax * kWordsA;
constexpr int kTmemCols = 256;                 // per CTA
constexpr int kStashCols = kTmemCols * 4 / kCons;  // per warp (kCons / 4 warps per lane quadrant)
constexpr int kSiblings = kCons / 4;           // warps per lane quadrant
constexpr int kMaxKb = 512;                    // x blocks of 32: K <= 16384
static_assert(kCons == 8 || kCons == 16, "consumer warps");
static_assert(kColsA + kStashMax * kWordsB <= kStashCols, "stash layout");

template <int FMT>
struct Tile;
template <>
struct Tile<GQ_FMT_Q4_0> {
  static constexpr int kBlkB = 18;          // bytes per block of 32 weights
  static constexpr int kPerTile = 64;       // blocks per row in a full tile
  static constexpr int kTileBytes = 18432;  // 16 rows x 64 blocks
  static constexpr int kUnitBlk = 2;        // a unit is a pair of blocks
  static constexpr int kUnitWords = 5;
  static constexpr int kUnitBytes = 512;    // code bytes of a unit
};
template <>
struct Tile<GQ_FMT_KSB> {
  static constexpr int kBlkB = 138;         // bytes per super-block of 256 weights
  static constexpr int kPerTile = 8;
  static constexpr int kTileBytes = 17664;
  static constexpr int kUnitBlk = 4;        // a unit is half a super-block: four sub-blocks
  static constexpr int kUnitWords = 10;
  static constexpr int kUnitBytes = 1024;
};
// units per warp in a full tile (every tile holds 64 blocks of 32 weights)
template <int FMT>
__host__ __device__ constexpr int units_w() { return 64 / Tile<FMT>::kUnitBlk / kCons; }
static_assert(units_w<GQ_FMT_Q4_0>() * Tile<GQ_FMT_Q4_0>::kUnitWords == kStageWords, "");
static_assert(units_w<GQ_FMT_KSB>() * Tile<GQ_FMT_KSB>::kUnitWords == kStageWords, "");

struct TArgs {
  const uint8_t* T;  // tiled storage
  const __half* x;
  void* y;
  int* dev_status;
  long long budget;
  int64_t M;
  int64_t group_bytes;  // 16 * canonical row bytes
  int K, ytype;
  int nblk;     // blocks (Q4_0) or super-blocks (KSB) per row
  int ntiles;   // tiles (stages) per row group
  int ngroups;  // row groups of 16
  int stash;    // most stages a CTA moves to tensor memory (0: none)
  int tgroups;  // row groups the partial-sum table holds
  uint32_t xf_off, xc_off, tab_off, bar_off;  // shared-memory layout
};

// Several matrices in one launch (they share K and x): their 16-row groups
// are numbered one after the other, matrix i owning groups [gend[i-1],
// gend[i]).  Passed by value, read from the kernel parameter space.
constexpr int kMaxTiledMats = 256;
struct TiledMat {
  const uint8_t* T;
  void* y;
  int64_t M;
  int gend;
  int pad;
};
struct TiledTable {
  TiledMat m[kMaxTiledMats];
};
struct OneMatrix {  // the single-matrix form: everything is in TArgs
  int unused;
};

// Where row group g lives: its tiles, its outputs, and its group within its
// matrix.  Each caller visits groups in increasing order, so the cursor mi
// only moves forward.
struct GroupAt {
  const uint8_t* T;
  void* y;
  int64_t M, lg;
};
template <class Tbl>
__device__ __forceinline__ GroupAt group_at(const TArgs& a, const Tbl& tbl, int64_t g, int& mi) {
  if constexpr (sizeof(Tbl) == sizeof(OneMatrix)) {
    return GroupAt{a.T, a.y, a.M, g};
  } else {
    while (g >= tbl.m[mi].gend) ++mi;
    const int gb = mi ? tbl.m[mi - 1].gend : 0;
    return GroupAt{tbl.m[mi].T, tbl.m[mi].y, tbl.m[mi].M, g - gb};
  }
}

extern __shared__ __align__(1024) uint8_t smem[];

__device__ __forceinline__ uint32_t ld32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}
__device__ __forceinline__ uint32_t ld16(uint32_t off) {
  return *reinterpret_cast<const uint16_t*>(smem + off);
}
__device__ __forceinline__ uint4 ld128(uint32_t off) {
  return *reinterpret_cast<const uint4*>(smem + off);
}

// ------------------------------------------------------------------ decode
// One block of 32 weights for rows g (wa = this lane's code word of the
// block) and g+8 (wb): two MMAs with zero accumulator input, then
// C_lo + C_hi / 16 for the row this lane accumulates (g for lanes t = 0, 1;
// g+8 for t = 2, 3).  xv: the block's B fragment for lane group t.  The
// caller adds the block's correction -8 * 2^-24 * sum(x over the block).
__device__ __forceinline__ float block_dot(uint32_t wa, uint32_t wb, uint4 xv, bool hi_row) {
  const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
  float cl[4], ch[4];
  mma_f16_z(cl, wa & 0x000F000Fu, wb & 0x000F000Fu, wa8 & 0x000F000Fu, wb8 & 0x000F000Fu, xv.x,
            xv.y);
  mma_f16_z(ch, wa & 0x00F000F0u, wb & 0x00F000F0u, wa8 & 0x00F000F0u, wb8 & 0x00F000F0u, xv.z,
            xv.w);
  const float lo = hi_row ? cl[2] : cl[0];
  const float hi = hi_row ? ch[2] : ch[0];
  return fmaf(hi, 0.0625f, lo);
}

// Non-negative INT8 sub-scale in byte h of q as a float (exact).
__device__ __forceinline__ float byte_to_float(uint32_t q, int h) {
  return __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7540u + h)) - 8388608.0f;
}

// The two fp16 values of a 32-bit word as floats (exact).
__device__ __forceinline__ float2 halves(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// --------------------------------------------------------- tile extraction
// Unit i of warp cw is unit u = cw + kCons * i of the tile.  Q4_0 unit:
// [code g, code g+8 of block 2u, of block 2u+1, the two scales of row ro];
// KSB unit (sub-blocks 4 (u % 2) .. +3 of super-block u / 2): [code g, code
// g+8] of each sub-block, row ro's four INT8 sub-scales, its super-scale S.
// Per-lane offsets inside a tile (for unit i add i * kCons times the unit's
// stride): codes at code_off, the lane's row's scales at scale_off (plus the
// scale section's base, 256 nb or 2048 nb), S at s_off (plus 2176 nb).
struct LaneOffs {
  uint32_t code_off, scale_off, s_off;
};
template <int FMT>
__device__ __forceinline__ LaneOffs lane_offs(int cw, int lane, int ro) {
  using F = Tile<FMT>;
  return LaneOffs{static_cast<uint32_t>(F::kUnitBytes * cw + (FMT == GQ_FMT_Q4_0 ? 16 : 32) * lane),
                  static_cast<uint32_t>(64 * cw + 4 * ro),
                  static_cast<uint32_t>(32 * (cw >> 1) + 2 * ro)};
}

// The words of one unit (i) of a tile at shared offset st with nb blocks
// (Q4_0) or super-blocks (KSB).
template <int FMT>
__device__ __forceinline__ void unit_words(uint32_t st, int nb, const LaneOffs& f, int i,
                                           uint32_t* w) {
  using F = Tile<FMT>;
  const uint32_t cofs = st + f.code_off + i * kCons * F::kUnitBytes;
  const uint4 c0 = ld128(cofs);
  w[0] = c0.x;
  w[1] = c0.y;
  w[2] = c0.z;
  w[3] = c0.w;
  if constexpr (FMT == GQ_FMT_Q4_0) {
    w[4] = ld32(st + 256 * nb + f.scale_off + i * kCons * 64);
  } else {
    const uint4 c1 = ld128(cofs + 16);
    w[4] = c1.x;
    w[5] = c1.y;
    w[6] = c1.z;
    w[7] = c1.w;
    w[8] = ld32(st + 2048 * nb + f.scale_off + i * kCons * 64);
    w[9] = ld16(st + 2176 * nb + f.s_off + i * kCons * 16);
  }
}

template <int FMT, bool FULL>
__device__ __forceinline__ void tile_words(uint32_t st, int nb, int cw, const LaneOffs& f,
                                           uint32_t* w) {
  using F = Tile<FMT>;
#pragma unroll
  for (int i = 0; i < units_w<FMT>(); ++i) {
    if (FULL || (cw + kCons * i) * F::kUnitBlk < nb * (FMT == GQ_FMT_Q4_0 ? 1 : 8))
      unit_words<FMT>(st, FULL ? F::kPerTile : nb, f, i, w + F::kUnitWords * i);
  }
}

// ------------------------------------------------------------- stage math
// Accumulate one stage of warp cw from its words: acc[] += scale * s over its
// blocks (two accumulators, alternating, so that the scale FMAs do not form
// one long chain).  xb / cb: shared offsets of the warp's first x fragment /
// block correction in this tile (lane group t included).
template <int FMT, bool FULL>
__device__ __forceinline__ void stage_math(const uint32_t* w, float* acc, uint32_t xb, uint32_t cb,
                                           int cw, int nb, bool hi_row) {
  using F = Tile<FMT>;
#pragma unroll
  for (int i = 0; i < units_w<FMT>(); ++i) {
    if (!(FULL || (cw + kCons * i) * F::kUnitBlk < nb * (FMT == GQ_FMT_Q4_0 ? 1 : 8))) continue;
    const uint32_t xo = xb + i * kCons * F::kUnitBlk * 64, co = cb + i * kCons * F::kUnitBlk * 4;
    const uint32_t* v = w + F::kUnitWords * i;
    if constexpr (FMT == GQ_FMT_Q4_0) {
      const uint4 x0 = ld128(xo), x1 = ld128(xo + 64);
      const float2 cx = *reinterpret_cast<const float2*>(smem + co);
      const float2 d = halves(v[4]);
      const float s0 = block_dot(v[0], v[1], x0, hi_row) + cx.x;
      const float s1 = block_dot(v[2], v[3], x1, hi_row) + cx.y;
      acc[0] = fmaf(d.x, s0, acc[0]);
      acc[1] = fmaf(d.y, s1, acc[1]);
    } else {
      const float4 c4 = *reinterpret_cast<const float4*>(smem + co);
      const uint4 x0 = ld128(xo), x1 = ld128(xo + 64), x2 = ld128(xo + 128), x3 = ld128(xo + 192);
      const float s0 = block_dot(v[0], v[1], x0, hi_row) + c4.x;
      const float s1 = block_dot(v[2], v[3], x1, hi_row) + c4.y;
      const float s2 = block_dot(v[4], v[5], x2, hi_row) + c4.z;
      const float s3 = block_dot(v[6], v[7], x3, hi_row) + c4.w;
      const float p0 = fmaf(byte_to_float(v[8], 1), s1, byte_to_float(v[8], 0) * s0);
      const float p1 = fmaf(byte_to_float(v[8], 3), s3, byte_to_float(v[8], 2) * s2);
      acc[i & 1] = fmaf(halves(v[9]).x, p0 + p1, acc[i & 1]);
    }
  }
}

// ------------------------------------------------------------- x fragments
// After the grid dependency: the B fragments of every x block this warp uses
// (for lane group t, 16 bytes: x[4t], x[4t+2], x[4t+1], x[4t+3], then the
// same at +16) and -8 * 2^-24 * (sum of the block's 32 values).  A warp uses
// 64 / kCons blocks of 32 per tile; a lane moves 8 consecutive values of one.
template <int FMT>
__device__ __forceinline__ void load_x(const TArgs& a, int cw, int lane) {
  using F = Tile<FMT>;
  constexpr int kLanesPerTile = 4 * (64 / kCons);     // 32 or 16
  constexpr int kTilesPerRound = 32 / kLanesPerTile;  // 1 or 2
  constexpr int kRounds = 8 / kTilesPerRound;         // 8 tiles: K <= 16384
  const int sub = lane / kLanesPerTile;
  const int lb = (lane % kLanesPerTile) >> 2, q = lane & 3;
  const int i = lb / F::kUnitBlk, h = lb % F::kUnitBlk;
  const int xoff = F::kUnitBlk * (cw + kCons * i) + h;  // x block of this lane in its tile
  const int nkb = a.K / 32;
  const uint4* src = reinterpret_cast<const uint4*>(a.x);
  constexpr int kBatch = 4;  // loads in flight per lane
#pragma unroll
  for (int r0 = 0; r0 < kRounds; r0 += kBatch) {
    uint4 raw[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int kb = ((r0 + r) * kTilesPerRound + sub) * 64 + xoff;
      if (r0 + r < kRounds && kb < nkb) raw[r] = src[kb * 4 + q];
    }
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int kb = ((r0 + r) * kTilesPerRound + sub) * 64 + xoff;
      const bool ok = r0 + r < kRounds && kb < nkb;
      float part = 0.f;
      if (ok) {
        const uint4 u = raw[r];
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
        const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
        part = ((f0.x + f0.y) + (f1.x + f1.y)) + ((f2.x + f2.y) + (f3.x + f3.y));
        // values 8q .. 8q+7 of the block: lane groups t0 and t0+1, half hi
        const int t0 = 2 * (q & 1), hi = q >> 1;
        const uint32_t d = a.xf_off + kb * 64 + hi * 8;
        *reinterpret_cast<uint2*>(smem + d + t0 * 16) =
            make_uint2(__byte_perm(u.x, u.y, 0x5410u), __byte_perm(u.x, u.y, 0x7632u));
        *reinterpret_cast<uint2*>(smem + d + (t0 + 1) * 16) =
            make_uint2(__byte_perm(u.z, u.w, 0x5410u), __byte_perm(u.z, u.w, 0x7632u));
      }
      part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
      part += __shfl_xor_sync(0xFFFFFFFFu, part, 2);
      if (ok && q == 0)
        *reinterpret_cast<float*>(smem + a.xc_off + kb * 4) = part * -4.76837158203125e-07f;  // -8 * 2^-24
    }
  }
}

// tensor memory: stash stage j of a warp at columns kWordsA * j (block A) and
// kColsA + kWordsB * j (block B) of its column range
__device__ __forceinline__ void stash_store(uint32_t tq, int j, const uint32_t* w) {
  if constexpr (kWordsA == 16) tmem_st16(tq + kWordsA * j, w);
  else tmem_st8(tq + kWordsA * j, w);
  if constexpr (kWordsB == 4) tmem_st4(tq + kColsA + kWordsB * j, w + kWordsA);
  else tmem_st2(tq + kColsA + kWordsB * j, w + kWordsA);
}
__device__ __forceinline__ void stash_load(uint32_t tq, int j, uint32_t* w) {
  if constexpr (kWordsA == 16) tmem_ld16(tq + kWordsA * j, w);
  else tmem_ld8(tq + kWordsA * j, w);
  if constexpr (kWordsB == 4) tmem_ld4(tq + kColsA + kWordsB * j, w + kWordsA);
  else tmem_ld2(tq + kColsA + kWordsB * j, w + kWordsA);
}

// ------------------------------------------------------------------ kernel
// Waits off the critical path (before the grid dependency resolves) let the
// warp sleep between tests, so that it takes no issue slots from the
// co-resident launch that is computing.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(2000u)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, long long budget) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(n)
               : "memory");
}

template <int FMT, class Tbl>
__global__ void __launch_bounds__(kThreads, 2) gemv_tiled_kernel(const TArgs a, const Tbl tbl) {
  using F = Tile<FMT>;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  uint64_t* empty = full + kRing;
  uint64_t* red_bar = empty + kRing;
  uint64_t* done_bar = red_bar + 1;
  uint64_t* stash_bar = done_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stash_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    mbar_init(red_bar, kCons);
    mbar_init(done_bar, kCons);
    mbar_init(stash_bar, 4);
    fence_barrier_init();
  }
  if (warp == 1 && a.stash) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();

  // This CTA's row groups g = blockIdx.x + i * gridDim.x; stage j is tile
  // j % ntiles of group i = j / ntiles.  Stages [0, nstash) go through tensor
  // memory, the rest through the ring.
  const int nwhole = (a.ngroups - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);
  const int ns = nwhole * a.ntiles;
  auto stage_tile = [&](int j, int64_t& g, int& c) {  // stage j -> (row group, tile)
    g = blockIdx.x + static_cast<int64_t>(j / a.ntiles) * gridDim.x;
    c = j % a.ntiles;
  };
  const int nstash = a.stash ? min(a.stash, max(0, ns - kRing)) : 0;
  const int last_nb = a.nblk - (a.ntiles - 1) * F::kPerTile;  // blocks in a row's last tile

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      bool ok = true;
      int s = 0, pmi = 0;
      uint32_t ph = 0;
      for (int j = 0; j < ns; ++j) {
        if (!mbar_wait(&empty[s], ph ^ 1u, a.budget)) {
          ok = false;
          break;
        }
        int64_t g;
        int c;
        stage_tile(j, g, c);
        const GroupAt at = group_at(a, tbl, g, pmi);
        const int nb = (c == a.ntiles - 1) ? last_nb : F::kPerTile;
        const uint32_t bytes = static_cast<uint32_t>(nb * kRows * F::kBlkB);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(smem + s * kStageBytes,
                 at.T + at.lg * a.group_bytes + static_cast<int64_t>(c) * F::kTileBytes, bytes,
                 &full[s], pol);
        ++issued;
        if (++s == kRing) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) report(a.dev_status, GQ_DEV_TIMEOUT);
      // every issued copy lands before the CTA's shared memory is released
      for (int u = max(0, issued - kRing); u < issued; ++u) {
        if (!mbar_wait(&full[u % kRing], static_cast<uint32_t>(u / kRing) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int g8 = lane >> 2, t = lane & 3;
  const bool hi_row = t >= 2;
  const int ro = g8 + (hi_row ? 8 : 0);
  const uint32_t tbase = a.stash ? *reinterpret_cast<volatile uint32_t*>(tmem_slot) : 0u;
  const uint32_t tlane = (32u * static_cast<uint32_t>(warp & 3)) << 16;
  const uint32_t tq = tbase + tlane + static_cast<uint32_t>(cw >> 2) * kStashCols;
  bool ok = true;

  // ---- before the grid dependency: warps 1..4 (one per lane quadrant) move
  // the first stages out of the ring into tensor memory, for themselves and
  // their sibling warps of the same quadrant (warps cw + 4k)
  if (cw < 4 && nstash) {
    for (int j = 0; j < nstash; ++j) {
      const int s = j % kRing;
      // every lane takes the same branch before the warp-wide tensor-memory stores
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_sleep(&full[s], (j / kRing) & 1u, a.budget))) {
        ok = false;
        break;
      }
      int64_t g_unused;
      int c;
      stage_tile(j, g_unused, c);
      const int nb = (c == a.ntiles - 1) ? last_nb : F::kPerTile;
#pragma unroll 1
      for (int k = 0; k < kSiblings; ++k) {
        const int sw = cw + 4 * k;  // the sibling warp's consumer index
        uint32_t w[kStageWords];
#pragma unroll
        for (int i = 0; i < kStageWords; ++i) w[i] = 0u;
        const LaneOffs f = lane_offs<FMT>(sw, lane, ro);
        tile_words<FMT, false>(static_cast<uint32_t>(s * kStageBytes), nb, sw, f, w);
        stash_store(tbase + tlane + static_cast<uint32_t>(k) * kStashCols, j, w);
      }
      tmem_wait_st();
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&empty[s], kSiblings);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(stash_bar);
  }

  pdl_wait();  // the preceding grid has finished: x is final, y may be written
  load_x<FMT>(a, cw, lane);
  __syncwarp();
  if (nstash) {
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(stash_bar, 0, a.budget))) ok = false;
    tc_fence_after();
  }

  // ---- compute, stage by stage.  Each warp writes its share of a row group
  // into the table of partial sums, tab[group][warp][row], as it leaves the
  // group; the shares meet once per batch of tgroups groups, rather than at
  // a barrier per group.  (Taking the ring-resident stages first, so that
  // the ring refills during the tensor-memory stages, measured slower.)
  const LaneOffs f = lane_offs<FMT>(cw, lane, ro);
  const uint32_t xlane = a.xf_off + t * 16 + F::kUnitBlk * cw * 64;
  const uint32_t clane = a.xc_off + F::kUnitBlk * cw * 4;
  float* tab = reinterpret_cast<float*>(smem + a.tab_off);
  uint32_t bar_uses = 0;
  float acc[2] = {0.f, 0.f};
  // a warp's share of a row group goes to table slot `slot`
  auto flush = [&](int slot) {
    if ((t & 1) == 0) tab[(slot * kCons + cw) * kRows + ro] = acc[0] + acc[1];
    acc[0] = acc[1] = 0.f;
  };
  // stages [j, jend), the first being tile c; each group's share goes to the
  // next table slot
  auto run = [&](int j, const int jend, int c, int slot) {
    for (const int je = min(jend, nstash); j < je; ++j) {  // in tensor memory
      uint32_t w[kStageWords];
      stash_load(tq, j, w);
      tmem_wait_ld();
      const uint32_t xb = xlane + c * 4096, cb = clane + c * 256;
      stage_math<FMT, false>(w, acc, xb, cb, cw, c == a.ntiles - 1 ? last_nb : F::kPerTile, hi_row);
      if (++c == a.ntiles) {
        flush(slot++);
        c = 0;
      }
    }
    for (; j < jend; ++j) {  // in the ring
      const int s = j & (kRing - 1);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (j / kRing) & 1u, a.budget))) {
        ok = false;
        return;
      }
      const uint32_t st = static_cast<uint32_t>(s * kStageBytes);
      const uint32_t xb = xlane + c * 4096, cb = clane + c * 256;
      const int nb = c == a.ntiles - 1 ? last_nb : F::kPerTile;
      uint32_t w[kStageWords];
      tile_words<FMT, false>(st, nb, cw, f, w);
      stage_math<FMT, false>(w, acc, xb, cb, cw, nb, hi_row);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++c == a.ntiles) {
        flush(slot++);
        c = 0;
      }
    }
  };
  // every warp's shares are in the table
  auto table_barrier = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(red_bar);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(red_bar, bar_uses & 1u, a.budget))) ok = false;
    ++bar_uses;
  };
  // the sum of slot `slot` over the warps (lanes 0..15: one row each): the
  // output of row group g
  int fmi = 0;
  auto finish = [&](int slot, int64_t g) {
    float v = 0.f;
#pragma unroll
    for (int ww = 0; ww < kCons; ++ww) v += tab[(slot * kCons + ww) * kRows + lane];
    const GroupAt at = group_at(a, tbl, g, fmi);
    const int64_t row = at.lg * kRows + lane;
    if (row < at.M) store_elem(at.y, row, v * 16777216.0f, a.ytype);  // * 2^24
  };

  int j = 0;
  // row groups, in batches of tgroups
  for (int w0 = 0; w0 < nwhole && ok; w0 += a.tgroups) {
    const int gn = min(a.tgroups, nwhole - w0);
    run(j, j + gn * a.ntiles, 0, 0);
    j += gn * a.ntiles;
    if (!ok) break;
    table_barrier();
    if (!ok) break;
    if (lane < kRows)
      for (int sl = cw; sl < gn; sl += kCons)
        finish(sl, blockIdx.x + static_cast<int64_t>(w0 + sl) * gridDim.x);
    if (w0 + gn < nwhole) table_barrier();  // the next batch reuses the table
  }
  if (!ok && lane == 0) report(a.dev_status, GQ_DEV_TIMEOUT);

  // tensor memory is released once every consumer warp is done with it
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(done_bar);
  mbar_wait(done_bar, 0, 4 * a.budget);
  tc_fence_after();
  if (warp == 1 && a.stash) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ repack
// One thread per 4-byte word of the tiled storage: find the canonical bytes
// it holds (rows past M hold zeros).
__device__ __forceinline__ uint32_t canon_bytes(const uint8_t* W, int64_t off, int n) {
  uint32_t v = 0;
  for (int b = 0; b < n; ++b) v |= static_cast<uint32_t>(__ldg(W + off + b)) << (8 * b);
  return v;
}

template <int FMT>
__global__ void __launch_bounds__(256) repack_kernel(const uint8_t* W, int64_t M, int64_t rowbytes,
                                                     int nblk, uint32_t* out, int64_t nwords) {
  using F = Tile<FMT>;
  const int64_t wi = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (wi >= nwords) return;
  const int64_t o = 4 * wi;
  const int64_t gbytes = kRows * rowbytes;
  const int64_t g = o / gbytes, og = o - g * gbytes;
  const int c = static_cast<int>(og / F::kTileBytes);
  const int ot = static_cast<int>(og - static_cast<int64_t>(c) * F::kTileBytes);
  const int nb = min(F::kPerTile, nblk - c * F::kPerTile);
  uint32_t v = 0;
  if constexpr (FMT == GQ_FMT_Q4_0) {
    if (ot < 256 * nb) {
      // code word: unit u, lane l, word position ws (block 2u + ws / 2, row gg + 8 (ws % 2))
      const int u = ot / 512, l = (ot % 512) / 16, ws = (ot % 16) / 4;
      const int64_t row = g * kRows + l / 4 + 8 * (ws & 1);
      const int64_t blk = static_cast<int64_t>(c) * F::kPerTile + 2 * u + (ws >> 1);
      if (row < M) v = canon_bytes(W, row * rowbytes + blk * 18 + 2 + 4 * (l % 4), 4);
    } else {
      // scales of unit u, row r: d of blocks 2u and 2u + 1
      const int os = ot - 256 * nb, u = os / 64, r = (os % 64) / 4;
      const int64_t row = g * kRows + r;
      const int64_t blk = static_cast<int64_t>(c) * F::kPerTile + 2 * u;
      if (row < M)
        v = canon_bytes(W, row * rowbytes + blk * 18, 2) |
            (canon_bytes(W, row * rowbytes + (blk + 1) * 18, 2) << 16);
    }
  } else {
    if (ot < 2048 * nb) {
      // code word: unit u, lane l, sub-block h of the unit, row gg + 8 (ws % 2)
      const int u = ot / 1024, l = (ot % 1024) / 32, h = (ot % 32) / 8, ws = (ot % 8) / 4;
      const int64_t row = g * kRows + l / 4 + 8 * ws;
      const int64_t sb = static_cast<int64_t>(c) * F::kPerTile + u / 2;
      const int jj = 4 * (u % 2) + h;
      if (row < M) v = canon_bytes(W, row * rowbytes + sb * 138 + 10 + 16 * jj + 4 * (l % 4), 4);
    } else if (ot < 2176 * nb) {
      // the four sub-scales of unit u, row r
      const int oq = ot - 2048 * nb, u = oq / 64, r = (oq % 64) / 4;
      const int64_t row = g * kRows + r;
      const int64_t sb = static_cast<int64_t>(c) * F::kPerTile + u / 2;
      if (row < M) v = canon_bytes(W, row * rowbytes + sb * 138 + 2 + 4 * (u % 2), 4);
    } else {
      // super-scales of super-block sbi, rows r and r + 1
      const int os = ot - 2176 * nb, sbi = os / 32, r = (os % 32) / 2;
      const int64_t sb = static_cast<int64_t>(c) * F::kPerTile + sbi;
      const int64_t row = g * kRows + r;
      if (row < M) v = canon_bytes(W, row * rowbytes + sb * 138, 2);
      if (row + 1 < M) v |= canon_bytes(W, (row + 1) * rowbytes + sb * 138, 2) << 16;
    }
  }
  out[wi] = v;
}

// ------------------------------------------------------------------- host
int64_t canon_row_bytes(int fmt, int64_t K) {
  return fmt == GQ_FMT_Q4_0 ? K / 32 * 18 : K / 256 * 138;
}

bool unit_shape(int fmt, int64_t K) { return K % (fmt == GQ_FMT_Q4_0 ? 64 : 256) == 0; }

// Shared memory of one CTA: the ring, x fragments and block corrections, the
// table of partial sums (tgroups row groups), barriers.  Two CTAs share an
// SM, so the table takes what the ring and x leave of half an SM.
constexpr size_t kCtaSmem = 113 * 1024;
constexpr int kMaxTableGroups = 16;
constexpr size_t kBarBytes = (2 * kRing + 3) * 8 + 16;
size_t tiled_smem(int K, int& tgroups, uint32_t& xf, uint32_t& xc, uint32_t& tab, uint32_t& bar) {
  const uint32_t nkb = static_cast<uint32_t>(K / 32);
  xf = kRing * kStageBytes;
  xc = xf + nkb * 64;
  tab = (xc + nkb * 4 + 15) & ~15u;
  const size_t group_bytes = kCons * kRows * 4;
  const size_t left = kCtaSmem - tab - kBarBytes;
  tgroups = static_cast<int>(left / group_bytes < kMaxTableGroups ? left / group_bytes : kMaxTableGroups);
  bar = tab + static_cast<uint32_t>(tgroups * group_bytes);
  return bar + kBarBytes;
}

template <int FMT, class Tbl>
gq_status launch_tiled(const TArgs& a0, const Tbl& tbl, int grid, size_t smem_bytes, bool pdl,
                       cudaStream_t stream) {
  auto kern = gemv_tiled_kernel<FMT, Tbl>;
  thread_local unsigned long long configured_ctx = 0;  // per host thread and context
  const unsigned long long ctx = context_id();
  if (ctx == 0 || ctx != configured_ctx) {
    // no layout exceeds the per-CTA budget, so one setting serves every call
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kCtaSmem)) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_ctx = ctx;
  }
  return launch(kern, dim3(grid), dim3(kThreads), smem_bytes, stream, pdl, a0, tbl);
}

template <int FMT>
gq_status gemv_tiled_entry(const void* T, int64_t M, int64_t K, const void* x, int x_dtype,
                           void* y, int y_dtype, unsigned flags, int* dev_status, void* stream) {
  if (M < 0 || K < 0) return GQ_ERR_INVALID_ARG;
  if (x_dtype != GQ_F16 || !valid_act_dtype(y_dtype)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (!unit_shape(FMT, K) || K > kMaxKb * 32 || M > 0x7FFFFFFFLL) return GQ_ERR_SHAPE;
  if (M == 0) return GQ_OK;
  if (!y) return GQ_ERR_INVALID_ARG;
  if (misaligned16(y)) return GQ_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  if (K == 0)
    return cudaMemsetAsync(y, 0, static_cast<size_t>(M * dtype_size(y_dtype)), s) == cudaSuccess
               ? GQ_OK
               : GQ_ERR_CUDA;
  if (!T || !x) return GQ_ERR_INVALID_ARG;
  if (misaligned16(T) || misaligned16(x)) return GQ_ERR_ALIGNMENT;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return GQ_ERR_ALIGNMENT;
  const bool pdl = (flags & GQ_GEMV_PDL) != 0;

  TArgs a{};
  a.T = static_cast<const uint8_t*>(T);
  a.x = static_cast<const __half*>(x);
  a.y = y;
  a.dev_status = dev_status;
  a.budget = kWaitBudget;
  a.M = M;
  a.group_bytes = kRows * canon_row_bytes(FMT, K);
  a.K = static_cast<int>(K);
  a.ytype = y_dtype;
  a.nblk = static_cast<int>(FMT == GQ_FMT_Q4_0 ? K / 32 : K / 256);
  a.ntiles = (a.nblk + Tile<FMT>::kPerTile - 1) / Tile<FMT>::kPerTile;
  const int64_t ngroups = (M + kRows - 1) / kRows;
  a.ngroups = static_cast<int>(ngroups);
  const int grid = static_cast<int>(ngroups < sm_count() ? ngroups : sm_count());
  const int64_t stages = ((ngroups + grid - 1) / grid) * a.ntiles;
  // tensor memory only pays when the next launch can stream while this one
  // waits, and only when the ring alone cannot hold the CTA's share
  a.stash = (pdl && stages > kRing) ? kStashMax : 0;
  const size_t smem_bytes = tiled_smem(a.K, a.tgroups, a.xf_off, a.xc_off, a.tab_off, a.bar_off);
  return launch_tiled<FMT>(a, OneMatrix{}, grid, smem_bytes, pdl, s);
}

// Several tiled matrices that share K and x: y_i = W_i x for each descriptor
// (W_i in tiled storage), in launches of up to kMaxTiledMats matrices whose
// CTAs stream the row groups of all of them back to back.
template <int FMT>
gq_status gemv_tiled_grouped_entry(const gq_gemv_desc* mats, int count, int64_t K,
                                   const void* x, int x_dtype, int y_dtype, unsigned flags,
                                   int* dev_status, void* stream) {
  if (count < 0 || K < 0) return GQ_ERR_INVALID_ARG;
  if (count > 0 && !mats) return GQ_ERR_INVALID_ARG;
  if (x_dtype != GQ_F16 || !valid_act_dtype(y_dtype)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (!unit_shape(FMT, K) || K > kMaxKb * 32) return GQ_ERR_SHAPE;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return GQ_ERR_ALIGNMENT;
  int64_t groups = 0;
  for (int i = 0; i < count; ++i) {
    const gq_gemv_desc& d = mats[i];
    if (d.M < 0) return GQ_ERR_INVALID_ARG;
    if (d.M > 0x7FFFFFFFLL) return GQ_ERR_SHAPE;
    if (d.M == 0) continue;
    if (!d.y || (K > 0 && !d.W)) return GQ_ERR_INVALID_ARG;
    if (misaligned16(d.y) || misaligned16(d.W)) return GQ_ERR_ALIGNMENT;
    groups += (d.M + kRows - 1) / kRows;
  }
  if (groups > 0x7FFFFFFFLL) return GQ_ERR_SHAPE;
  if (groups == 0) return GQ_OK;
  cudaStream_t s = as_stream(stream);
  if (K == 0) {
    for (int i = 0; i < count; ++i)
      if (mats[i].M > 0 &&
          cudaMemsetAsync(mats[i].y, 0, static_cast<size_t>(mats[i].M * dtype_size(y_dtype)), s) !=
              cudaSuccess)
        return GQ_ERR_CUDA;
    return GQ_OK;
  }
  if (!x) return GQ_ERR_INVALID_ARG;
  if (misaligned16(x)) return GQ_ERR_ALIGNMENT;
  const bool pdl = (flags & GQ_GEMV_PDL) != 0;

  TArgs a{};
  a.x = static_cast<const __half*>(x);
  a.dev_status = dev_status;
  a.budget = kWaitBudget;
  a.group_bytes = kRows * canon_row_bytes(FMT, K);
  a.K = static_cast<int>(K);
  a.ytype = y_dtype;
  a.nblk = static_cast<int>(FMT == GQ_FMT_Q4_0 ? K / 32 : K / 256);
  a.ntiles = (a.nblk + Tile<FMT>::kPerTile - 1) / Tile<FMT>::kPerTile;
  const size_t smem_bytes = tiled_smem(a.K, a.tgroups, a.xf_off, a.xc_off, a.tab_off, a.bar_off);
  TiledTable tbl{};  // one launch's table, passed to the kernel by value
  int i = 0;
  while (i < count) {
    int n = 0, g = 0;
    for (; i < count && n < kMaxTiledMats; ++i) {
      const gq_gemv_desc& d = mats[i];
      if (d.M == 0) continue;
      g += static_cast<int>((d.M + kRows - 1) / kRows);
      tbl.m[n] = TiledMat{static_cast<const uint8_t*>(d.W), d.y, d.M, g, 0};
      ++n;
    }
    if (n == 0) break;
    a.ngroups = g;
    // Two CTAs per SM from this one launch, each taking its first stages
    // through tensor memory whether or not the launch overlaps another: on
    // long grouped streams this measured faster than one CTA per SM (with or
    // without the stash) and than two CTAs per SM without it.
    const int grid = g < 2 * sm_count() ? g : 2 * sm_count();
    const int64_t stages = ((static_cast<int64_t>(g) + grid - 1) / grid) * a.ntiles;
    a.stash = stages > kRing ? kStashMax : 0;
    const gq_status st = launch_tiled<FMT>(a, tbl, grid, smem_bytes, pdl, s);
    if (st != GQ_OK) return st;
  }
  return GQ_OK;
}

template <int FMT>
gq_status repack_entry(const void* W, int64_t M, int64_t K, void* out, void* stream) {
  if (M < 0 || K < 0) return GQ_ERR_INVALID_ARG;
  if (!unit_shape(FMT, K)) return GQ_ERR_SHAPE;
  const int64_t bytes = (M + kRows - 1) / kRows * kRows * canon_row_bytes(FMT, K);
  if (bytes == 0) return GQ_OK;
  if (!W || !out) return GQ_ERR_INVALID_ARG;
  if (misaligned16(W) || misaligned16(out)) return GQ_ERR_ALIGNMENT;
  const int64_t nwords = bytes / 4;
  const int64_t blocks = (nwords + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return GQ_ERR_SHAPE;
  repack_kernel<FMT><<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      static_cast<const uint8_t*>(W), M, canon_row_bytes(FMT, K),
      static_cast<int>(FMT == GQ_FMT_Q4_0 ? K / 32 : K / 256), static_cast<uint32_t*>(out), nwords);
  return cudaGetLastError() == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

}  // namespace
}  // namespace gq

extern "C" {

GQ_API size_t gq_tiled_bytes(int fmt, int64_t M, int64_t K) {
  if ((fmt != GQ_FMT_Q4_0 && fmt != GQ_FMT_KSB) || M < 0 || K < 0 || !gq::unit_shape(fmt, K))
    return 0;
  return static_cast<size_t>((M + 15) / 16 * 16 * gq::canon_row_bytes(fmt, K));
}

GQ_API gq_status gq_repack_q4_0(const void* W, int64_t M, int64_t K, void* out, void* stream) {
  return gq::repack_entry<GQ_FMT_Q4_0>(W, M, K, out, stream);
}

GQ_API gq_status gq_repack_ksb(const void* W, int64_t M, int64_t K, void* out, void* stream) {
  return gq::repack_entry<GQ_FMT_KSB>(W, M, K, out, stream);
}

GQ_API gq_status gq_gemv_q4_0_tiled(const void* T, int64_t M, int64_t K, const void* x,
                                    int x_dtype, void* y, int y_dtype, unsigned flags,
                                    int* dev_status, void* stream) {
  return gq::gemv_tiled_entry<GQ_FMT_Q4_0>(T, M, K, x, x_dtype, y, y_dtype, flags, dev_status,
                                           stream);
}

GQ_API gq_status gq_gemv_ksb_tiled(const void* T, int64_t M, int64_t K, const void* x, int x_dtype,
                                   void* y, int y_dtype, unsigned flags, int* dev_status,
                                   void* stream) {
  return gq::gemv_tiled_entry<GQ_FMT_KSB>(T, M, K, x, x_dtype, y, y_dtype, flags, dev_status,
                                          stream);
}

GQ_API gq_status gq_gemv_q4_0_tiled_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                            const void* x, int x_dtype, int y_dtype,
                                            unsigned flags, int* dev_status, void* stream) {
  return gq::gemv_tiled_grouped_entry<GQ_FMT_Q4_0>(mats, count, K, x, x_dtype, y_dtype, flags,
                                                   dev_status, stream);
}

GQ_API gq_status gq_gemv_ksb_tiled_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                           const void* x, int x_dtype, int y_dtype,
                                           unsigned flags, int* dev_status, void* stream) {
  return gq::gemv_tiled_grouped_entry<GQ_FMT_KSB>(mats, count, K, x, x_dtype, y_dtype, flags,
                                                  dev_status, stream);
}

}  // extern "C"
