// gq_gemv_i8.cu -- batch-1 Q4_0 GEMV on the integer tensor-core path.
//
// y = W_hat x with one fp16 activation vector (Q4_0 chapter 4.3: each weight
// is d * (q - 8); the product consumes the decoded block; the TurboQuant W4A8
// post, section 2.3: decode is bound by the weight stream).  With a single
// vector, seven of the eight columns of a warp MMA would be idle; this path
// fills six of them with an exact split of x instead:
//
//   x * 2^24 = sum_{i<6} L_i * 2^(7 i),   L_i = sign(x) * digit_i(|x| * 2^24)
//
// where digit_i is the i-th 7-bit digit.  Every fp16 value is an integer
// multiple of 2^-24 below 2^16, so six digits (42 bits) represent it exactly
// and every L_i fits in a signed byte.  The codes enter the MMA unchanged as
// unsigned bytes (a nibble mask, no float decode), and
//
//   sum_k (q_k - 8) L_{k,i} = mma(q, L)_i - 8 * sum_k L_{k,i}
//
// is an exact int32.  The correction and a float-conversion bias enter as the
// MMA's accumulator input, so the MMA returns 1.5 * 2^23 + the exact integer;
// one packed subtract turns it into an exact float, one packed FMA applies the
// block scale d.  Only the fp32 accumulation over blocks, and the final sum of
// the six digit columns weighted by 2^(7i-24), round.
//
// One kernel, one persistent CTA per SM, four roles:
//   warp 0       streams the matrix.  It is cut into units of 16 rows x 8
//                blocks (16 x 144 bytes, whole 16-byte granules); each CTA
//                takes an equal contiguous run of units in row-major order,
//                so the work is balanced to one unit.  One 2-D TMA load per
//                unit fills a ring of stages (up to 8 units of one row group).
//   warps 1-19   first split x into the MMA B fragments of the six digit
//                columns, with the per-block corrections, in shared memory
//                (every CTA needs the whole row; this overlaps the first
//                loads of the ring).
//   warps 1-16   then consume the ring, each taking two pairs of blocks of
//                every stage; at the end of a row group each folds its digit
//                columns and hands 16 row sums to the epilogue.
//   warps 17-19  write y: warp 17 the whole row groups, warps 18 and 19 one
//                row group each that is cut between two CTAs.  A cut row
//                group is combined through fp32 partial sums in the
//                workspace: the CTA that completes it last (an atomic unit
//                count) sums the parts in CTA order, so the result does not
//                depend on scheduling, and resets the count.  CTAs do their
//                cut row groups first, on their own warps, so the exchange
//                overlaps the rest of the work.
//
// The split costs about 30 instructions per element on every SM and is
// shared by only M / (number of SMs) rows, so this path pays off for tall
// matrices; the entry points take it only when the caller passes a workspace.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_gemv_i8.h"
#include "gq_host.h"
#include "gq_tc.cuh"

namespace gq {
namespace {

constexpr int kRows = 16;               // rows per unit (one m16 MMA tile)
constexpr int kUnitBlk = 8;             // blocks per unit: 8 x 18 = 144 bytes per row
constexpr int kUnitRowBytes = kUnitBlk * 18;
constexpr int kUnitBytes = kRows * kUnitRowBytes;  // 2304
constexpr int kStageUnits = 8;          // units per stage (64 blocks)
constexpr int kStageBytes = kStageUnits * kUnitBytes;
constexpr int kMaxStages = 8;
constexpr int kConsumers = 16;          // consumer warps 1..16
constexpr int kEpiWarp = 1 + kConsumers;  // warp 17: whole row groups
constexpr int kCutWarp = 2 + kConsumers;  // warps 18, 19: the two cut row groups
constexpr int kWarps = 4 + kConsumers;
constexpr int kSplitters = kWarps - 1;  // every warp but the producer splits x
constexpr int kThreads = 32 * kWarps;
constexpr int kRed = 4;                 // reduction ring depth
constexpr int kSplitIters = 6;          // ceil(kMaxBlk / (4 * kSplitters))
constexpr int kLimbBlkBytes = 288;      // 256 B of B fragments + 8 int32 corrections
constexpr int kMaxBlk = 448;            // fragments of K <= 14336 stay resident
static_assert(kSplitIters * 4 * (kWarps - 1) >= kMaxBlk, "split registers");
constexpr int kMaxCtas = 256;           // counters in the workspace
constexpr uint32_t kMagicBits = 0x4B400000u;  // 1.5 * 2^23 as float bits
constexpr float kMagic = 12582912.0f;
// Accumulator input of a block that holds a NaN or an infinity: a quiet-NaN
// pattern that stays NaN for every MMA sum (|sum| < 2^16).
constexpr uint32_t kPoisonBits = 0x7FC00000u;
constexpr size_t kSmemBudget = 227 * 1024;

// rows g and g+8 of a warp hit distinct banks (row pitch / 4 == 4 mod 32)
static_assert((kUnitRowBytes / 4) % 32 == 4, "unit row pitch");

extern __shared__ __align__(1024) uint8_t smem[];

__device__ __forceinline__ uint32_t ld32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}
__device__ __forceinline__ uint32_t ld16(uint32_t off) {
  return *reinterpret_cast<const uint16_t*>(smem + off);
}
__device__ __forceinline__ uint2 ld64(uint32_t off) {
  return *reinterpret_cast<const uint2*>(smem + off);
}
__device__ __forceinline__ void st32(uint32_t off, uint32_t v) {
  *reinterpret_cast<uint32_t*>(smem + off) = v;
}

// ------------------------------------------------------------ activation split
// Signed digits of one fp16 value, little-endian: bytes 0-3 of `lo` are
// L_0..L_3, bytes 0-1 of `hi` are L_4, L_5.  |x| * 2^24 = m * 2^s with an
// 11-bit m, so the value touches at most three consecutive digits: with
// s = 7a + r, the digits a, a+1, a+2 are those of m * 2^r (< 2^18).
__device__ __forceinline__ void fp16_digits(uint32_t h, uint32_t& lo, uint32_t& hi, bool& bad) {
  const uint32_t mag = h & 0x7FFFu, e = mag >> 10;
  bad = (e == 31u);
  uint32_t m = e ? ((mag & 0x3FFu) | 0x400u) : mag;
  if (bad) m = 0;
  const uint32_t s = e ? e - 1u : 0u;        // 0..29
  const uint32_t a = (s * 37u) >> 8;         // s / 7 for s < 64
  const uint32_t w = m << (s - 7u * a);      // m * 2^r
  const uint32_t d3 = (w & 0x7Fu) | ((w << 1) & 0x7F00u) | ((w << 2) & 0x7F0000u);
  const uint64_t f = static_cast<uint64_t>(d3) << (8u * a);
  lo = static_cast<uint32_t>(f);
  hi = static_cast<uint32_t>(f >> 32);
  if (h & 0x8000u) {
    // negate every byte (each is <= 0x7F, so no borrow crosses a byte)
    lo = (0x80808080u - lo) ^ 0x80808080u;
    hi = (0x80808080u - hi) ^ 0x80808080u;
  }
}

// Splitter warp `sw` of kSplitters: blocks in groups of four, eight lanes per
// block, four consecutive elements per lane.  The B fragment of lane (g, t)
// of a block holds digit column g of elements 4t..4t+3 (bytes 0-3) and
// 16+4t..16+4t+3 (bytes 4-7); columns 6 and 7 are zero.  The correction
// words come from one integer MMA of the fragments with an all-ones A.
// Returns whether any of this warp's elements is a NaN or an infinity.
__device__ __forceinline__ bool split_x(const uint16_t* __restrict__ x, int nblk, int sw,
                                        int lane, uint32_t limb_off) {
  const int q = lane & 7, t = q & 3, half = q >> 2;
  bool anybad = false;
  // all of this warp's x words first, so their latencies overlap
  uint2 xr[kSplitIters];
#pragma unroll
  for (int it = 0; it < kSplitIters; ++it) {
    const int b = sw * 4 + it * kSplitters * 4 + (lane >> 3);
    xr[it] = b < nblk ? __ldg(reinterpret_cast<const uint2*>(x + static_cast<int64_t>(b) * 32 + 4 * q))
                      : make_uint2(0u, 0u);
  }
#pragma unroll
  for (int it = 0; it < kSplitIters; ++it) {
    const int b4 = sw * 4 + it * kSplitters * 4;
    if (b4 >= nblk) break;  // warp-uniform
    const int b = b4 + (lane >> 3);
    bool bad = false;
    if (b < nblk) {
      const uint2 raw = xr[it];
      uint32_t lo[4], hi[4];
      bool bd[4];
      fp16_digits(raw.x & 0xFFFFu, lo[0], hi[0], bd[0]);
      fp16_digits(raw.x >> 16, lo[1], hi[1], bd[1]);
      fp16_digits(raw.y & 0xFFFFu, lo[2], hi[2], bd[2]);
      fp16_digits(raw.y >> 16, lo[3], hi[3], bd[3]);
      bad = bd[0] | bd[1] | bd[2] | bd[3];
      // 4 x 6 byte transpose: digit column i <- byte i of the four elements
      const uint32_t l01a = __byte_perm(lo[0], lo[1], 0x5140u);
      const uint32_t l01b = __byte_perm(lo[0], lo[1], 0x7362u);
      const uint32_t l23a = __byte_perm(lo[2], lo[3], 0x5140u);
      const uint32_t l23b = __byte_perm(lo[2], lo[3], 0x7362u);
      const uint32_t h01 = __byte_perm(hi[0], hi[1], 0x5140u);
      const uint32_t h23 = __byte_perm(hi[2], hi[3], 0x5140u);
      const uint32_t col[6] = {__byte_perm(l01a, l23a, 0x5410u), __byte_perm(l01a, l23a, 0x7632u),
                               __byte_perm(l01b, l23b, 0x5410u), __byte_perm(l01b, l23b, 0x7632u),
                               __byte_perm(h01, h23, 0x5410u), __byte_perm(h01, h23, 0x7632u)};
      const uint32_t base = limb_off + static_cast<uint32_t>(b) * kLimbBlkBytes + t * 8 + half * 4;
#pragma unroll
      for (int i = 0; i < 6; ++i) st32(base + i * 32, col[i]);
      st32(base + 6 * 32, 0u);
      st32(base + 7 * 32, 0u);
    }
    const uint32_t badmask = __ballot_sync(0xFFFFFFFFu, bad);
    anybad |= (badmask != 0);
    __syncwarp();
    // corrections: D = ones * B gives sum_k L_{k,c} in every row
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int bj = b4 + j;
      if (bj >= nblk) break;  // warp-uniform
      const uint32_t blk = limb_off + static_cast<uint32_t>(bj) * kLimbBlkBytes;
      const uint2 bf = ld64(blk + lane * 8);
      int sm[4];
      asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%4,%4,%4}, "
          "{%5,%6}, {%7,%7,%7,%7};"
          : "=r"(sm[0]), "=r"(sm[1]), "=r"(sm[2]), "=r"(sm[3])
          : "r"(0x01010101u), "r"(bf.x), "r"(bf.y), "r"(0));
      const int s0 = sm[0], s1 = sm[1];
      if (lane < 4) {  // row 0: columns 2t, 2t+1
        const bool poisoned = ((badmask >> (8 * j)) & 0xFFu) != 0;
        const uint32_t c0 = poisoned ? kPoisonBits : kMagicBits - 8u * static_cast<uint32_t>(s0);
        const uint32_t c1 = poisoned ? kPoisonBits : kMagicBits - 8u * static_cast<uint32_t>(s1);
        *reinterpret_cast<uint2*>(smem + blk + 256 + lane * 8) = make_uint2(c0, c1);
      }
    }
    __syncwarp();
  }
  return anybad;
}

// ------------------------------------------------------------ work split
// Units: row group rg (16 rows) x unit column j (8 blocks); Cu columns per
// row, U = G * Cu in all.  CTA i owns units [U*i/P, U*(i+1)/P).
struct Split {
  int64_t U;
  int Cu, G, P;
};

__device__ __forceinline__ int64_t unit_begin(const Split& sp, int i) {
  return sp.U * i / sp.P;
}
// the CTA that owns unit u
__device__ __forceinline__ int unit_owner(const Split& sp, int64_t u) {
  const int64_t i = ((u + 1) * sp.P - 1) / sp.U;
  return static_cast<int>(i < sp.P - 1 ? i : sp.P - 1);
}

// This CTA's row segments in processing order: the cut row groups first
// (slots 0 and 1 of its partial sums), then whole row groups f0 .. f1-1.
struct Segments {
  int npart;
  int prg[2], pua[2], pub[2], pslot[2];
  int f0, f1;
  __device__ __forceinline__ int count() const { return npart + (f1 - f0); }
  __device__ __forceinline__ void get(int k, int cu, int& rg, int& ua, int& ub, int& slot) const {
    if (k < npart) {  // constant indices keep the struct in registers
      const bool first = (k == 0);
      rg = first ? prg[0] : prg[1];
      ua = first ? pua[0] : pua[1];
      ub = first ? pub[0] : pub[1];
      slot = first ? pslot[0] : pslot[1];
    } else {
      rg = f0 + (k - npart);
      ua = 0;
      ub = cu;
      slot = -1;
    }
  }
};

__device__ __forceinline__ Segments make_segments(const Split& sp, int i) {
  Segments sg;
  const int64_t u0 = unit_begin(sp, i), u1 = unit_begin(sp, i + 1);
  const int rga = static_cast<int>(u0 / sp.Cu), rgb = static_cast<int>((u1 - 1) / sp.Cu);
  const int a0 = static_cast<int>(u0 - static_cast<int64_t>(rga) * sp.Cu);
  const int b1 = static_cast<int>(u1 - static_cast<int64_t>(rgb) * sp.Cu);
  sg.npart = 0;
  if (rga == rgb) {
    sg.prg[0] = sg.prg[1] = rga;
    sg.pua[0] = sg.pua[1] = a0;
    sg.pub[0] = sg.pub[1] = b1;
    sg.pslot[0] = sg.pslot[1] = 0;
    if (a0 == 0 && b1 == sp.Cu) {
      sg.f0 = rga;
      sg.f1 = rga + 1;
    } else {
      sg.npart = 1;
      sg.f0 = sg.f1 = 0;
    }
    return sg;
  }
  const bool cut_tail = b1 < sp.Cu, cut_head = a0 > 0;
  sg.f0 = cut_head ? rga + 1 : rga;
  sg.f1 = cut_tail ? rgb : rgb + 1;
  // the cut tail row group first (slot 1), then the cut head (slot 0)
  sg.prg[0] = cut_tail ? rgb : rga;
  sg.pua[0] = cut_tail ? 0 : a0;
  sg.pub[0] = cut_tail ? b1 : sp.Cu;
  sg.pslot[0] = cut_tail ? 1 : 0;
  sg.prg[1] = rga;
  sg.pua[1] = a0;
  sg.pub[1] = sp.Cu;
  sg.pslot[1] = 0;
  sg.npart = (cut_tail ? 1 : 0) + (cut_head ? 1 : 0);
  return sg;
}

struct I8Args {
  const uint16_t* x;
  int M, nblk, nstages;
  Split sp;
  float* partials;   // [P][2][16]
  int* counters;     // [kMaxCtas], zero between calls
  void* y;
  int ytype;
  int* dev_status;
  long long budget;
};

// One block for rows g (codes qa, scale da) and g+8 (qb, db); b = this
// lane's B fragment, c = the biased corrections of its two columns.
__device__ __forceinline__ void block_i8(float2& acc0, float2& acc1, uint32_t qa, uint32_t qb,
                                         float da, float db, uint2 b, uint2 c) {
  const uint32_t a0 = qa & 0x0F0F0F0Fu, a1 = qb & 0x0F0F0F0Fu;
  const uint32_t a2 = (qa >> 4) & 0x0F0F0F0Fu, a3 = (qb >> 4) & 0x0F0F0F0Fu;
  int d0, d1, d2, d3;
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%10,%11};"
      : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y), "r"(c.x), "r"(c.y));
  const float2 mg = make_float2(-kMagic, -kMagic);
  const float2 f0 = __fadd2_rn(make_float2(__int_as_float(d0), __int_as_float(d1)), mg);
  const float2 f1 = __fadd2_rn(make_float2(__int_as_float(d2), __int_as_float(d3)), mg);
  acc0 = __ffma2_rn(make_float2(da, da), f0, acc0);
  acc1 = __ffma2_rn(make_float2(db, db), f1, acc1);
}

__device__ __forceinline__ float half_to_f(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv_i8_kernel(const __grid_constant__ CUtensorMap wmap, const I8Args a) {
  const int nst = a.nstages;
  const uint32_t limb_off = 0;
  const uint32_t stage_off = static_cast<uint32_t>((a.nblk * kLimbBlkBytes + 1023) & ~1023);
  // row sums of the consumer warps: [kRed][kConsumers][16]
  float* red = reinterpret_cast<float*>(smem + stage_off + nst * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kRed * kConsumers * kRows);
  uint64_t* empty = full + kMaxStages;
  uint64_t* rfull = empty + kMaxStages;
  uint64_t* rempty = rfull + kRed;
  uint64_t* lready = rempty + kRed;
  int* flags = reinterpret_cast<int*>(lready + 1);  // [0] abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Segments sg = make_segments(a.sp, blockIdx.x);
  const int Cu = a.sp.Cu;
  const int nseg = sg.count();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    for (int b = 0; b < kRed; ++b) {
      mbar_init(&rfull[b], kConsumers);
      mbar_init(&rempty[b], 1);
    }
    mbar_init(lready, kSplitters);
    flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // W is not written by the kernels this one may overlap, so the stream
    // starts before the wait for the preceding grid.
    const uint64_t pol = policy_evict_first();
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    for (int k = 0; k < nseg && ok; ++k) {
      int rg, ua, ub, slot;
      sg.get(k, Cu, rg, ua, ub, slot);
      for (int c = ua / kStageUnits; c * kStageUnits < ub; ++c, ++issued) {
        const int ja = max(ua - c * kStageUnits, 0), jb = min(ub - c * kStageUnits, kStageUnits);
        if (!mbar_wait(&empty[s], ph ^ 1u, a.budget) ||
            *reinterpret_cast<volatile int*>(&flags[0])) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>((jb - ja) * kUnitBytes));
        __syncwarp();
        const int j = ja + lane;
        if (j < jb)
          tma_load_2d_hint(smem + stage_off + s * kStageBytes + j * kUnitBytes, &wmap,
                           (c * kStageUnits + j) * kUnitRowBytes, rg * kRows, &full[s], pol);
        if (++s == nst) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      report(a.dev_status, GQ_DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(&flags[0]) = 1;
    }
    // every issued copy lands before the CTA's shared memory is released
    if (lane == 0) {
      for (int u = issued > nst ? issued - nst : 0; u < issued; ++u) {
        if (!mbar_wait(&full[u % nst], static_cast<uint32_t>(u / nst) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // -------------------------------------------- activation split (all others)
  pdl_wait();  // x is ready; y and the workspace are ours
  const bool nonfinite = split_x(a.x, a.nblk, warp - 1, lane, limb_off);
  if (nonfinite && blockIdx.x == 0 && lane == 0) report(a.dev_status, GQ_DEV_NONFINITE);
  __syncwarp();
  if (lane == 0) mbar_arrive(lready);

  bool ok = true;
  if (warp >= kEpiWarp) {
    // ------------------------------------------------------------ epilogue
    // warp 17 writes whole row groups; warps 18 and 19 each take one cut row
    // group, so the exchange's fences and atomics overlap everything else
    int kbeg = sg.npart, kend = nseg;
    if (warp != kEpiWarp) {
      kbeg = warp - kCutWarp;
      kend = kbeg < sg.npart ? kbeg + 1 : kbeg;
    }
    for (int k = kbeg; k < kend; ++k) {
      int rg, ua, ub, slot;
      sg.get(k, Cu, rg, ua, ub, slot);
      const int b = k % kRed;
      if (!mbar_wait(&rfull[b], static_cast<uint32_t>(k / kRed) & 1u, a.budget) ||
          *reinterpret_cast<volatile int*>(&flags[0])) {
        ok = false;
        break;
      }
      float mine = 0.f;
      if (lane < kRows) {
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) mine += red[(b * kConsumers + w) * kRows + lane];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[b]);
      const int64_t row = static_cast<int64_t>(rg) * kRows + lane;
      const bool row_ok = lane < kRows && row < a.M;
      if (slot < 0) {
        if (row_ok) store_elem(a.y, row, mine, a.ytype);
        continue;
      }
      // a row group cut between CTAs: publish this part, and sum all parts if
      // it completes the group.  The count lives at the index of the CTA that
      // owns the group's first unit (unique among cut groups).
      const int64_t ufirst = static_cast<int64_t>(rg) * Cu;
      const int i0 = unit_owner(a.sp, ufirst), i1 = unit_owner(a.sp, ufirst + Cu - 1);
      if (lane < kRows) a.partials[(static_cast<int64_t>(blockIdx.x) * 2 + slot) * kRows + lane] = mine;
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(&a.counters[i0], ub - ua) + (ub - ua) == Cu);
      last = __shfl_sync(0xFFFFFFFFu, last, 0);
      if (!last) continue;
      __threadfence();
      float v = 0.f;
      for (int i = i0; i <= i1; ++i) {
        const int sl = (unit_begin(a.sp, i) / Cu == rg) ? 0 : 1;
        if (lane < kRows) v += __ldcg(&a.partials[(static_cast<int64_t>(i) * 2 + sl) * kRows + lane]);
      }
      if (row_ok) store_elem(a.y, row, v, a.ytype);
      if (lane == 0) a.counters[i0] = 0;  // ready for the next call
    }
  } else {
    // ----------------------------------------------------------- consumers
    const int cw = warp - 1;
    const int t = lane & 3;
    // digit column c carries weight 2^(7c - 24); this lane holds c = 2t, 2t+1
    const float w_lo = __int_as_float((127 + 14 * t - 24) << 23);
    const float w_hi = __int_as_float((127 + 14 * t - 17) << 23);
    // this warp's pairs in a stage: units jw and jw + 4, blocks 2 (cw & 3)
    // and 2 (cw & 3) + 1 of each
    const int jw = cw >> 2;
    const uint32_t row_a = static_cast<uint32_t>((lane >> 2) * kUnitRowBytes + 36 * (cw & 3) +
                                                 jw * kUnitBytes);
    const uint32_t row_b = row_a + 8 * kUnitRowBytes;
    const uint32_t limb_lane = limb_off + static_cast<uint32_t>(lane * 8);
    const uint32_t limb_c = limb_off + 256 + static_cast<uint32_t>(t * 8);
    if (!mbar_wait(lready, 0, a.budget)) ok = false;
    int s = 0;
    uint32_t ph = 0;
    for (int k = 0; k < nseg && ok; ++k) {
      int rg, ua, ub, slot;
      sg.get(k, Cu, rg, ua, ub, slot);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      for (int c = ua / kStageUnits; c * kStageUnits < ub; ++c) {
        const int ja = ua - c * kStageUnits, jb = ub - c * kStageUnits;  // valid units [ja, jb)
        if (!mbar_wait(&full[s], ph, a.budget) || *reinterpret_cast<volatile int*>(&flags[0])) {
          ok = false;
          break;
        }
        const uint32_t st = stage_off + static_cast<uint32_t>(s * kStageBytes);
        const uint32_t blk0 =
            static_cast<uint32_t>(c * (kStageUnits * kUnitBlk) + jw * kUnitBlk + 2 * (cw & 3));
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = jw + 4 * i;
          if (j >= ja && j < jb) {  // warp-uniform
            const uint32_t pa = st + row_a + i * 4 * kUnitBytes, pb = st + row_b + i * 4 * kUnitBytes;
            // even block: scale at +0, codes at +2 (2 mod 4); odd block: scale
            // at +18, codes at +20 (4-aligned)
            const uint32_t qa0 = __byte_perm(ld32(pa + 4 * t), ld32(pa + 4 * t + 4), 0x5432u);
            const uint32_t qb0 = __byte_perm(ld32(pb + 4 * t), ld32(pb + 4 * t + 4), 0x5432u);
            const uint32_t qa1 = ld32(pa + 20 + 4 * t), qb1 = ld32(pb + 20 + 4 * t);
            const float da0 = half_to_f(ld16(pa)), db0 = half_to_f(ld16(pb));
            const float da1 = half_to_f(ld16(pa + 18)), db1 = half_to_f(ld16(pb + 18));
            const uint32_t lb = (blk0 + i * 4 * kUnitBlk) * kLimbBlkBytes;
            block_i8(acc0, acc1, qa0, qb0, da0, db0, ld64(limb_lane + lb), ld64(limb_c + lb));
            block_i8(acc0, acc1, qa1, qb1, da1, db1, ld64(limb_lane + lb + kLimbBlkBytes),
                     ld64(limb_c + lb + kLimbBlkBytes));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == nst) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      // fold the digit columns, sum over the lane quad, and hand the 16 row
      // sums of this warp to the epilogue
      float va = fmaf(acc0.y, w_hi, acc0.x * w_lo);  // row g
      float vb = fmaf(acc1.y, w_hi, acc1.x * w_lo);  // row g + 8
      va += __shfl_xor_sync(0xFFFFFFFFu, va, 1);
      vb += __shfl_xor_sync(0xFFFFFFFFu, vb, 1);
      va += __shfl_xor_sync(0xFFFFFFFFu, va, 2);
      vb += __shfl_xor_sync(0xFFFFFFFFu, vb, 2);
      // lane l < 16 takes row l: g = l (l < 8) or g + 8 (l >= 8), held by lane 4g
      const float sa = __shfl_sync(0xFFFFFFFFu, va, (lane & 7) * 4);
      const float sb = __shfl_sync(0xFFFFFFFFu, vb, (lane & 7) * 4);
      const int b = k % kRed;
      if (!mbar_wait(&rempty[b], (static_cast<uint32_t>(k / kRed) & 1u) ^ 1u, a.budget)) {
        ok = false;
        break;
      }
      if (lane < kRows) red[(b * kConsumers + cw) * kRows + lane] = lane < 8 ? sa : sb;
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[b]);
    }
  }
  if (!ok && lane == 0) {
    report(a.dev_status, GQ_DEV_TIMEOUT);
    *reinterpret_cast<volatile int*>(&flags[0]) = 1;
  }
}

size_t fixed_smem(int nblk) {
  return static_cast<size_t>((nblk * kLimbBlkBytes + 1023) & ~1023) +
         static_cast<size_t>(kRed) * kConsumers * kRows * sizeof(float) +
         (2 * kMaxStages + 2 * kRed + 1) * sizeof(uint64_t) + 16;
}

int stages_for(int nblk) {
  const size_t fixed = fixed_smem(nblk);
  if (fixed >= kSmemBudget) return 0;
  const int n = static_cast<int>((kSmemBudget - fixed) / kStageBytes);
  return n < kMaxStages ? n : kMaxStages;
}

// Workspace: the counts of cut row groups (one int per CTA, zero between
// calls), then two 16-row partial sums per CTA.  The size does not depend on
// the shape, so one workspace serves every call of a stream.
constexpr size_t kCountersBytes = kMaxCtas * sizeof(int);
constexpr size_t kWsBytes = kCountersBytes + static_cast<size_t>(kMaxCtas) * 2 * kRows * sizeof(float);

Split make_split(int64_t M, int64_t K) {
  Split sp;
  sp.Cu = static_cast<int>(K / 32 / kUnitBlk);
  sp.G = static_cast<int>((M + kRows - 1) / kRows);
  sp.U = static_cast<int64_t>(sp.G) * sp.Cu;
  const int sms = sm_count();
  sp.P = static_cast<int>(sp.U < sms ? sp.U : sms);
  return sp;
}

// Scratch of gq_gemv_q4_0_noalloc: the same counts and partial sums as a
// caller's workspace, in static device memory instead.
__device__ __align__(256) uint8_t g_noalloc_scratch[kWsBytes];

}  // namespace

bool i8_shape_ok(int fmt, int64_t M, int64_t K, int64_t B, int xt, const void* W) {
  if (fmt != GQ_FMT_Q4_0 || B != 1 || xt != GQ_F16 || M <= 0) return false;
  if (K <= 0 || K % 256 != 0 || K / 32 > kMaxBlk) return false;  // whole 16-byte granules
  if (reinterpret_cast<uintptr_t>(W) & 15u) return false;
  if (M > (1LL << 30)) return false;
  return stages_for(static_cast<int>(K / 32)) >= 2;
}

bool i8_eligible(int fmt, int64_t M, int64_t K, int64_t B, int xt, const void* W) {
  return i8_shape_ok(fmt, M, K, B, xt, W) && sm_count() <= kMaxCtas;
}

size_t i8_workspace_bytes(int64_t, int64_t) { return kWsBytes; }

gq_status i8_gemv(const void* W, int64_t M, int64_t K, const void* x, void* y, int yt,
                  void* workspace, size_t ws_bytes, bool pdl, int* dev_status,
                  cudaStream_t stream) {
  if (!workspace || ws_bytes < kWsBytes) return GQ_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GQ_ERR_ALIGNMENT;
  const Split sp = make_split(M, K);
  const int nblk = static_cast<int>(K / 32);
  const int nst = stages_for(nblk);
  if (nst < 2) return GQ_ERR_SHAPE;

  EncodeTiled enc = tensor_map_encoder();
  if (!enc) return GQ_ERR_CUDA;
  // W as a 2-D byte matrix: M rows of K/32*18 bytes; a box is one unit,
  // 144 bytes x 16 rows (rows past M read as zeros)
  CUtensorMap wmap;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(nblk) * 18, static_cast<cuuint64_t>(M)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(nblk) * 18};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kUnitRowBytes), static_cast<cuuint32_t>(kRows)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(W), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQ_ERR_CUDA;

  thread_local unsigned long long configured_ctx = 0;  // per host thread and context
  const unsigned long long ctx = context_id();
  if (ctx == 0 || ctx != configured_ctx) {
    if (cudaFuncSetAttribute(gemv_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBudget)) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_ctx = ctx;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  I8Args a;
  a.x = static_cast<const uint16_t*>(x);
  a.M = static_cast<int>(M);
  a.nblk = nblk;
  a.nstages = nst;
  a.sp = sp;
  a.counters = reinterpret_cast<int*>(ws);
  a.partials = reinterpret_cast<float*>(ws + kCountersBytes);
  a.y = y;
  a.ytype = yt;
  a.dev_status = dev_status;
  a.budget = kWaitBudget;
  const size_t smem = fixed_smem(nblk) + static_cast<size_t>(nst) * kStageBytes;
  return launch(gemv_i8_kernel, dim3(sp.P), dim3(kThreads), smem, stream, pdl, wmap, a);
}

}  // namespace gq

namespace gq {

// Address of the static scratch in the calling thread's current context,
// looked up once per context: a context created after another one was
// destroyed (e.g. by cudaDeviceReset) holds the array at a new address.  The
// first call in a context should come before any stream capture.
static gq_status noalloc_scratch(uint8_t** out) {
  static std::mutex mu;
  static unsigned long long ctx_of[64];  // zero: no context seen
  static void* addr_of[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return GQ_ERR_CUDA;
  const unsigned long long ctx = context_id();
  if (dev < 64 && ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    if (ctx_of[dev] == ctx) {
      *out = static_cast<uint8_t*>(addr_of[dev]);
      return GQ_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQ_ERR_CUDA;
  const unsigned long long now = context_id();  // the lookup made a context current if none was
  if (dev < 64 && now != 0) {
    std::lock_guard<std::mutex> lock(mu);
    ctx_of[dev] = now;
    addr_of[dev] = p;
  }
  *out = static_cast<uint8_t*>(p);
  return GQ_OK;
}

gq_status i8_gemv_noalloc(const void* W, int64_t M, int64_t K, const void* x, void* y, int yt,
                          bool pdl, int* dev_status, cudaStream_t stream) {
  if (make_split(M, K).P > kMaxCtas) return GQ_ERR_WORKSPACE;  // beyond the static scratch
  uint8_t* scratch = nullptr;
  const gq_status st = noalloc_scratch(&scratch);
  if (st != GQ_OK) return st;
  // the counts must start at zero: clear them in stream order before the launch
  if (cudaMemsetAsync(scratch, 0, kCountersBytes, stream) != cudaSuccess) return GQ_ERR_CUDA;
  return i8_gemv(W, M, K, x, y, yt, scratch, kWsBytes, pdl, dev_status, stream);
}

}  // namespace gq
