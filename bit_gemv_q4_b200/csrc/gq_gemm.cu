// gq_gemm.cu -- dequantize-fused batched product Y = W_hat * X on the
// tcgen05 tensor cores, for batches large enough to be a dense contraction.
//
// Operation: Y[n][m] = sum_k W_hat[m][k] * X[n][k], with W_hat decoded from
// Q4_0 blocks ("GGUF 量化内幕 第4章" 4.3: d * (code - 8)) or super-blocks
// ("GGUF K-quants" 套娃: (S * q_j) * (code - 8)).  X is bf16, Y fp32/bf16/fp16.
//
// Exactness: a decoded weight has at most 14 significant bits, so it is the
// exact sum of two bfloat16 numbers, hi = its top 8 significant bits and
// lo = the rest.  Both tiles go through the tensor core against the same X
// tile into one fp32 accumulator: every product is exact, only the fp32
// accumulation rounds.
//
// Design (sm_100a; tiles of 128 rows of W with all of the batch as N, cut
// into 64-wide k-steps; one CTA per SM):
//  * work split: the tiles' k-steps are divided evenly over the CTAs
//    (stream-K) when N <= 64, where the number of MMA instructions per SM
//    sets the speed; wider batches give each CTA whole tiles.  A tile cut
//    between CTAs is combined through fp32 partial sums in the workspace:
//    the CTA that completes it sums every part in CTA order (deterministic)
//    and resets the tile's count.  CTAs do their (at most two) cut tiles
//    first.
//  * warp 0 (W producer): streams the tile's packed rows, 512 weights per
//    row per stage -- one 2-D TMA load of 128 rows x 304 bytes when rows are
//    whole 16-byte granules, else one 1-D bulk copy per row (no multicast);
//  * warp 18 (X producer): the X k-slices (64 x N bf16) with a 2-D TMA load
//    in the 128-byte swizzle, on their own ring, so that waiting for a free
//    W stage never delays an activation slice;
//  * warps 2..9 (dequant, one thread per W row and half k-step): decode
//    each k-step into the hi and lo bf16 tiles, written straight into the
//    K-major 128-byte-swizzled UMMA layout, then fence the async proxy;
//  * warp 1 (MMA): allocates two fp32 accumulator buffers in tensor memory
//    and one thread issues tcgen05.mma (M=128, N, K=16) for hi and lo per
//    k16, releasing stages with tcgen05.commit; a tile's buffer alternates
//    so the next tile's MMAs overlap the previous tile's read-back;
//  * warps 10..17 (epilogue, two per TMEM lane quarter): read the
//    accumulator with tcgen05.ld and store Y, or publish and combine the
//    parts of a cut tile.
//  * Every wait is bounded; on expiry the kernel sets GQ_DEV_TIMEOUT, lets
//    its own copies and MMAs land (bounded), frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_gemv.h"
#include "gq_host.h"
#include "gq_tc.cuh"

namespace gq {
namespace {

constexpr int kBM = 128;                       // W rows per tile (UMMA M)
constexpr int kBK = 64;                        // k per A/X stage (128-byte bf16 rows)
constexpr int kWChunk = 512;                   // weights per W row per stage
constexpr int kWPitch = 304;                   // 19 granules >= 12 + 288
constexpr int kWStageBytes = kBM * kWPitch;    // 38 KB, a multiple of 1024
constexpr int kWStages = 2;
constexpr int kAStagesMax = 3;                 // decoded hi/lo tile pairs
constexpr int kXStagesMax = 8;                 // activation k-slices
constexpr int kSmemBudget = 227 * 1024;
constexpr int kATile = kBM * kBK * 2;          // one bf16 tile (hi or lo): 16 KB
constexpr int kStepsPerChunk = kWChunk / kBK;  // 8
constexpr int kDequantWarps = 8;   // two per scheduler; each thread decodes one block per k-step
constexpr int kEpiWarps = 8;       // two per TMEM lane quarter, alternate 16-column slices
constexpr int kXWarp = 2 + kDequantWarps + kEpiWarps;  // the activation producer
constexpr int kThreads = 32 * (kXWarp + 1);

template <int FMT>
struct GFmt;
template <>
struct GFmt<GQ_FMT_Q4_0> {
  static constexpr int kBlkW = 32, kBlkB = 18;
};
template <>
struct GFmt<GQ_FMT_KSB> {
  static constexpr int kBlkW = 256, kBlkB = 138;
};

// Units of work: (tile t of 128 rows, 64-wide k-step ks); S steps per tile,
// U = T * S in all.  CTA i owns units [U*i/P, U*(i+1)/P): an equal share, so
// every SM gets the same number of MMAs.  A CTA's run covers whole tiles and
// at most two cut ones (its first and last), whose fp32 partial sums go
// through the workspace.
struct GSplit {
  int64_t U;
  int S, T, P;
};

struct GemmArgs {
  const uint8_t* W;
  int64_t M, K, rowbytes;
  void* Y;
  int* dev_status;
  long long budget;
  int B, N, ytype, nsteps, nchunks;
  int astages, xstages;  // ring depths chosen from the shared-memory budget
  uint32_t tmem_cols;     // two accumulator buffers of N columns
  int w_tma;              // rows are whole 16-byte granules: one TMA load per W stage
  GSplit sp;
  float* partials;        // [P][2][128][N] fp32 parts of cut tiles
  int* counters;          // [T] k-steps done per cut tile, zero between calls
};

struct Smem {
  uint32_t a, x, w;  // byte offsets of the A, X and W rings
  uint32_t x_stage;  // bytes per X stage
};

extern __shared__ __align__(1024) uint8_t gsm[];

// Ring offsets inside dynamic shared memory, from a 1024-byte-aligned base
// (the 128-byte swizzle atoms and the TMA destinations need that alignment).
__device__ __forceinline__ Smem smem_layout(int N, int astages, int xstages) {
  Smem s;
  const uint32_t base = smem_addr(gsm);
  s.a = ((base + 1023u) & ~1023u) - base;
  s.x = s.a + astages * 2 * kATile;
  s.x_stage = static_cast<uint32_t>(N) * kBK * 2;
  s.w = s.x + xstages * s.x_stage;
  return s;
}

__device__ __forceinline__ uint32_t g_ld32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(gsm + off);
}
__device__ __forceinline__ uint32_t g_ld16(uint32_t off) {
  return *reinterpret_cast<const uint16_t*>(gsm + off);
}

// Eight decoded weights in two float2-packed halves -> one 16-byte chunk of
// the hi tile and one of the lo tile.  A decoded weight has at most 14
// significant bits, so hi (its top bfloat16 bits, by truncation) and
// lo = w - hi are both exact bfloat16 numbers.
__device__ __forceinline__ void split8(const float2 w[4], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t u0 = __float_as_uint(w[p].x), u1 = __float_as_uint(w[p].y);
    const float2 hf = make_float2(__uint_as_float(u0 & 0xFFFF0000u), __uint_as_float(u1 & 0xFFFF0000u));
    const float2 lf = __ffma2_rn(hf, make_float2(-1.0f, -1.0f), w[p]);  // w - hi, exact
    h[p] = __byte_perm(u0, u1, 0x7632u);
    l[p] = __byte_perm(__float_as_uint(lf.x), __float_as_uint(lf.y), 0x7632u);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Weights s * (code - 8) for the eight nibbles held, one per byte, in
// (m0, m1) -- low nibbles in place (HI = false) or high nibbles left at bits
// 4..7 (HI = true, values 16 * code).  PRMT drops each byte into the mantissa
// of 2^23, so a float add removes the bias exactly: (2^23 + c) - (2^23 + 8)
// = c - 8, or (2^23 + 16c) - (2^23 + 128) = 16 (c - 8) with s / 16 folded in.
template <bool HI>
__device__ __forceinline__ void decode8(uint32_t m0, uint32_t m1, float2 s2, uint4& hi, uint4& lo) {
  const float bias = HI ? -8388736.0f : -8388616.0f;  // -(2^23 + 128), -(2^23 + 8)
  const float2 b2 = make_float2(bias, bias);
  float2 w[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t src = (p < 2) ? m0 : m1;
    const uint32_t sel0 = 0x7440u | (2 * (p & 1)), sel1 = 0x7440u | (2 * (p & 1) + 1);
    const float2 f = make_float2(__uint_as_float(__byte_perm(src, 0x4B000000u, sel0)),
                                 __uint_as_float(__byte_perm(src, 0x4B000000u, sel1)));
    w[p] = __fmul2_rn(__fadd2_rn(f, b2), s2);
  }
  split8(w, hi, lo);
}

// Store chunk c (k = 8c .. 8c+7 of the 64-wide step) of row `row` into a
// K-major 128-byte-swizzled bf16 tile.
__device__ __forceinline__ void st_chunk(uint32_t tile, int row, int c, uint4 v) {
  const uint32_t off = tile + (row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4);
  *reinterpret_cast<uint4*>(gsm + off) = v;
}

// 16 code bytes at an even shared offset, as four words.
__device__ __forceinline__ void load_codes(uint32_t qs, uint32_t q[4]) {
  const uint32_t b = qs & ~3u;
  const uint32_t sel = (qs & 2u) ? 0x5432u : 0x3210u;
  uint32_t w[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) w[i] = g_ld32(b + 4 * i);
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = __byte_perm(w[i], w[i + 1], sel);
}

// Decode one 32-weight block (scale s, 16 code bytes at `qs`) into chunks
// c0 .. c0+3 of the hi and lo tiles: weights j and j+16 are the low and high
// nibbles of code byte j.
__device__ __forceinline__ void block_to_tiles(uint32_t qs, float s, uint32_t a_hi, uint32_t a_lo,
                                               int row, int c0) {
  uint32_t q[4];
  load_codes(qs, q);
  const float2 s1 = make_float2(s, s);
  const float2 s16 = make_float2(s * 0.0625f, s * 0.0625f);  // exact power-of-two scaling
  uint4 h, l;
  decode8<false>(q[0] & 0x0F0F0F0Fu, q[1] & 0x0F0F0F0Fu, s1, h, l);  // weights 0..7
  st_chunk(a_hi, row, c0 + 0, h);
  st_chunk(a_lo, row, c0 + 0, l);
  decode8<false>(q[2] & 0x0F0F0F0Fu, q[3] & 0x0F0F0F0Fu, s1, h, l);  // weights 8..15
  st_chunk(a_hi, row, c0 + 1, h);
  st_chunk(a_lo, row, c0 + 1, l);
  decode8<true>(q[0] & 0xF0F0F0F0u, q[1] & 0xF0F0F0F0u, s16, h, l);  // weights 16..23
  st_chunk(a_hi, row, c0 + 2, h);
  st_chunk(a_lo, row, c0 + 2, l);
  decode8<true>(q[2] & 0xF0F0F0F0u, q[3] & 0xF0F0F0F0u, s16, h, l);  // weights 24..31
  st_chunk(a_hi, row, c0 + 3, h);
  st_chunk(a_lo, row, c0 + 3, l);
}

__device__ __forceinline__ void zero_chunks(uint32_t a_hi, uint32_t a_lo, int row, int c0) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    st_chunk(a_hi, row, c0 + i, z);
    st_chunk(a_lo, row, c0 + i, z);
  }
}

__device__ __forceinline__ int64_t g_unit_begin(const GSplit& sp, int i) {
  return sp.U * i / sp.P;
}
__device__ __forceinline__ int g_unit_owner(const GSplit& sp, int64_t u) {
  const int64_t i = ((u + 1) * sp.P - 1) / sp.U;
  return static_cast<int>(i < sp.P - 1 ? i : sp.P - 1);
}

// This CTA's tiles ta..tb, with the k-step range of each, in processing
// order: the first and last tile (the ones other CTAs share) before the
// whole tiles between them, so that shared tiles complete early.
struct GSegs {
  int ta, tb, S;
  int64_t u0, u1;
  __device__ __forceinline__ int count() const { return tb - ta + 1; }
  __device__ __forceinline__ void get(int k, int& t, int& k0, int& k1) const {
    t = (k == 0) ? ta : (k == 1) ? tb : ta + k - 1;
    k0 = (t == ta) ? static_cast<int>(u0 - static_cast<int64_t>(ta) * S) : 0;
    k1 = (t == tb) ? static_cast<int>(u1 - static_cast<int64_t>(tb) * S) : S;
  }
};

__device__ __forceinline__ GSegs g_segs(const GSplit& sp, int i) {
  GSegs g;
  g.S = sp.S;
  g.u0 = g_unit_begin(sp, i);
  g.u1 = g_unit_begin(sp, i + 1);
  g.ta = static_cast<int>(g.u0 / sp.S);
  g.tb = static_cast<int>((g.u1 - 1) / sp.S);
  return g;
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                const GemmArgs a) {
  constexpr int kBlkW = GFmt<FMT>::kBlkW, kBlkB = GFmt<FMT>::kBlkB;
  constexpr int kChunkBytes = kWChunk / kBlkW * kBlkB;  // 288 or 276
  const int kAStages = a.astages, kXStages = a.xstages;
  const Smem L = smem_layout(a.N, kAStages, kXStages);
  const uint32_t sbase = smem_addr(gsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gsm + L.w + kWStages * kWStageBytes);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + kWStages;
  uint64_t* a_full = w_empty + kWStages;
  uint64_t* a_empty = a_full + kAStagesMax;
  uint64_t* x_full = a_empty + kAStagesMax;
  uint64_t* x_empty = x_full + kXStagesMax;
  uint64_t* d_full = x_empty + kXStagesMax;  // [2] accumulator buffer ready
  uint64_t* d_empty = d_full + 2;            // [2] accumulator buffer read back
  uint64_t* d_done = d_empty + 2;            // every MMA of the CTA finished
  uint64_t* e_bar = d_done + 1;              // epilogue warps' group barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(e_bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nblk_row = a.K / kBlkW;
  const GSegs sg = g_segs(a.sp, blockIdx.x);
  const int nseg = sg.count();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], kDequantWarps);
    }
    for (int i = 0; i < kAStagesMax; ++i) {
      mbar_init(&a_full[i], kDequantWarps);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kXStagesMax; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kEpiWarps);
    }
    mbar_init(d_done, 1);
    mbar_init(e_bar, kEpiWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(abort_flag) != 0; };
  auto fail = [&]() {
    report(a.dev_status, GQ_DEV_TIMEOUT);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------- W producer
    // Per segment, the W chunks (512 weights of the tile's 128 rows) of its
    // k-steps.  The X k-slices come from their own warp (kXWarp), so that a
    // wait for a free W stage never holds back an activation load.
    int wseq = 0, g = 0;
    bool ok = true;
    for (int k = 0; k < nseg && ok; ++k) {
      int t, k0, k1;
      sg.get(k, t, k0, k1);
      const int64_t m0 = static_cast<int64_t>(t) * kBM;
      for (int ks = k0; ks < k1; ++ks, ++g) {
        if (ks == k0 || ks % kStepsPerChunk == 0) {
          const int s = wseq % kWStages;
          if (!mbar_wait(&w_empty[s], ((wseq / kWStages) & 1u) ^ 1u, a.budget) || aborted()) {
            ok = false;
            break;
          }
          const int64_t b0 = static_cast<int64_t>(ks / kStepsPerChunk) * (kWChunk / kBlkW);
          if (a.w_tma) {
            // the 128 rows x 304 bytes (19 granules) that hold the chunk; rows
            // past M and bytes past the row end read as zeros
            if (lane == 0) {
              mbar_arrive_expect_tx(&w_full[s], kWStageBytes);
              tma_load_2d_hint(gsm + L.w + s * kWStageBytes, &wmap,
                               static_cast<int>((b0 * kBlkB) >> 4) * 2, static_cast<int>(m0),
                               &w_full[s], policy_evict_first());
            }
            __syncwarp();
          } else {
            const uint32_t nbytes =
                static_cast<uint32_t>(i64min(kWChunk / kBlkW, nblk_row - b0) * kBlkB);
            uint32_t total = 0;
            uintptr_t lo[4];
            uint32_t len[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = lane + 32 * i;
              len[i] = 0;
              if (m0 + r < a.M) {
                const uintptr_t src = reinterpret_cast<uintptr_t>(a.W) +
                                      static_cast<uintptr_t>((m0 + r) * a.rowbytes + b0 * kBlkB);
                lo[i] = src & ~static_cast<uintptr_t>(15);
                len[i] = static_cast<uint32_t>(((src + nbytes + 15) & ~static_cast<uintptr_t>(15)) - lo[i]);
              }
              total += len[i];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xFFFFFFFFu, total, o);
            if (lane == 0) mbar_arrive_expect_tx(&w_full[s], total);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (len[i])
                bulk_g2s(gsm + L.w + s * kWStageBytes + (lane + 32 * i) * kWPitch,
                         reinterpret_cast<const void*>(lo[i]), len[i], &w_full[s],
                         policy_evict_first());
          }
          ++wseq;
        }
      }
    }
    if (!ok && lane == 0) fail();
    // let every issued copy land before shared memory is released
    if (lane == 0) {
      for (int c = max(0, wseq - kWStages); c < wseq; ++c)
        if (!mbar_wait(&w_full[c % kWStages], (c / kWStages) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, a.N);
      bool ok = true;
      int g = 0;
      for (int k = 0; k < nseg && ok; ++k) {
        int t, k0, k1;
        sg.get(k, t, k0, k1);
        const int buf = k & 1;
        // the epilogue has read this accumulator buffer (two segments ago)
        if (!mbar_wait(&d_empty[buf], ((k >> 1) & 1u) ^ 1u, a.budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem_d + static_cast<uint32_t>(buf * a.N);
        for (int ks = k0; ks < k1; ++ks, ++g) {
          const int sa = g % kAStages, sx = g % kXStages;
          if (!mbar_wait(&a_full[sa], (g / kAStages) & 1u, a.budget) ||
              !mbar_wait(&x_full[sx], (g / kXStages) & 1u, a.budget) || aborted()) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_hi = sbase + L.a + sa * 2 * kATile, a_lo = a_hi + kATile;
          const uint32_t xs = sbase + L.x + sx * L.x_stage;
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) {
            const uint64_t xd = umma_desc_sw128(xs + 32 * k16);
            umma_bf16(dacc, umma_desc_sw128(a_hi + 32 * k16), xd, idesc, (ks != k0 || k16 != 0));
            umma_bf16(dacc, umma_desc_sw128(a_lo + 32 * k16), xd, idesc, 1u);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&x_empty[sx]);
        }
        if (!ok) break;
        umma_commit(&d_full[buf]);
      }
      if (!ok) fail();
      // d_done completes once every MMA issued above has finished (also on the
      // abort path, so that TMEM and shared memory are quiet before exit)
      umma_commit(d_done);
    }
    __syncwarp();
  } else if (warp < 2 + kDequantWarps) {
    // ----------------------------------------------------------- dequant
    const int row = (warp & 3) * 32 + lane;
    const int half = (warp - 2) >> 2;  // which 32-weight block of each k-step
    bool ok = true;
    int wseq = 0, g = 0, sw = 0;
    for (int k = 0; k < nseg && ok; ++k) {
      int t, k0, k1;
      sg.get(k, t, k0, k1);
      const int64_t m0 = static_cast<int64_t>(t) * kBM;
      const bool row_ok = m0 + row < a.M;
      const uintptr_t row_addr = reinterpret_cast<uintptr_t>(a.W) +
                                 static_cast<uintptr_t>((m0 + (row_ok ? row : 0)) * a.rowbytes);
      for (int ks = k0; ks < k1; ++ks, ++g) {
        const int c = ks / kStepsPerChunk, j = ks % kStepsPerChunk;
        if (ks == k0 || j == 0) {
          sw = wseq % kWStages;
          if (!mbar_wait(&w_full[sw], (wseq / kWStages) & 1u, a.budget) || aborted()) {
            ok = false;
            break;
          }
          ++wseq;
        }
        const int sa = g % kAStages;
        if (!mbar_wait(&a_empty[sa], ((g / kAStages) & 1u) ^ 1u, a.budget) || aborted()) {
          ok = false;
          break;
        }
        const uint32_t a_hi = L.a + sa * 2 * kATile, a_lo = a_hi + kATile;
        // this row's piece of the chunk, from its offset inside the first granule
        const uint32_t slot = L.w + sw * kWStageBytes + row * kWPitch +
                              static_cast<uint32_t>((row_addr + static_cast<uintptr_t>(c) * kChunkBytes) & 15u);
        const int64_t blk0 = static_cast<int64_t>(c) * (kWChunk / kBlkW);  // first block of the chunk
        if constexpr (FMT == GQ_FMT_Q4_0) {
          const int jb = 2 * j + half;  // block within the chunk
          if (blk0 + jb < nblk_row) {
            const uint32_t o = slot + jb * 18;
            block_to_tiles(o + 2, half_bits_to_float(g_ld16(o)), a_hi, a_lo, row, 4 * half);
          } else {
            zero_chunks(a_hi, a_lo, row, 4 * half);
          }
        } else {
          const int sb = j >> 2;  // super-block within the chunk
          const uint32_t o = slot + sb * 138;
          if (blk0 + sb < nblk_row) {
            const int sub = 2 * (j & 3) + half;
            const float S = half_bits_to_float(g_ld16(o));
            const uint32_t qw = g_ld16(o + 2 + (sub & ~1));
            const int qj = static_cast<int8_t>((qw >> (8 * (sub & 1))) & 0xFFu);
            block_to_tiles(o + 10 + 16 * sub, __fmul_rn(S, static_cast<float>(qj)), a_hi, a_lo, row,
                           4 * half);
          } else {
            zero_chunks(a_hi, a_lo, row, 4 * half);
          }
        }
        fence_proxy_async_smem();  // generic writes -> visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_full[sa]);
          if (j == kStepsPerChunk - 1 || ks == k1 - 1) mbar_arrive(&w_empty[sw]);
        }
      }
    }
    if (!ok && lane == 0) fail();
  } else if (warp < kXWarp) {
    // ---------------------------------------------------------- epilogue
    // TMEM lane quarter = warp % 4: warps 10..17 cover the 128 rows twice,
    // each pair of warps on one quarter splitting the columns
    const int row = (warp & 3) * 32 + lane;
    const int col0 = 16 * ((warp - 2 - kDequantWarps) >> 2);  // 0 or 16
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const bool leader = (warp == 2 + kDequantWarps) && lane == 0;
    bool ok = true;
    uint32_t ephase = 0;
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(e_bar);
      const bool done = mbar_wait(e_bar, ephase & 1u, a.budget);
      ++ephase;
      return done;
    };
    for (int k = 0; k < nseg; ++k) {
      int t, k0, k1;
      sg.get(k, t, k0, k1);
      const int buf = k & 1;
      if (!mbar_wait(&d_full[buf], (k >> 1) & 1u, a.budget) || aborted()) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t m0 = static_cast<int64_t>(t) * kBM;
      const bool row_ok = m0 + row < a.M;
      const bool cut = (k1 - k0) < a.sp.S;
      const int slot = (t == sg.ta) ? 0 : 1;
      // a part is [128 rows][N] fp32: each thread's row is contiguous
      float* part = a.partials + ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * kBM + row) * a.N;
      for (int n0 = col0; n0 < a.N; n0 += 32) {
        uint32_t v[16];
        tmem_ld16(tmem_d + lane_base + static_cast<uint32_t>(buf * a.N + n0), v);
        tmem_wait_ld();
        if (!cut) {
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n0 + i < a.B)
                store_elem(a.Y, static_cast<int64_t>(n0 + i) * a.M + m0 + row, __uint_as_float(v[i]), a.ytype);
          }
        } else if (n0 < a.B) {
          uint4* dst = reinterpret_cast<uint4*>(part + n0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[buf]);  // the MMA may refill this buffer
      if (!cut) continue;
      // a tile cut between CTAs: publish this part; the CTA that completes
      // the tile sums every part in CTA order and resets the count
      __threadfence();
      if (!epi_sync()) {
        ok = false;
        break;
      }
      if (leader)
        *reinterpret_cast<volatile int*>(last_flag) =
            (atomicAdd(&a.counters[t], k1 - k0) + (k1 - k0) == a.sp.S);
      if (!epi_sync()) {
        ok = false;
        break;
      }
      if (!*reinterpret_cast<volatile int*>(last_flag)) continue;
      __threadfence();
      const int64_t ufirst = static_cast<int64_t>(t) * a.sp.S;
      const int i0 = g_unit_owner(a.sp, ufirst), i1 = g_unit_owner(a.sp, ufirst + a.sp.S - 1);
      for (int n0 = col0; n0 < a.B; n0 += 32) {
        float acc[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) acc[u] = 0.f;
        for (int i = i0; i <= i1; ++i) {
          const int sl = (g_unit_begin(a.sp, i) / a.sp.S == t) ? 0 : 1;
          const float4* src = reinterpret_cast<const float4*>(
              a.partials + ((static_cast<int64_t>(i) * 2 + sl) * kBM + row) * a.N + n0);
          float4 v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) v[q] = __ldcg(src + q);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[4 * q] += v[q].x;
            acc[4 * q + 1] += v[q].y;
            acc[4 * q + 2] += v[q].z;
            acc[4 * q + 3] += v[q].w;
          }
        }
        if (row_ok) {
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (n0 + u < a.B) store_elem(a.Y, static_cast<int64_t>(n0 + u) * a.M + m0 + row, acc[u], a.ytype);
        }
      }
      if (leader) a.counters[t] = 0;
    }
    if (!ok && lane == 0) fail();
  } else {
    // ------------------------------------------------------- X producer
    // the X k-slice (64 x N bf16, 128-byte swizzle) of every k-step, in the
    // MMA's order, as far ahead as the X ring allows
    int g = 0;
    bool ok = true;
    for (int k = 0; k < nseg && ok; ++k) {
      int t, k0, k1;
      sg.get(k, t, k0, k1);
      for (int ks = k0; ks < k1; ++ks, ++g) {
        const int sx = g % kXStages;
        if (!mbar_wait(&x_empty[sx], ((g / kXStages) & 1u) ^ 1u, a.budget) || aborted()) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&x_full[sx], L.x_stage);
          tma_load_2d(gsm + L.x + sx * L.x_stage, &xmap, ks * kBK, 0, &x_full[sx]);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) fail();
    // let every issued copy land before shared memory is released
    if (lane == 0) {
      for (int k = max(0, g - kXStages); k < g; ++k)
        if (!mbar_wait(&x_full[k % kXStages], (k / kXStages) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
    }
  }

  // teardown: every MMA has finished before tensor memory is freed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && !mbar_wait(d_done, 0, a.budget)) report(a.dev_status, GQ_DEV_TIMEOUT);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, a.tmem_cols);
  }
}

size_t gemm_smem_bytes(int N, int astages, int xstages) {
  return static_cast<size_t>(astages) * 2 * kATile + static_cast<size_t>(xstages) * N * kBK * 2 +
         static_cast<size_t>(kWStages) * kWStageBytes +
         (2 * kWStages + 2 * kAStagesMax + 2 * kXStagesMax + 6) * sizeof(uint64_t) + 16 + 1024;
}

// Deepest rings that fit: activations first (their loads wait on the MMA of
// the slot they refill), then a third decoded-tile stage if room is left.
// A third decoded-tile stage decouples the dequant warps from the MMA more
// than X stages beyond four help (X has its own producer), so it is taken
// first when it fits.
void choose_stages(int N, int& astages, int& xstages) {
  const auto fits = [&](int as, int xs) {
    return gemm_smem_bytes(N, as, xs) <= static_cast<size_t>(kSmemBudget);
  };
  for (astages = kAStagesMax; astages > 2; --astages) {
    for (xstages = kXStagesMax; xstages >= 4 && !fits(astages, xstages); --xstages) {
    }
    if (xstages >= 4) return;
  }
  astages = 2;
  xstages = kXStagesMax;
  while (xstages > 2 && !fits(astages, xstages)) --xstages;
}

// The work split and the workspace it needs: counts of the cut tiles (one
// int per tile, zero between calls) then two fp32 parts of 128 x N per CTA.
// Narrow batches (N <= 64) are bound by the number of MMA instructions per
// SM, so their units are spread over every SM; wider ones are bound by the
// tensor rate, where the exchange of 128 x N partial sums would cost more
// than the idle SMs, so each CTA then takes whole tiles.
constexpr int kSplitMaxN = 64;

GSplit gemm_split(int64_t M, int64_t K, int N) {
  GSplit sp;
  sp.T = static_cast<int>((M + kBM - 1) / kBM);
  sp.S = static_cast<int>((K + kBK - 1) / kBK);
  sp.U = static_cast<int64_t>(sp.T) * sp.S;
  const int64_t ctas = (N <= kSplitMaxN) ? static_cast<int64_t>(sm_count()) : sp.T;
  sp.P = static_cast<int>(sp.U < ctas ? sp.U : ctas);
  return sp;
}

size_t ws_round(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

size_t gemm_ws_bytes(int64_t M, int64_t K, int N, size_t* parts_off) {
  const GSplit sp = gemm_split(M, K, N);
  const size_t counters = ws_round(static_cast<size_t>(sp.T) * sizeof(int));
  if (parts_off) *parts_off = counters;
  return counters + ws_round(static_cast<size_t>(sp.P) * 2 * N * kBM * sizeof(float));
}

template <int FMT>
gq_status gemm_entry(const void* W, int64_t M, int64_t K, const void* X, int xt, int64_t B, void* Y,
                     int yt, void* workspace, size_t ws_bytes, int* dev_status, void* stream) {
  constexpr int kBlkW = GFmt<FMT>::kBlkW, kBlkB = GFmt<FMT>::kBlkB;
  if (M < 0 || K < 0 || B < 0) return GQ_ERR_INVALID_ARG;
  if (xt != GQ_BF16 || !valid_act_dtype(yt)) return GQ_ERR_DTYPE;
  if (K % kBlkW) return GQ_ERR_SHAPE;
  if (B > 256 || M > 0x7FFFFFFFLL || K > (1LL << 24)) return GQ_ERR_SHAPE;
  if (M == 0 || B == 0) return GQ_OK;
  if (!Y) return GQ_ERR_INVALID_ARG;
  if (misaligned16(Y)) return GQ_ERR_ALIGNMENT;
  if (K == 0) {
    return cudaMemsetAsync(Y, 0, static_cast<size_t>(B * M * dtype_size(yt)), as_stream(stream)) ==
                   cudaSuccess
               ? GQ_OK
               : GQ_ERR_CUDA;
  }
  if (!W || !X) return GQ_ERR_INVALID_ARG;
  if (misaligned16(W) || misaligned16(X)) return GQ_ERR_ALIGNMENT;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return GQ_ERR_ALIGNMENT;
  const int N = static_cast<int>((B + 15) / 16 * 16);
  size_t parts_off = 0;
  const size_t need = gemm_ws_bytes(M, K, N, &parts_off);
  if (!workspace || ws_bytes < need) return GQ_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GQ_ERR_ALIGNMENT;
  // narrow batches: the warp-MMA product (every weight decoded once for all
  // columns, no tcgen05 instruction per 16 columns)
  if (B <= kWarpMmaMaxB)
    return gemv_batched(FMT, W, M, K, X, xt, B, Y, yt, dev_status, as_stream(stream));

  EncodeTiled enc = tensor_map_encoder();
  if (!enc) return GQ_ERR_CUDA;
  CUtensorMap xmap;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(B)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(N)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQ_ERR_CUDA;

  // W as rows of 8-byte elements when rows are whole 16-byte granules: a W
  // stage is then one box of 38 elements (304 bytes) x 128 rows, already at
  // the row pitch the dequant warps read
  const int64_t rowbytes = K / kBlkW * kBlkB;
  const bool w_tma = (rowbytes % 16 == 0) && rowbytes >= kWPitch && M >= kBM;
  CUtensorMap wmap = {};
  if (w_tma) {
    const cuuint64_t wdim[2] = {static_cast<cuuint64_t>(rowbytes / 8), static_cast<cuuint64_t>(M)};
    const cuuint64_t wstride[1] = {static_cast<cuuint64_t>(rowbytes)};
    const cuuint32_t wbox[2] = {static_cast<cuuint32_t>(kWPitch / 8), static_cast<cuuint32_t>(kBM)};
    const cuuint32_t westride[2] = {1, 1};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(W), wdim, wstride, wbox,
            westride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQ_ERR_CUDA;
  }

  GemmArgs a;
  a.w_tma = w_tma ? 1 : 0;
  a.W = static_cast<const uint8_t*>(W);
  a.M = M;
  a.K = K;
  a.rowbytes = K / kBlkW * kBlkB;
  a.Y = Y;
  a.dev_status = dev_status;
  a.budget = kWaitBudget;
  a.B = static_cast<int>(B);
  a.N = N;
  a.ytype = yt;
  a.nsteps = static_cast<int>((K + kBK - 1) / kBK);
  a.nchunks = static_cast<int>((K + kWChunk - 1) / kWChunk);
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * N)) cols <<= 1;  // two accumulator buffers
  a.tmem_cols = cols;
  a.sp = gemm_split(M, K, N);
  a.counters = static_cast<int*>(workspace);
  a.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + parts_off);

  choose_stages(N, a.astages, a.xstages);
  const size_t smem = gemm_smem_bytes(N, a.astages, a.xstages);
  thread_local unsigned long long configured_ctx = 0;  // per host thread and context
  const unsigned long long ctx = context_id();
  if (ctx == 0 || ctx != configured_ctx) {
    if (cudaFuncSetAttribute(gemm_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBudget) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_ctx = ctx;
  }
  return launch(gemm_kernel<FMT>, dim3(static_cast<unsigned>(a.sp.P)), dim3(kThreads), smem,
                as_stream(stream), false, xmap, wmap, a);
}

}  // namespace
}  // namespace gq

extern "C" {

GQ_API size_t gq_gemm_workspace_bytes(int fmt, int64_t M, int64_t K, int64_t B) {
  if (fmt != GQ_FMT_Q4_0 && fmt != GQ_FMT_KSB) return 0;
  if (M <= 0 || K <= 0 || B <= 0 || B > 256) return 0;
  return gq::gemm_ws_bytes(M, K, static_cast<int>((B + 15) / 16 * 16), nullptr);
}

GQ_API gq_status gq_gemm_q4_0(const void* W, int64_t M, int64_t K, const void* X, int x_dtype,
                              int64_t B, void* Y, int y_dtype, void* workspace, size_t ws_bytes,
                              int* dev_status, void* stream) {
  return gq::gemm_entry<GQ_FMT_Q4_0>(W, M, K, X, x_dtype, B, Y, y_dtype, workspace, ws_bytes,
                                     dev_status, stream);
}

GQ_API gq_status gq_gemm_ksb(const void* W, int64_t M, int64_t K, const void* X, int x_dtype,
                             int64_t B, void* Y, int y_dtype, void* workspace, size_t ws_bytes,
                             int* dev_status, void* stream) {
  return gq::gemm_entry<GQ_FMT_KSB>(W, M, K, X, x_dtype, B, Y, y_dtype, workspace, ws_bytes,
                                    dev_status, stream);
}

}  // extern "C"
