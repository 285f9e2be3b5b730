// gq_gemv.cu -- dequantize-fused matrix-vector product for decode,
// y[b][m] = sum_k W_hat[m][k] * x[b][k], for 1..8 activation vectors.
//
// Operation: the matrix multiply that consumes decoded blocks ("GGUF 量化内幕
// 第4章" 4.3: w = d * (code - 8); "GGUF K-quants" 套娃: s~_j = S * q_j), in the
// memory-bound decode setting (TurboQuant W4A8 post, section 2.3).
//
// Design (sm_100a):
//  * Work unit: a group of 16 consecutive rows (one m16 MMA tile) over all of
//    K.  The rows of a group are contiguous in HBM.  CTAs are persistent and
//    take groups g = blockIdx.x, blockIdx.x + gridDim.x, ...
//  * Warp 0 produces: for each K chunk of 1024 weights of a group it issues
//    one 1-D bulk async copy (cp.async.bulk, no multicast) per row into a
//    6-stage shared-memory ring, completion tracked by mbarrier transaction
//    counts, running ahead across group boundaries.  Row pieces need not be
//    16-byte aligned (18-byte / 138-byte blocks): a copy covers the enclosing
//    16-byte granules and consumers index from the piece's offset.
//  * Warps 1..8 consume: each takes an eighth of every chunk, decodes the
//    4-bit codes straight into MMA A fragments (code - 8, exactly, by
//    exponent-bias tricks on packed halves) and runs warp MMA m16n8k16 with
//    fp32 accumulation.  Batch columns are the MMA's N dimension (N = 8
//    covers B <= 8; with B = 1 every column holds the same vector).  Each
//    block has its own scale, so the two MMAs of a 32-weight block write a
//    fresh fragment that is scaled and added in fp32: all products are exact
//    (4-bit integer x fp16/bf16), no weight is ever rounded.
//  * When every row starts on a 16-byte boundary (Q4_0 with K % 256 == 0,
//    ksb with K % 2048 == 0) all byte offsets inside a stage are known at
//    compile time; otherwise they are taken per row at run time.
//  * fp32 activations are split exactly into three bfloat16 terms (three MMAs
//    per k-step); fp16 and bf16 activations use one.  Activations sit in
//    shared memory in B-fragment order (one 16-byte load per lane per block)
//    and are loaded once per CTA when they fit, else per window.
//  * Batches whose activations do not fit beside the ring at one CTA per SM
//    run gemv_split_kernel: K is split over a thread-block cluster of 2..8
//    CTAs, each holding its slice of x, and rank 0 adds the ranks' fp32 sums
//    in rank order through distributed shared memory.
//  * Programmatic dependent launch: the producer streams W at once; consumers
//    wait for the preceding grid before reading x or writing y.
//  * Every wait is bounded; on expiry the kernel sets GQ_DEV_TIMEOUT, drains
//    its own in-flight copies (bounded) and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_gemv.h"
#include "gq_gemv_i8.h"
#include "gq_host.h"

namespace gq {
namespace {

#ifndef GQ_GEMV_CHUNK
#define GQ_GEMV_CHUNK 2048
#endif
#ifndef GQ_GEMV_STAGES
#define GQ_GEMV_STAGES 4
#endif

#ifndef GQ_GEMV_CONSUMERS
#define GQ_GEMV_CONSUMERS 8
#endif
#ifndef GQ_GEMV_MINB
#define GQ_GEMV_MINB 2
#endif

constexpr int kRows = 16;                           // rows per group (MMA M)
constexpr int kConsumers = GQ_GEMV_CONSUMERS;       // consumer warps
constexpr int kThreads = 32 * (1 + kConsumers);
constexpr int kChunkW = GQ_GEMV_CHUNK;              // weights per row per stage
constexpr int kSubPerWarp = kChunkW / 32 / kConsumers;  // 32-weight blocks per warp
// bytes per row slot: the row piece plus up to 14 bytes of leading offset,
// rounded to 16, and chosen so that rows r = 0..7 fall on distinct banks
constexpr int kPitch = (kChunkW == 1024) ? 592 : 1168;
constexpr int kStageBytes = kRows * kPitch + 16;    // +16: window-read slack
constexpr int kStages = GQ_GEMV_STAGES;
constexpr int kXBlk = 64;                           // B-fragment bytes per 32 weights
constexpr int kXStride = (kChunkW / 32) * kXBlk + 64;  // per (chunk, batch row), padded
// The batch occupies NT n8 tiles of the MMA's N dimension: NT = 0 is one
// activation vector (with its own fragment layout, x_frag), NT = 1 covers
// B <= 8 and NT = 2 covers B <= 16.  Fragments and accumulators hold four
// floats per tile.
constexpr int acc_len(int nt) { return 4 * (nt > 1 ? nt : 1); }
constexpr int kMaxNT = 2;
// cross-warp reduction buffer of a launch with NT tiles (two groups in flight)
constexpr int red_bytes(int nt) { return 2 * kConsumers * 32 * acc_len(nt) * 4; }
constexpr int kRedBytes = red_bytes(kMaxNT);  // the largest
// exchange slots of a cluster's K split (groups one rank may run ahead)
constexpr int kSplitSlots = 4;
// activation window budget: what the stages and the reduction leave of the
// 227 KB a CTA may hold, at most 72 KB
constexpr int kXSmemFree = 227 * 1024 - kStages * kStageBytes - kRedBytes - 1024;
constexpr int kXSmemMax = kXSmemFree < 72 * 1024 ? kXSmemFree : 72 * 1024;
static_assert(kXSmemMax >= 16 * 1024, "pipeline shape");
static_assert(kChunkW == 1024 || kChunkW == 2048, "supported chunk sizes");
static_assert(kSubPerWarp % 2 == 0, "blocks per warp come in pairs");

enum { XT_F16 = 0, XT_BF16 = 1, XT_F32 = 2 };

// Smallest batch that keeps all of x resident beyond the window budget.  The
// large-table configuration keeps its windows so that its small CTAs stay
// several per SM.
#if GQ_GEMV_MANY_TU
constexpr int kResidentMinB = 9;
#else
constexpr int kResidentMinB = 2;
#endif


template <int FMT>
struct Fmt;
template <>
struct Fmt<GQ_FMT_Q4_0> {
  static constexpr int kBlkW = 32, kBlkB = 18;
};
template <>
struct Fmt<GQ_FMT_KSB> {
  static constexpr int kBlkW = 256, kBlkB = 138;
};

struct GemvArgs {
  const uint8_t* W;
  int64_t M, K, rowbytes;
  const void* x;
  void* y;
  int* dev_status;
  long long budget;
  int B, ytype, nchunks, win, ngroups;  // win: chunks per activation window
  int skip_first;  // self-test only: never fill the first stage, so waits run out
  // K split over a cluster: chunks per CTA, and the shared-memory offset of
  // the exchange area (barriers, then the partial sums)
  int split_cps;
  uint32_t split_off;
};

// Matrices of one launch.  A single product reads W, M and y from GemvArgs
// (NoTable); a grouped product (several matrices sharing K and x) numbers
// the 16-row groups of all its matrices consecutively and finds a group's
// matrix in a table passed by value (GemvTable, read from the kernel's
// parameter space).
struct NoTable {
  int unused;
};
constexpr int kMaxMats = 256;  // matrices per grouped launch
struct GemvMat {
  const uint8_t* W;
  void* y;
  int64_t M;
  int gend;  // groups of matrices 0..i
  int pad;
};
struct GemvTable {
  GemvMat m[kMaxMats];
};

struct Unit {
  const uint8_t* W;
  void* y;
  int64_t M, m0;  // the matrix and the first row of the group
};

// The matrix of group g.  Each CTA visits groups in increasing order, so
// its cursor mi only moves forward.
template <class Tbl>
__device__ __forceinline__ Unit unit_of(const GemvArgs& a, const Tbl& tbl, int g, int& mi) {
  if constexpr (sizeof(Tbl) == sizeof(NoTable)) {
    return Unit{a.W, a.y, a.M, static_cast<int64_t>(g) * kRows};
  } else {
    while (g >= tbl.m[mi].gend) ++mi;
    const int gb = mi ? tbl.m[mi - 1].gend : 0;
    return Unit{tbl.m[mi].W, tbl.m[mi].y, tbl.m[mi].M, static_cast<int64_t>(g - gb) * kRows};
  }
}

// ---- decode 8 codes (one 32-bit word = qs[4t..4t+3]) into four A registers
// holding (code - 8) as packed halves:
//   r0 = (w[4t],    w[4t+2])     r1 = (w[4t+16], w[4t+18])
//   r2 = (w[4t+1],  w[4t+3])     r3 = (w[4t+17], w[4t+19])
// fp16: 0x6400 | n is 1024 + n; 0x6400 | (n << 4) is 1024 + 16n.  Placing
// a 4-bit code in the mantissa of 1024.0 and subtracting the bias is the
// integer-to-fp16 conversion published by Kim et al., "Who Says Elephants
// Can't Run: Bringing Large Scale MoE Models into Cloud Scale Production"
// (arXiv:2211.10017).
__device__ __forceinline__ void decode_f16(uint32_t q, uint32_t r[4]) {
  const uint32_t q8 = __umulhi(q, 0x01000000u);  // q >> 8, on the FMA pipe
  uint32_t t0 = lop3_and_or(q, 0x000F000Fu, 0x64006400u);
  uint32_t t1 = lop3_and_or(q, 0x00F000F0u, 0x64006400u);
  uint32_t t2 = lop3_and_or(q8, 0x000F000Fu, 0x64006400u);
  uint32_t t3 = lop3_and_or(q8, 0x00F000F0u, 0x64006400u);
  const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  const __half2 k16th = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
  const __half2 km72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
  __half2 h0 = __hsub2(*reinterpret_cast<__half2*>(&t0), k1032);
  __half2 h1 = __hfma2(*reinterpret_cast<__half2*>(&t1), k16th, km72);
  __half2 h2 = __hsub2(*reinterpret_cast<__half2*>(&t2), k1032);
  __half2 h3 = __hfma2(*reinterpret_cast<__half2*>(&t3), k16th, km72);
  r[0] = *reinterpret_cast<uint32_t*>(&h0);
  r[1] = *reinterpret_cast<uint32_t*>(&h1);
  r[2] = *reinterpret_cast<uint32_t*>(&h2);
  r[3] = *reinterpret_cast<uint32_t*>(&h3);
}

// bf16: 0x4300 | n is 128 + n (7 mantissa bits, so nibbles are shifted down).
__device__ __forceinline__ void decode_bf16(uint32_t q, uint32_t r[4]) {
  const __nv_bfloat162 k136 =
      __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
  uint32_t t[4];
  t[0] = lop3_and_or(q, 0x000F000Fu, 0x43004300u);
  t[1] = lop3_and_or(q >> 4, 0x000F000Fu, 0x43004300u);
  t[2] = lop3_and_or(q >> 8, 0x000F000Fu, 0x43004300u);
  t[3] = lop3_and_or(q >> 12, 0x000F000Fu, 0x43004300u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&t[i]), k136);
    r[i] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// The dynamic shared-memory array of every kernel in this file.  Loads below
// index it by 32-bit byte offsets, so they are plain shared-memory loads with
// immediate offsets, ordered after the stage's mbarrier wait.
extern __shared__ __align__(128) uint8_t smem[];

__device__ __forceinline__ uint32_t ld32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}
__device__ __forceinline__ uint32_t ld16(uint32_t off) {
  return *reinterpret_cast<const uint16_t*>(smem + off);
}
__device__ __forceinline__ uint4 ld128(uint32_t off) {
  return *reinterpret_cast<const uint4*>(smem + off);
}
// four bytes at an offset that is 2 mod 4 (MIS == 2) or 0 mod 4 (MIS == 0)
template <int MIS>
__device__ __forceinline__ uint32_t ld32_at(uint32_t off) {
  if constexpr (MIS == 0) {
    return ld32(off);
  } else {
    return __byte_perm(ld32(off - 2), ld32(off + 2), 0x5432u);
  }
}
// four bytes at an even offset whose alignment is known only at run time
__device__ __forceinline__ uint32_t ld32_even(uint32_t off) {
  const uint32_t b = off & ~3u;
  return __byte_perm(ld32(b), ld32(b + 4), (off & 2u) ? 0x5432u : 0x3210u);
}

// The activation fragment of one block.  With one activation vector only B
// columns 0 and 2 carry it (lane groups 0 and 2 load, every other lane holds
// zeros): the shared-memory load then touches 2 of the warp's 8 lane
// quarters, and columns 0 and 2 of the result put row r in lane t = 0 and
// row r+8 in lane t = 1.
template <int NT>
__device__ __forceinline__ uint4 x_frag(uint32_t xp) {
  if constexpr (NT == 0) {
    const int lane = threadIdx.x & 31;
    return (lane & 0x14) == 0 ? ld128(xp) : make_uint4(0u, 0u, 0u, 0u);
  } else {
    return ld128(xp);
  }
}

// One 32-weight block for rows r (codes qa) and r+8 (codes qb): both k16
// MMAs over every activation term and every n8 tile, into a fresh fragment c
// (tile n in c[4n..4n+3]).  The codes are decoded once for all tiles; tile 1
// reads the batch row xt1 bytes past tile 0's.
template <int XT, int NT>
__device__ __forceinline__ void block_mma(float* c, uint32_t qa, uint32_t qb, uint32_t xp,
                                          uint32_t term_stride, uint32_t xt1) {
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  constexpr int kTiles = NT > 1 ? NT : 1;
  uint32_t ra[4], rb[4];
  if constexpr (XT == XT_F16) {
    decode_f16(qa, ra);
    decode_f16(qb, rb);
#pragma unroll
    for (int n = 0; n < kTiles; ++n) {
      const uint4 xv = x_frag<NT>(xp + n * xt1);
      mma_f16_z(c + 4 * n, ra[0], rb[0], ra[2], rb[2], xv.x, xv.y);
      mma_f16(c + 4 * n, ra[1], rb[1], ra[3], rb[3], xv.z, xv.w);
    }
  } else {
    decode_bf16(qa, ra);
    decode_bf16(qb, rb);
#pragma unroll
    for (int n = 0; n < kTiles; ++n) {
#pragma unroll
      for (int tm = 0; tm < kTerms; ++tm) {
        const uint4 xv = x_frag<NT>(xp + n * xt1 + tm * term_stride);
        if (tm == 0)
          mma_bf16_z(c + 4 * n, ra[0], rb[0], ra[2], rb[2], xv.x, xv.y);
        else
          mma_bf16(c + 4 * n, ra[0], rb[0], ra[2], rb[2], xv.x, xv.y);
        mma_bf16(c + 4 * n, ra[1], rb[1], ra[3], rb[3], xv.z, xv.w);
      }
    }
  }
}

// Scale a block's fragment and accumulate: acc[i] += d(row) * c[i].  With one
// activation vector (x_frag) lane t = 0 keeps row r (c[0], column 0) and
// lane t = 1 row r+8 (c[2], column 2), each in acc[0] with its own row's
// scale d0; lanes t = 2, 3 accumulate zeros.
template <int NT>
__device__ __forceinline__ void scale_acc(float* acc, const float* c, float d0, float d1) {
  if constexpr (NT == 0) {
    const int t = threadIdx.x & 3;
    acc[0] = fmaf(d0, (t & 1) ? c[2] : c[0], acc[0]);
  } else {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      acc[4 * n + 0] = fmaf(d0, c[4 * n + 0], acc[4 * n + 0]);
      acc[4 * n + 2] = fmaf(d1, c[4 * n + 2], acc[4 * n + 2]);
      acc[4 * n + 1] = fmaf(d0, c[4 * n + 1], acc[4 * n + 1]);
      acc[4 * n + 3] = fmaf(d1, c[4 * n + 3], acc[4 * n + 3]);
    }
  }
}

// ---------------------------------------------------------------- Q4_0 body
// Block j of a stage: its two rows' code words and scales (with one
// activation vector only the scale of this lane's output row, at rowd).
template <bool ALIGNED, int J, int NT>
__device__ __forceinline__ void q40_load(uint32_t row0, uint32_t row1, uint32_t rowd, int t,
                                         int jb, uint32_t& qa, uint32_t& qb, float& da,
                                         float& db) {
  const uint32_t a = row0 + jb * 18;
  const uint32_t b = row1 + jb * 18;
  if constexpr (ALIGNED) {
    // rows start on 16-byte boundaries and jb has the parity of J: the codes
    // of an even block start 2 mod 4, of an odd block 0 mod 4
    qa = ld32_at<(J & 1) ? 0 : 2>(a + 2 + 4 * t);
    qb = ld32_at<(J & 1) ? 0 : 2>(b + 2 + 4 * t);
  } else {
    qa = ld32_even(a + 2 + 4 * t);
    qb = ld32_even(b + 2 + 4 * t);
  }
  if constexpr (NT == 0) {
    da = half_bits_to_float(ld16(rowd + jb * 18));
    db = da;
  } else {
    da = half_bits_to_float(ld16(a));
    db = half_bits_to_float(ld16(b));
  }
}

// A consumer warp's blocks w*kSubPerWarp .. +kSubPerWarp-1 of one stage.  A
// full share is unrolled without branches -- every load is issued before the
// first decode -- so the warp keeps many loads and MMAs in flight.
template <int XT, int NT, bool ALIGNED>
__device__ __forceinline__ void q40_chunk(float* acc, uint32_t row0, uint32_t row1, uint32_t xw,
                                          uint32_t term_stride, uint32_t xt1, int w, int t,
                                          int nvalid) {
  const int jw = w * kSubPerWarp;  // even
  const uint32_t rowd = (t & 1) ? row1 : row0;
  if (nvalid >= kSubPerWarp) {
    uint32_t qa[kSubPerWarp], qb[kSubPerWarp];
    float da[kSubPerWarp], db[kSubPerWarp];
#pragma unroll
    for (int j = 0; j < kSubPerWarp; j += 2) {
      q40_load<ALIGNED, 0, NT>(row0, row1, rowd, t, jw + j, qa[j], qb[j], da[j], db[j]);
      q40_load<ALIGNED, 1, NT>(row0, row1, rowd, t, jw + j + 1, qa[j + 1], qb[j + 1], da[j + 1],
                               db[j + 1]);
    }
#pragma unroll
    for (int j = 0; j < kSubPerWarp; ++j) {
      float c[acc_len(NT)];
      block_mma<XT, NT>(c, qa[j], qb[j], xw + (jw + j) * kXBlk, term_stride, xt1);
      scale_acc<NT>(acc, c, da[j], db[j]);
    }
  } else {
    // ragged last chunk of a row
    for (int j = 0; j < nvalid; ++j) {
      uint32_t qa, qb;
      float da, db;
      q40_load<false, 0, NT>(row0, row1, rowd, t, jw + j, qa, qb, da, db);
      float c[acc_len(NT)];
      block_mma<XT, NT>(c, qa, qb, xw + (jw + j) * kXBlk, term_stride, xt1);
      scale_acc<NT>(acc, c, da, db);
    }
  }
}

// ----------------------------------------------------------------- ksb body
// A consumer warp's kSubPerWarp sub-blocks of one super-block of the stage.
// s~_j = S * q_j is applied as q_j per sub-block and S once at the end.  All
// loads are issued before the first decode.
// MIS: offset mod 4 of the super-block's code and sub-scale words when rows
// are 16-byte aligned (then fixed per warp: 138-byte super-blocks alternate
// between 0 and 2 mod 4 and chunks start on multiples of 8 bytes); -1 when
// it is known only at run time.
template <int MIS>
__device__ __forceinline__ uint32_t ld32_w(uint32_t off) {
  if constexpr (MIS < 0) {
    return ld32_even(off);
  } else {
    return ld32_at<MIS>(off);
  }
}

template <int XT, int NT, int MIS>
__device__ __forceinline__ void ksb_chunk(float* acc, uint32_t row0, uint32_t row1, uint32_t xw,
                                          uint32_t term_stride, uint32_t xt1, int w, int t) {
  constexpr bool kOne = (NT == 0);
  const int sb = (w * kSubPerWarp) >> 3, j0 = (w * kSubPerWarp) & 7;
  const uint32_t a = row0 + sb * 138;
  const uint32_t b = row1 + sb * 138;
  // scales of rows r and r+8; with one activation vector only this lane's
  // output row (scale_acc), read into both
  const uint32_t sa = kOne ? ((t & 1) ? b : a) : a;
  const float Sa = half_bits_to_float(ld16(sa));
  const float Sb = kOne ? Sa : half_bits_to_float(ld16(b));
  uint32_t qja[2], qjb[2];
  qja[0] = ld32_w<MIS>(sa + 2 + j0);
  qjb[0] = kOne ? qja[0] : ld32_w<MIS>(b + 2 + j0);
  if constexpr (kSubPerWarp > 4) {
    qja[1] = ld32_w<MIS>(sa + 6 + j0);
    qjb[1] = kOne ? qja[1] : ld32_w<MIS>(b + 6 + j0);
  }
  float sacc[acc_len(NT)];
#pragma unroll
  for (int i = 0; i < acc_len(NT); ++i) sacc[i] = 0.f;
  constexpr int kBatch = kSubPerWarp < 4 ? kSubPerWarp : 4;
#pragma unroll
  for (int h = 0; h < kSubPerWarp; h += kBatch) {  // batches of up to four sub-blocks
    uint32_t na[kBatch], nb[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      na[j] = ld32_w<MIS>(a + 10 + 16 * (j0 + h + j) + 4 * t);
      nb[j] = ld32_w<MIS>(b + 10 + 16 * (j0 + h + j) + 4 * t);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      float c[acc_len(NT)];
      block_mma<XT, NT>(c, na[j], nb[j], xw + (8 * sb + j0 + h + j) * kXBlk, term_stride, xt1);
      const int q = h + j;  // sub-block index within this warp's share
      const float fa = static_cast<float>(static_cast<int8_t>((qja[q >> 2] >> (8 * (q & 3))) & 0xFFu));
      const float fb = static_cast<float>(static_cast<int8_t>((qjb[q >> 2] >> (8 * (q & 3))) & 0xFFu));
      scale_acc<NT>(sacc, c, fa, fb);
    }
  }
  if constexpr (kOne) {
    acc[0] = fmaf(Sa, sacc[0], acc[0]);
  } else {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      acc[4 * n + 0] = fmaf(Sa, sacc[4 * n + 0], acc[4 * n + 0]);
      acc[4 * n + 1] = fmaf(Sa, sacc[4 * n + 1], acc[4 * n + 1]);
      acc[4 * n + 2] = fmaf(Sb, sacc[4 * n + 2], acc[4 * n + 2]);
      acc[4 * n + 3] = fmaf(Sb, sacc[4 * n + 3], acc[4 * n + 3]);
    }
  }
}

// ---------------------------------------------------- activation windows
// Load activations [k_begin, k_end) of all batch rows into shared memory in
// B-fragment order: for each 32 weights and lane-group t (0..3), 16 bytes
//   x[4t], x[4t+2], x[4t+1], x[4t+3], x[4t+16], x[4t+18], x[4t+17], x[4t+19]
// Each thread moves 8 consecutive values as two 8-byte stores per term.
template <int XT>
__device__ __forceinline__ void store_x8(uint8_t* xs, const void* xsrc, int B, int b, int k8,
                                         uint32_t term_stride, const uint4* raw) {
  static_assert((kChunkW & (kChunkW - 1)) == 0, "chunk is a power of two");
  const int cw = k8 / kChunkW, blk = (k8 & (kChunkW - 1)) >> 5, p = k8 & 31;
  const int hi = p >> 4, t0 = (p & 15) >> 2;
  // lane-group t0 gets (v0 v2 v1 v3) at slot 4*hi, lane-group t0+1 the next four
  uint8_t* dst = xs + (cw * B + b) * kXStride + blk * kXBlk + t0 * 16 + hi * 8;
  if constexpr (XT == XT_F32) {
    const float v[8] = {__uint_as_float(raw[0].x), __uint_as_float(raw[0].y),
                        __uint_as_float(raw[0].z), __uint_as_float(raw[0].w),
                        __uint_as_float(raw[1].x), __uint_as_float(raw[1].y),
                        __uint_as_float(raw[1].z), __uint_as_float(raw[1].w)};
    uint32_t term[3][4];  // per term: bf16 pairs (v0,v1)(v2,v3)(v4,v5)(v6,v7)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t parts[3][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // exact split v = b1 + b2 + b3 into bfloat16 terms
        const float vv = v[2 * i + h];
        const __nv_bfloat16 b1 = __float2bfloat16_rn(vv);
        const float r1 = __fsub_rn(vv, __bfloat162float(b1));
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(b2));
        const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
        parts[0][h] = __bfloat16_as_ushort(b1);
        parts[1][h] = __bfloat16_as_ushort(b2);
        parts[2][h] = __bfloat16_as_ushort(b3);
      }
#pragma unroll
      for (int tm = 0; tm < 3; ++tm) term[tm][i] = parts[tm][0] | (parts[tm][1] << 16);
    }
#pragma unroll
    for (int tm = 0; tm < 3; ++tm) {
      uint8_t* d = dst + tm * term_stride;
      *reinterpret_cast<uint2*>(d) = make_uint2(__byte_perm(term[tm][0], term[tm][1], 0x5410),
                                                __byte_perm(term[tm][0], term[tm][1], 0x7632));
      *reinterpret_cast<uint2*>(d + 16) = make_uint2(__byte_perm(term[tm][2], term[tm][3], 0x5410),
                                                     __byte_perm(term[tm][2], term[tm][3], 0x7632));
    }
  } else {
    const uint4 u = raw[0];
    *reinterpret_cast<uint2*>(dst) = make_uint2(__byte_perm(u.x, u.y, 0x5410), __byte_perm(u.x, u.y, 0x7632));
    *reinterpret_cast<uint2*>(dst + 16) = make_uint2(__byte_perm(u.z, u.w, 0x5410), __byte_perm(u.z, u.w, 0x7632));
  }
}

// Load activations [k_begin, k_end) of all batch rows into shared memory in
// B-fragment order: for each 32 weights and lane-group t (0..3), 16 bytes
//   x[4t], x[4t+2], x[4t+1], x[4t+3], x[4t+16], x[4t+18], x[4t+17], x[4t+19]
// Each thread moves groups of 8 consecutive values; the global loads of eight
// groups (four for fp32) are issued together before any of them is stored.
template <int XT>
__device__ void load_x_window(uint8_t* xs, const void* x, int64_t K, int B, int c0, int nwin,
                              uint32_t term_stride, int tid) {
  constexpr int kVec = (XT == XT_F32) ? 2 : 1;  // uint4 per 8 values
  constexpr int kBatch = 4;
  constexpr int kStride = 32 * kConsumers;
  const int64_t k_begin = static_cast<int64_t>(c0) * kChunkW;
  const int per_row = static_cast<int>((i64min(K, k_begin + static_cast<int64_t>(nwin) * kChunkW) - k_begin) / 8);
  for (int b = 0; b < B; ++b) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) +
                                                      (b * K + k_begin) * (XT == XT_F32 ? 4 : 2));
    for (int base = tid; base < per_row; base += kBatch * kStride) {
      uint4 raw[kBatch][kVec];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int g8 = base + i * kStride;
        if (g8 < per_row) {
#pragma unroll
          for (int v = 0; v < kVec; ++v) raw[i][v] = src[g8 * kVec + v];
        }
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int g8 = base + i * kStride;
        if (g8 < per_row) store_x8<XT>(xs, x, B, b, g8 * 8, term_stride, raw[i]);
      }
    }
  }
}

template <int FMT, int XT, int NT, bool ALIGNED, class Tbl>
__global__ void __launch_bounds__(kThreads, GQ_GEMV_MINB)
    gemv_kernel(const GemvArgs a, const __grid_constant__ Tbl tbl) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW, kBlkB = Fmt<FMT>::kBlkB;
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  constexpr int kBlkPerChunk = kChunkW / kBlkW;
  constexpr int kChunkBytes = kBlkPerChunk * kBlkB;

  uint8_t* stages = smem;
  uint8_t* xs = smem + kStages * kStageBytes;
  const uint32_t term_stride = static_cast<uint32_t>(a.win * a.B * kXStride);
  // [2][kConsumers][32][acc_len(NT)]
  float* red = reinterpret_cast<float*>(xs + kTerms * term_stride);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kConsumers * 32 * acc_len(NT));
  uint64_t* empty = full + kStages;
  uint64_t* cbar = empty + kStages;  // consumer-group barrier (bounded waits)
  int* abort_flag = reinterpret_cast<int*>(cbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk_row = static_cast<int>(a.K / kBlkW);
  const int nfull = nblk_row / kBlkPerChunk;  // chunks with every block present

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    mbar_init(cbar, kConsumers);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = policy_evict_first();
    int issued = 0;      // stage uses issued so far (all groups)
    int s = 0;           // stage of the next use
    uint32_t ph = 0;     // its phase parity
    bool ok = true;
    const uint32_t tail_bytes = static_cast<uint32_t>((nblk_row - nfull * kBlkPerChunk) * kBlkB);
    int pmi = 0;  // matrix cursor
    for (int g = blockIdx.x; g < a.ngroups && ok; g += gridDim.x) {
      const Unit un = unit_of(a, tbl, g, pmi);
      const int64_t m0 = un.m0;
      const bool row_ok = lane < kRows && m0 + lane < un.M;
      uintptr_t src = reinterpret_cast<uintptr_t>(un.W) +
                      static_cast<uintptr_t>((m0 + (row_ok ? lane : 0)) * a.rowbytes);
      for (int c = 0; c < a.nchunks; ++c, ++issued, src += kChunkBytes) {
        if (!mbar_wait(&empty[s], ph ^ 1u, a.budget) ||
            *reinterpret_cast<volatile int*>(abort_flag)) {
          ok = false;
          break;
        }
        if (a.skip_first && issued == 0) {  // self-test: this stage never fills
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
          continue;
        }
        const uint32_t nbytes = (c < nfull) ? static_cast<uint32_t>(kChunkBytes) : tail_bytes;
        uint32_t len = 0;
        uintptr_t lo = 0;
        if (row_ok) {
          lo = src & ~static_cast<uintptr_t>(15);
          len = static_cast<uint32_t>(((src + nbytes + 15) & ~static_cast<uintptr_t>(15)) - lo);
        }
        uint32_t total = len;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xFFFFFFFFu, total, o);
        if (lane == 0) mbar_arrive_expect_tx(&full[s], total);
        __syncwarp();
        if (len)
          bulk_g2s(stages + s * kStageBytes + lane * kPitch, reinterpret_cast<const void*>(lo), len,
                   &full[s], pol);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      report(a.dev_status, GQ_DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
    }
    // Drain: every issued copy must land before this CTA's shared memory is
    // released, whatever the consumers did.
    if (lane == 0) {
      for (int u = max(0, issued - kStages); u < issued; ++u) {
        if (a.skip_first && u == 0) continue;  // never issued
        if (!mbar_wait(&full[u % kStages], static_cast<uint32_t>(u / kStages) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;                // consumer index, also its share of a chunk
  const int ctid = threadIdx.x - 32;      // 0 .. 32 * kConsumers - 1
  const int r = lane >> 2, t = lane & 3;  // fragment row group / thread in group
  const int bsel = min(r, a.B - 1);       // batch column this lane's B fragment reads
  bool ok = true;
  uint32_t cphase = 0;
  // All consumer warps pass the same sequence of group barriers; a barrier is
  // an mbarrier phase (one arrival per warp) so that waiting on it is bounded.
  auto group_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    const bool done = mbar_wait(cbar, cphase & 1u, a.budget);
    ++cphase;
    return done;
  };

  // this warp's share of a ragged last chunk
  int tail_valid;
  if constexpr (FMT == GQ_FMT_Q4_0)
    tail_valid = min(max(nblk_row - nfull * kBlkPerChunk - kSubPerWarp * cw, 0), kSubPerWarp);
  else
    tail_valid = ((cw * kSubPerWarp) >> 3) < nblk_row - nfull * kBlkPerChunk;

  pdl_wait();  // the preceding grid has finished: x is ready, y may be written

  const bool x_resident = (a.win >= a.nchunks);
  if (x_resident) {
    load_x_window<XT>(xs, a.x, a.K, a.B, 0, a.win, term_stride, ctid);
    ok = group_sync();
  }
  const uint32_t x_chunk = static_cast<uint32_t>(a.B * kXStride);
  const uint32_t x_lane = static_cast<uint32_t>(xs - smem) + bsel * kXStride + t * 16;
  // n8 tile 1 holds batch rows 8..15: this lane's row there, relative to tile 0
  const uint32_t xt1 = static_cast<uint32_t>((min(8 + r, a.B - 1) - bsel) * kXStride);

  int s = 0;        // stage of the next use
  uint32_t ph = 0;  // its phase parity
  int gi = 0;       // groups done by this CTA
  int cmi = 0;  // matrix cursor
  for (int g = blockIdx.x; g < a.ngroups && ok; g += gridDim.x, ++gi) {
    const Unit un = unit_of(a, tbl, g, cmi);
    const int64_t m0 = un.m0;
    float acc[acc_len(NT)];
#pragma unroll
    for (int q = 0; q < acc_len(NT); ++q) acc[q] = 0.f;
    // offset of row r's (and r+8's) first byte inside its 16-byte granule
    uint32_t off0 = static_cast<uint32_t>(
        (reinterpret_cast<uintptr_t>(un.W) + static_cast<uintptr_t>((m0 + r) * a.rowbytes)) & 15u);
    uint32_t off1 = static_cast<uint32_t>(
        (reinterpret_cast<uintptr_t>(un.W) + static_cast<uintptr_t>((m0 + r + 8) * a.rowbytes)) &
        15u);
    uint32_t xw = x_lane;
    int cw_in_win = 0;
    for (int c = 0; c < a.nchunks; ++c) {
      if (!x_resident && cw_in_win == 0) {
        if (!group_sync()) { ok = false; break; }
        load_x_window<XT>(xs, a.x, a.K, a.B, c, a.win, term_stride, ctid);
        if (!group_sync()) { ok = false; break; }
        xw = x_lane;
      }
      if (!mbar_wait(&full[s], ph, a.budget) || *reinterpret_cast<volatile int*>(abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t stg = static_cast<uint32_t>(s * kStageBytes);  // stages start at offset 0
      const bool whole = c < nfull;
      if constexpr (FMT == GQ_FMT_Q4_0) {
        const int nvalid = whole ? kSubPerWarp : tail_valid;
        if constexpr (ALIGNED) {
          q40_chunk<XT, NT, true>(acc, stg + r * kPitch, stg + (r + 8) * kPitch, xw,
                                  term_stride, xt1, cw, t, nvalid);
        } else {
          q40_chunk<XT, NT, false>(acc, stg + r * kPitch + off0, stg + (r + 8) * kPitch + off1,
                                   xw, term_stride, xt1, cw, t, nvalid);
        }
      } else {
        if (whole || tail_valid) {
          const uint32_t p0 = stg + r * kPitch + off0, p1 = stg + (r + 8) * kPitch + off1;
          if constexpr (ALIGNED) {
            // this warp's super-block: even ones put their words at 2 mod 4
            if (((cw * kSubPerWarp) >> 3) & 1)
              ksb_chunk<XT, NT, 0>(acc, p0, p1, xw, term_stride, xt1, cw, t);
            else
              ksb_chunk<XT, NT, 2>(acc, p0, p1, xw, term_stride, xt1, cw, t);
          } else {
            ksb_chunk<XT, NT, -1>(acc, p0, p1, xw, term_stride, xt1, cw, t);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == kStages) {
        s = 0;
        ph ^= 1u;
      }
      off0 = (off0 + kChunkBytes) & 15u;
      off1 = (off1 + kChunkBytes) & 15u;
      xw += x_chunk;
      if (++cw_in_win == a.win) cw_in_win = 0;
    }
    if (!ok) break;

    // reduce the consumer warps' partial sums (double-buffered by group
    // parity, so one barrier per group suffices), then store
    constexpr int kTiles = NT > 1 ? NT : 1;
    float4* rb = reinterpret_cast<float4*>(red) + (gi & 1) * kConsumers * 32 * kTiles;
#pragma unroll
    for (int n = 0; n < kTiles; ++n)
      rb[(cw * 32 + lane) * kTiles + n] =
          make_float4(acc[4 * n], acc[4 * n + 1], acc[4 * n + 2], acc[4 * n + 3]);
    if (!group_sync()) { ok = false; break; }
    if (cw == 0) {
      float s4[acc_len(NT)];
#pragma unroll
      for (int q = 0; q < acc_len(NT); ++q) s4[q] = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
#pragma unroll
        for (int n = 0; n < kTiles; ++n) {
          const float4 v = rb[(w * 32 + lane) * kTiles + n];
          s4[4 * n + 0] += v.x;
          s4[4 * n + 1] += v.y;
          s4[4 * n + 2] += v.z;
          s4[4 * n + 3] += v.w;
        }
      }
      const int64_t ra = m0 + r, rbw = m0 + r + 8;
      if constexpr (NT == 0) {
        // lane t = 0 holds row r, lane t = 1 row r + 8 (scale_acc)
        const int64_t row = (t == 0) ? ra : rbw;
        if (t < 2 && row < un.M) store_elem(un.y, row, s4[0], a.ytype);
      } else {
#pragma unroll
        for (int n = 0; n < kTiles; ++n) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int col = 8 * n + 2 * t + i;
            if (col < a.B) {
              if (ra < un.M) store_elem(un.y, col * un.M + ra, s4[4 * n + i], a.ytype);
              if (rbw < un.M) store_elem(un.y, col * un.M + rbw, s4[4 * n + 2 + i], a.ytype);
            }
          }
        }
      }
    }
  }

  if (!ok && lane == 0) {
    report(a.dev_status, GQ_DEV_TIMEOUT);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
  }
}

// One matrix with K split over a thread-block cluster.  The CTAs of a
// cluster share each of the cluster's row groups g = clusterid,
// clusterid + nclusters, ...: rank q takes chunks [q * split_cps,
// (q + 1) * split_cps) of every row, with its slice of x resident (the host
// sizes the slice to fit).  At the end of a group every rank leaves its fp32
// sums in slot gi % kSplitSlots of its own shared memory; rank 0 adds them
// up one group later, in rank order, reading the other ranks' slots through
// distributed shared memory, and stores y.  A slice of x fills more than half
// of the shared memory, so these CTAs run one per SM.  Apart from the chunk
// range, the group sequence and the exchange, each step is gemv_kernel's.
template <int FMT, int XT, int NT, bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) gemv_split_kernel(const GemvArgs a) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW, kBlkB = Fmt<FMT>::kBlkB;
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  constexpr int kBlkPerChunk = kChunkW / kBlkW;
  constexpr int kChunkBytes = kBlkPerChunk * kBlkB;
  constexpr int kTiles = NT > 1 ? NT : 1;

  uint8_t* stages = smem;
  uint8_t* xs = smem + kStages * kStageBytes;
  const uint32_t term_stride = static_cast<uint32_t>(a.win * a.B * kXStride);
  // [2][kConsumers][32][acc_len(NT)]
  float* red = reinterpret_cast<float*>(xs + kTerms * term_stride);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kConsumers * 32 * acc_len(NT));
  uint64_t* empty = full + kStages;
  uint64_t* cbar = empty + kStages;  // consumer-group barrier (bounded waits)
  int* abort_flag = reinterpret_cast<int*>(cbar + 1);
  // the exchange: part_full[p] (used in rank 0) completes when every lane of
  // every other rank has left its sums of a group in its slot p; part_free[p]
  // (other ranks) when rank 0's lanes have read them
  uint64_t* part_full = reinterpret_cast<uint64_t*>(smem + a.split_off);
  uint64_t* part_free = part_full + kSplitSlots;
  float* xred = reinterpret_cast<float*>(part_free + kSplitSlots);  // [slots][32][acc_len(NT)]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk_row = static_cast<int>(a.K / kBlkW);
  const int nfull = nblk_row / kBlkPerChunk;  // chunks with every block present
  const uint32_t rank = cluster_ctarank(), nrank = cluster_nctarank();
  const int c_begin = static_cast<int>(rank) * a.split_cps;
  const int c_end = min(a.nchunks, c_begin + a.split_cps);
  const int g_first = static_cast<int>(cluster_id_x());
  const int g_step = static_cast<int>(cluster_count_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    mbar_init(cbar, kConsumers);
    for (int p = 0; p < kSplitSlots; ++p) {
      mbar_init(&part_full[p], 32 * (nrank - 1));
      mbar_init(&part_free[p], 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // every CTA's barriers exist before any other CTA of the cluster arrives on them
  cluster_sync_all();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = policy_evict_first();
    int issued = 0;      // stage uses issued so far (all groups)
    int s = 0;           // stage of the next use
    uint32_t ph = 0;     // its phase parity
    bool ok = true;
    const uint32_t tail_bytes = static_cast<uint32_t>((nblk_row - nfull * kBlkPerChunk) * kBlkB);
    for (int g = g_first; g < a.ngroups && ok; g += g_step) {
      const int64_t m0 = static_cast<int64_t>(g) * kRows;
      const bool row_ok = lane < kRows && m0 + lane < a.M;
      uintptr_t src = reinterpret_cast<uintptr_t>(a.W) +
                      static_cast<uintptr_t>((m0 + (row_ok ? lane : 0)) * a.rowbytes +
                                             static_cast<int64_t>(c_begin) * kChunkBytes);
      for (int c = c_begin; c < c_end; ++c, ++issued, src += kChunkBytes) {
        if (!mbar_wait(&empty[s], ph ^ 1u, a.budget) ||
            *reinterpret_cast<volatile int*>(abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t nbytes = (c < nfull) ? static_cast<uint32_t>(kChunkBytes) : tail_bytes;
        uint32_t len = 0;
        uintptr_t lo = 0;
        if (row_ok) {
          lo = src & ~static_cast<uintptr_t>(15);
          len = static_cast<uint32_t>(((src + nbytes + 15) & ~static_cast<uintptr_t>(15)) - lo);
        }
        uint32_t total = len;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xFFFFFFFFu, total, o);
        if (lane == 0) mbar_arrive_expect_tx(&full[s], total);
        __syncwarp();
        if (len)
          bulk_g2s(stages + s * kStageBytes + lane * kPitch, reinterpret_cast<const void*>(lo), len,
                   &full[s], pol);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      report(a.dev_status, GQ_DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
    }
    // Drain: every issued copy must land before this CTA's shared memory is
    // released, whatever the consumers did.
    if (lane == 0) {
      for (int u = max(0, issued - kStages); u < issued; ++u) {
        if (!mbar_wait(&full[u % kStages], static_cast<uint32_t>(u / kStages) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
      }
    }
    // no CTA of the cluster leaves while another may still read its memory
    cluster_sync_all();
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;                // consumer index, also its share of a chunk
  const int ctid = threadIdx.x - 32;      // 0 .. 32 * kConsumers - 1
  const int r = lane >> 2, t = lane & 3;  // fragment row group / thread in group
  const int bsel = min(r, a.B - 1);       // batch column this lane's B fragment reads
  bool ok = true;
  uint32_t cphase = 0;
  auto group_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    const bool done = mbar_wait(cbar, cphase & 1u, a.budget);
    ++cphase;
    return done;
  };

  // this warp's share of a ragged last chunk
  int tail_valid;
  if constexpr (FMT == GQ_FMT_Q4_0)
    tail_valid = min(max(nblk_row - nfull * kBlkPerChunk - kSubPerWarp * cw, 0), kSubPerWarp);
  else
    tail_valid = ((cw * kSubPerWarp) >> 3) < nblk_row - nfull * kBlkPerChunk;

  pdl_wait();  // the preceding grid has finished: x is ready, y may be written

  // this rank's slice of x, resident for the whole kernel
  load_x_window<XT>(xs, a.x, a.K, a.B, c_begin, a.win, term_stride, ctid);
  ok = group_sync();
  const uint32_t x_chunk = static_cast<uint32_t>(a.B * kXStride);
  const uint32_t x_lane = static_cast<uint32_t>(xs - smem) + bsel * kXStride + t * 16;
  // n8 tile 1 holds batch rows 8..15: this lane's row there, relative to tile 0
  const uint32_t xt1 = static_cast<uint32_t>((min(8 + r, a.B - 1) - bsel) * kXStride);

  // rank 0, warp 0: add up group gj (row group gg) from every rank's slot,
  // in rank order, and store it; each lane reads and releases only its own
  // entries
  auto finish = [&](int gj, int gg) -> bool {
    const int p = gj % kSplitSlots;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&part_full[p],
                                                   static_cast<uint32_t>(gj / kSplitSlots) & 1u,
                                                   a.budget)))
      return false;
    const float4* slot = reinterpret_cast<const float4*>(xred) + (p * 32 + lane) * kTiles;
    float v[acc_len(NT)];
#pragma unroll
    for (int n = 0; n < kTiles; ++n) {
      const float4 o = slot[n];
      v[4 * n + 0] = o.x;
      v[4 * n + 1] = o.y;
      v[4 * n + 2] = o.z;
      v[4 * n + 3] = o.w;
    }
    const uint32_t sa = smem_addr(slot);
    for (uint32_t q = 1; q < nrank; ++q) {
#pragma unroll
      for (int n = 0; n < kTiles; ++n) {
        const float4 w = ld_cluster_f4(sa + 16u * n, q);
        v[4 * n + 0] += w.x;
        v[4 * n + 1] += w.y;
        v[4 * n + 2] += w.z;
        v[4 * n + 3] += w.w;
      }
    }
    for (uint32_t q = 1; q < nrank; ++q) mbar_arrive_remote(&part_free[p], q);
    const int64_t ra = static_cast<int64_t>(gg) * kRows + r, rbw = ra + 8;
#pragma unroll
    for (int n = 0; n < kTiles; ++n) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int col = 8 * n + 2 * t + i;
        if (col < a.B) {
          if (ra < a.M) store_elem(a.y, col * a.M + ra, v[4 * n + i], a.ytype);
          if (rbw < a.M) store_elem(a.y, col * a.M + rbw, v[4 * n + 2 + i], a.ytype);
        }
      }
    }
    return true;
  };

  int s = 0;        // stage of the next use
  uint32_t ph = 0;  // its phase parity
  int gi = 0;       // groups done by this CTA
  for (int g = g_first; g < a.ngroups && ok; g += g_step, ++gi) {
    const int64_t m0 = static_cast<int64_t>(g) * kRows;
    float acc[acc_len(NT)];
#pragma unroll
    for (int q = 0; q < acc_len(NT); ++q) acc[q] = 0.f;
    // offset of row r's (and r+8's) first byte of chunk c_begin inside its
    // 16-byte granule
    const int64_t cb_off = static_cast<int64_t>(c_begin) * kChunkBytes;
    uint32_t off0 = static_cast<uint32_t>(
        (reinterpret_cast<uintptr_t>(a.W) + static_cast<uintptr_t>((m0 + r) * a.rowbytes + cb_off)) &
        15u);
    uint32_t off1 = static_cast<uint32_t>(
        (reinterpret_cast<uintptr_t>(a.W) +
         static_cast<uintptr_t>((m0 + r + 8) * a.rowbytes + cb_off)) &
        15u);
    uint32_t xw = x_lane;
    for (int c = c_begin; c < c_end; ++c) {
      if (!mbar_wait(&full[s], ph, a.budget) || *reinterpret_cast<volatile int*>(abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t stg = static_cast<uint32_t>(s * kStageBytes);  // stages start at offset 0
      const bool whole = c < nfull;
      if constexpr (FMT == GQ_FMT_Q4_0) {
        const int nvalid = whole ? kSubPerWarp : tail_valid;
        if constexpr (ALIGNED) {
          q40_chunk<XT, NT, true>(acc, stg + r * kPitch, stg + (r + 8) * kPitch, xw,
                                  term_stride, xt1, cw, t, nvalid);
        } else {
          q40_chunk<XT, NT, false>(acc, stg + r * kPitch + off0, stg + (r + 8) * kPitch + off1,
                                   xw, term_stride, xt1, cw, t, nvalid);
        }
      } else {
        if (whole || tail_valid) {
          const uint32_t p0 = stg + r * kPitch + off0, p1 = stg + (r + 8) * kPitch + off1;
          if constexpr (ALIGNED) {
            if (((cw * kSubPerWarp) >> 3) & 1)
              ksb_chunk<XT, NT, 0>(acc, p0, p1, xw, term_stride, xt1, cw, t);
            else
              ksb_chunk<XT, NT, 2>(acc, p0, p1, xw, term_stride, xt1, cw, t);
          } else {
            ksb_chunk<XT, NT, -1>(acc, p0, p1, xw, term_stride, xt1, cw, t);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == kStages) {
        s = 0;
        ph ^= 1u;
      }
      off0 = (off0 + kChunkBytes) & 15u;
      off1 = (off1 + kChunkBytes) & 15u;
      xw += x_chunk;
    }
    if (!ok) break;

    // the consumer warps' sums meet in the reduction buffer (double-buffered
    // by group parity), then warp 0 hands this CTA's part to the exchange
    float4* rb = reinterpret_cast<float4*>(red) + (gi & 1) * kConsumers * 32 * kTiles;
#pragma unroll
    for (int n = 0; n < kTiles; ++n)
      rb[(cw * 32 + lane) * kTiles + n] =
          make_float4(acc[4 * n], acc[4 * n + 1], acc[4 * n + 2], acc[4 * n + 3]);
    if (!group_sync()) { ok = false; break; }
    if (cw == 0) {
      float s4[acc_len(NT)];
#pragma unroll
      for (int q = 0; q < acc_len(NT); ++q) s4[q] = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
#pragma unroll
        for (int n = 0; n < kTiles; ++n) {
          const float4 v = rb[(w * 32 + lane) * kTiles + n];
          s4[4 * n + 0] += v.x;
          s4[4 * n + 1] += v.y;
          s4[4 * n + 2] += v.z;
          s4[4 * n + 3] += v.w;
        }
      }
      const int p = gi % kSplitSlots;
      float4* slot = reinterpret_cast<float4*>(xred) + (p * 32 + lane) * kTiles;
      // rank 0 has read what this slot held kSplitSlots groups ago (its own
      // slot it read itself, one group after writing it)
      if (rank != 0 && gi >= kSplitSlots &&
          !__all_sync(0xFFFFFFFFu,
                      mbar_wait_cluster(&part_free[p],
                                        static_cast<uint32_t>(gi / kSplitSlots - 1) & 1u,
                                        a.budget))) {
        ok = false;
      } else {
#pragma unroll
        for (int n = 0; n < kTiles; ++n)
          slot[n] = make_float4(s4[4 * n], s4[4 * n + 1], s4[4 * n + 2], s4[4 * n + 3]);
        if (rank != 0) mbar_arrive_remote(&part_full[p], 0);
        // the previous group's parts are in, or about to be
        if (rank == 0 && gi >= 1 && !finish(gi - 1, g - g_step)) ok = false;
      }
    }
  }
  // rank 0 adds up its last group
  if (ok && cw == 0 && rank == 0 && gi >= 1 && !finish(gi - 1, g_first + (gi - 1) * g_step))
    ok = false;

  if (!ok && lane == 0) {
    report(a.dev_status, GQ_DEV_TIMEOUT);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
  }
  // no CTA of the cluster leaves while another may still read its memory
  cluster_sync_all();
}

size_t gemv_smem_bytes(int B, int terms, int win) {
  const int nt = B == 1 ? 0 : (B <= 8 ? 1 : 2);
  return static_cast<size_t>(kStages) * kStageBytes +
         static_cast<size_t>(terms) * win * B * kXStride + red_bytes(nt) +
         (2 * kStages + 1) * sizeof(uint64_t) + 16;
}

template <int FMT, int XT, int NT, bool ALIGNED, class Tbl>
gq_status launch_gemv(const GemvArgs& a, const Tbl& tbl, cudaStream_t stream, bool pdl) {
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  auto kern = gemv_kernel<FMT, XT, NT, ALIGNED, Tbl>;
  const size_t smem = gemv_smem_bytes(a.B, kTerms, a.win);
  // per host thread, so that concurrent callers (possibly on other devices)
  // never see each other's half-updated state
  thread_local unsigned long long configured_ctx = 0;
  thread_local size_t configured_smem = 0;
  thread_local size_t occ_smem = 0;
  thread_local int occupancy = 1;
  const unsigned long long ctx = context_id();
  if (ctx == 0 || ctx != configured_ctx || smem > configured_smem) {
    // at least the common sizes, and always this launch's own requirement
    const size_t want = smem > gemv_smem_bytes(1, kTerms, 0) + kXSmemMax
                            ? smem
                            : gemv_smem_bytes(1, kTerms, 0) + kXSmemMax;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(want)) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_ctx = ctx;
    configured_smem = want;
    occ_smem = 0;
  }
  if (occ_smem != smem) {
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    occupancy = per_sm;
    occ_smem = smem;
  }
  const int64_t slots = static_cast<int64_t>(sm_count()) * occupancy;
  const int grid = static_cast<int>(a.ngroups < slots ? a.ngroups : slots);
  return launch(kern, dim3(grid), dim3(kThreads), smem, stream, pdl, a, tbl);
}

// Bytes of the K-split exchange area: kSplitSlots barriers each way, then
// the partial sums [kSplitSlots][32][acc_len(nt)].
constexpr size_t split_extra(int nt) {
  return 16 * kSplitSlots + static_cast<size_t>(kSplitSlots) * 32 * acc_len(nt) * 4;
}

// One matrix with K split over clusters of `cluster` CTAs (a.split_cps chunks
// each, a.win == a.split_cps).  Sets `launched` when it launched (or failed
// to); leaves it false when no cluster of that size fits on the device.
template <int FMT, int XT, int NT, bool ALIGNED>
gq_status launch_gemv_split(GemvArgs a, int cluster, cudaStream_t stream, bool pdl,
                            bool& launched) {
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  auto kern = gemv_split_kernel<FMT, XT, NT, ALIGNED>;
  const size_t base = (gemv_smem_bytes(a.B, kTerms, a.win) + 15) & ~static_cast<size_t>(15);
  a.split_off = static_cast<uint32_t>(base);
  const size_t smem = base + split_extra(NT);
  // per host thread, as launch_gemv
  thread_local unsigned long long configured_ctx = 0;
  thread_local size_t configured_smem = 0;
  thread_local size_t occ_smem = 0;
  thread_local int occ_cluster = 0;
  thread_local int max_clusters = 0;
  const unsigned long long ctx = context_id();
  launched = true;
  if (ctx == 0 || ctx != configured_ctx || smem > configured_smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_ctx = ctx;
    configured_smem = smem;
    occ_smem = 0;
  }
  if (occ_smem != smem || occ_cluster != cluster) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster * sm_count()));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    max_clusters = n;
    occ_smem = smem;
    occ_cluster = cluster;
  }
  if (max_clusters < 1) {
    launched = false;
    return GQ_OK;
  }
  const int nclusters = a.ngroups < max_clusters ? a.ngroups : max_clusters;
  return launch_cluster(kern, dim3(static_cast<unsigned>(nclusters * cluster)), dim3(kThreads),
                        smem, stream, pdl, static_cast<unsigned>(cluster), a);
}

template <int FMT, int XT>
gq_status dispatch_split(const GemvArgs& a, int cluster, bool w_aligned, cudaStream_t s, bool pdl,
                         bool& launched) {
  const bool aligned = (a.rowbytes % 16 == 0) && w_aligned;
  if (a.B <= 8)
    return aligned ? launch_gemv_split<FMT, XT, 1, true>(a, cluster, s, pdl, launched)
                   : launch_gemv_split<FMT, XT, 1, false>(a, cluster, s, pdl, launched);
  return aligned ? launch_gemv_split<FMT, XT, 2, true>(a, cluster, s, pdl, launched)
                 : launch_gemv_split<FMT, XT, 2, false>(a, cluster, s, pdl, launched);
}

// w_aligned: every matrix of the launch starts on a 16-byte boundary.
template <int FMT, int XT, class Tbl>
gq_status dispatch_gemv(const GemvArgs& a, const Tbl& tbl, bool w_aligned, cudaStream_t s,
                        bool pdl) {
  // Q4_0 rows of whole granules keep every chunk on a 16-byte boundary; ksb
  // rows of whole granules fix each warp's word alignment (ksb_chunk)
  const bool aligned = (a.rowbytes % 16 == 0) && w_aligned;
  if (a.B == 1) {
    return aligned ? launch_gemv<FMT, XT, 0, true>(a, tbl, s, pdl)
                   : launch_gemv<FMT, XT, 0, false>(a, tbl, s, pdl);
  }
  if (a.B <= 8) {
    return aligned ? launch_gemv<FMT, XT, 1, true>(a, tbl, s, pdl)
                   : launch_gemv<FMT, XT, 1, false>(a, tbl, s, pdl);
  }
  return aligned ? launch_gemv<FMT, XT, 2, true>(a, tbl, s, pdl)
                 : launch_gemv<FMT, XT, 2, false>(a, tbl, s, pdl);
}

template <int FMT, class Tbl>
gq_status dispatch_xt(const GemvArgs& a, const Tbl& tbl, int xt, bool w_aligned, cudaStream_t s,
                      bool pdl) {
  switch (xt) {
    case GQ_F16: return dispatch_gemv<FMT, XT_F16>(a, tbl, w_aligned, s, pdl);
    case GQ_BF16: return dispatch_gemv<FMT, XT_BF16>(a, tbl, w_aligned, s, pdl);
    default: return dispatch_gemv<FMT, XT_F32>(a, tbl, w_aligned, s, pdl);
  }
}

// The fields of GemvArgs that depend only on K, B and the dtypes.
template <int FMT>
void fill_common(GemvArgs& a, int64_t K, const void* x, int xt, int64_t B, int yt,
                 int* dev_status, long long budget) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW, kBlkB = Fmt<FMT>::kBlkB;
  a.K = K;
  a.rowbytes = K / kBlkW * kBlkB;
  a.x = x;
  a.dev_status = dev_status;
  a.budget = budget;
  a.B = static_cast<int>(B);
  a.ytype = yt;
  a.nchunks = static_cast<int>((K + kChunkW - 1) / kChunkW);
  a.skip_first = 0;
  a.split_cps = 0;
  a.split_off = 0;
  const int terms = (xt == GQ_F32) ? 3 : 1;
  const int64_t per_chunk = static_cast<int64_t>(terms) * a.B * kXStride;
  int win = static_cast<int>(kXSmemMax / per_chunk);
  // batches keep all of x resident when it fits beside the ring at one CTA
  // per SM, rather than reloading windows for every row group: a CTA whose
  // x needs more than the window budget runs one per SM either way
  if (a.B >= kResidentMinB && per_chunk * a.nchunks <= kXSmemFree) win = a.nchunks;
  if (win < 1) win = 1;
  if (win > a.nchunks) win = a.nchunks;
  a.win = win;
}

template <int FMT>
gq_status gemv_entry(const void* W, int64_t M, int64_t K, const void* x, int xt, int64_t B,
                     void* y, int yt, void* workspace, size_t ws_bytes, unsigned flags,
                     int* dev_status, void* stream, long long budget = kWaitBudget,
                     int skip_first = 0, int64_t max_b = 8) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW;
  if (M < 0 || K < 0 || B < 0) return GQ_ERR_INVALID_ARG;
  if (!valid_act_dtype(xt) || !valid_act_dtype(yt)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (K % kBlkW) return GQ_ERR_SHAPE;
  if (B > max_b || M > 0x7FFFFFFFLL || K > (1LL << 24)) return GQ_ERR_SHAPE;
  if (M == 0 || B == 0) return GQ_OK;
  if (!y) return GQ_ERR_INVALID_ARG;
  if (misaligned16(y)) return GQ_ERR_ALIGNMENT;
  if (K == 0) {
    return cudaMemsetAsync(y, 0, static_cast<size_t>(B * M * dtype_size(yt)), as_stream(stream)) ==
                   cudaSuccess
               ? GQ_OK
               : GQ_ERR_CUDA;
  }
  if (!W || !x) return GQ_ERR_INVALID_ARG;
  if (misaligned16(W) || misaligned16(x)) return GQ_ERR_ALIGNMENT;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return GQ_ERR_ALIGNMENT;

  GemvArgs a;
  fill_common<FMT>(a, K, x, xt, B, yt, dev_status, budget);
  a.W = static_cast<const uint8_t*>(W);
  a.M = M;
  a.y = y;
  a.ngroups = static_cast<int>((M + kRows - 1) / kRows);
  a.skip_first = skip_first;

  const bool pdl = (flags & GQ_GEMV_PDL) != 0;
  cudaStream_t s = as_stream(stream);
  if (workspace && ws_bytes && !skip_first && i8_eligible(FMT, M, K, B, xt, W))
    return i8_gemv(W, M, K, x, y, yt, workspace, ws_bytes, pdl, dev_status, s);
  if (B > 1 && !skip_first && a.win < a.nchunks) {
    // x does not fit beside the ring: split K over a cluster of up to 8 CTAs
    // whose slices of x do, rather than reload windows for every row group
    const int terms = (xt == GQ_F32) ? 3 : 1;
    const int64_t per_chunk = static_cast<int64_t>(terms) * B * kXStride;
    const int64_t room = kXSmemFree - 16 - static_cast<int64_t>(split_extra(B <= 8 ? 1 : 2));
    const int cps_max = static_cast<int>(room / per_chunk);
    const int cluster = cps_max >= 1 ? (a.nchunks + cps_max - 1) / cps_max : 0;
    if (cluster >= 2 && cluster <= 8) {
      GemvArgs sa = a;
      sa.split_cps = (a.nchunks + cluster - 1) / cluster;  // every rank gets a chunk
      sa.win = sa.split_cps;
      bool launched = false;
      gq_status st = GQ_OK;
      switch (xt) {
        case GQ_F16: st = dispatch_split<FMT, XT_F16>(sa, cluster, !misaligned16(W), s, pdl, launched); break;
        case GQ_BF16: st = dispatch_split<FMT, XT_BF16>(sa, cluster, !misaligned16(W), s, pdl, launched); break;
        default: st = dispatch_split<FMT, XT_F32>(sa, cluster, !misaligned16(W), s, pdl, launched); break;
      }
      if (launched) return st;
    }
  }
  return dispatch_xt<FMT>(a, NoTable{0}, xt, !misaligned16(W), s, pdl);
}

// Several matrices that share K and the activations x: y_i = W_i x for each
// descriptor, in launches of up to kMaxMats matrices whose CTAs stream the
// groups of all their matrices back to back.
template <int FMT>
gq_status gemv_grouped_entry(const gq_gemv_desc* mats, int count, int64_t K, const void* x,
                             int xt, int64_t B, int yt, unsigned flags, int* dev_status,
                             void* stream) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW;
  if (count < 0 || K < 0 || B < 0) return GQ_ERR_INVALID_ARG;
  if (count > 0 && !mats) return GQ_ERR_INVALID_ARG;
  if (!valid_act_dtype(xt) || !valid_act_dtype(yt)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (K % kBlkW) return GQ_ERR_SHAPE;
  if (B > 8 || K > (1LL << 24)) return GQ_ERR_SHAPE;
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
  if (B == 0 || groups == 0) return GQ_OK;
  cudaStream_t s = as_stream(stream);
  if (K == 0) {
    for (int i = 0; i < count; ++i)
      if (mats[i].M > 0 && cudaMemsetAsync(mats[i].y, 0,
                                           static_cast<size_t>(B * mats[i].M * dtype_size(yt)),
                                           s) != cudaSuccess)
        return GQ_ERR_CUDA;
    return GQ_OK;
  }
  if (!x) return GQ_ERR_INVALID_ARG;
  if (misaligned16(x)) return GQ_ERR_ALIGNMENT;

  GemvArgs a;
  fill_common<FMT>(a, K, x, xt, B, yt, dev_status, kWaitBudget);
  a.W = nullptr;
  a.M = 0;
  a.y = nullptr;
  const bool pdl = (flags & GQ_GEMV_PDL) != 0;
  GemvTable tbl{};  // one launch's table, passed to the kernel by value
  int i = 0;
  while (i < count) {
    int n = 0, g = 0;
    for (; i < count && n < kMaxMats; ++i) {
      const gq_gemv_desc& d = mats[i];
      if (d.M == 0) continue;
      g += static_cast<int>((d.M + kRows - 1) / kRows);
      tbl.m[n] = GemvMat{static_cast<const uint8_t*>(d.W), d.y, d.M, g, 0};
      ++n;
    }
    if (n == 0) break;
    a.ngroups = g;
    const gq_status st = dispatch_xt<FMT>(a, tbl, xt, true, s, pdl);
    if (st != GQ_OK) return st;
  }
  return GQ_OK;
}

}  // namespace

#if GQ_GEMV_MANY_TU
// The large-table grouped product, compiled in its own translation unit with
// the pipeline constants set there (gq_gemv_grouped.cu).
gq_status gemv_grouped_many(int fmt, const gq_gemv_desc* mats, int count, int64_t K,
                            const void* x, int xt, int64_t B, int yt, unsigned flags,
                            int* dev_status, cudaStream_t stream) {
  if (fmt == GQ_FMT_Q4_0)
    return gemv_grouped_entry<GQ_FMT_Q4_0>(mats, count, K, x, xt, B, yt, flags, dev_status,
                                           stream);
  return gemv_grouped_entry<GQ_FMT_KSB>(mats, count, K, x, xt, B, yt, flags, dev_status, stream);
}

}  // namespace gq
#else
gq_status gemv_batched(int fmt, const void* W, int64_t M, int64_t K, const void* x, int xt,
                       int64_t B, void* y, int yt, int* dev_status, cudaStream_t stream) {
  if (fmt == GQ_FMT_Q4_0)
    return gemv_entry<GQ_FMT_Q4_0>(W, M, K, x, xt, B, y, yt, nullptr, 0, 0u, dev_status, stream,
                                   kWaitBudget, 0, kWarpMmaMaxB);
  return gemv_entry<GQ_FMT_KSB>(W, M, K, x, xt, B, y, yt, nullptr, 0, 0u, dev_status, stream,
                                kWaitBudget, 0, kWarpMmaMaxB);
}

// Row groups of a grouped call's valid descriptors (validation happens in
// the entry point that is then chosen).
int64_t grouped_groups(const gq_gemv_desc* mats, int count) {
  int64_t g = 0;
  for (int i = 0; mats && i < count; ++i)
    if (mats[i].M > 0) g += (mats[i].M + kRows - 1) / kRows;
  return g;
}

// Grouped calls with at least this many row groups per SM stream on the
// large-table configuration (four small CTAs per SM, gq_gemv_grouped.cu):
// with that much work per SM, more independent pipelines per SM beat fewer
// wide ones, while a single matrix or a short table keeps this file's
// configuration (wide CTAs whose early exit lets the next launch start).
constexpr int64_t kManyGroupsPerSm = 8;

}  // namespace gq

extern "C" {

GQ_API size_t gq_gemv_workspace_bytes(int fmt, int64_t M, int64_t K, int64_t B, int x_dtype) {
  if (M <= 0 || K <= 0) return 0;
  // eligibility apart from the pointer: a 16-byte-aligned stand-in
  if (!gq::i8_eligible(fmt, M, K, B, x_dtype, reinterpret_cast<const void*>(uintptr_t{16})))
    return 0;
  return gq::i8_workspace_bytes(M, K);
}

GQ_API gq_status gq_gemv_q4_0(const void* W, int64_t M, int64_t K, const void* x, int x_dtype,
                              int64_t B, void* y, int y_dtype, void* workspace, size_t ws_bytes,
                              unsigned flags, int* dev_status, void* stream) {
  return gq::gemv_entry<GQ_FMT_Q4_0>(W, M, K, x, x_dtype, B, y, y_dtype, workspace, ws_bytes,
                                     flags, dev_status, stream);
}

GQ_API gq_status gq_gemv_ksb(const void* W, int64_t M, int64_t K, const void* x, int x_dtype,
                             int64_t B, void* y, int y_dtype, void* workspace, size_t ws_bytes,
                             unsigned flags, int* dev_status, void* stream) {
  return gq::gemv_entry<GQ_FMT_KSB>(W, M, K, x, x_dtype, B, y, y_dtype, workspace, ws_bytes,
                                    flags, dev_status, stream);
}

GQ_API gq_status gq_gemv_q4_0_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                      const void* x, int x_dtype, int64_t B, int y_dtype,
                                      unsigned flags, int* dev_status, void* stream) {
  if (count > 0 && gq::grouped_groups(mats, count) >= gq::kManyGroupsPerSm * gq::sm_count())
    return gq::gemv_grouped_many(GQ_FMT_Q4_0, mats, count, K, x, x_dtype, B, y_dtype, flags,
                                 dev_status, gq::as_stream(stream));
  return gq::gemv_grouped_entry<GQ_FMT_Q4_0>(mats, count, K, x, x_dtype, B, y_dtype, flags,
                                             dev_status, stream);
}

GQ_API gq_status gq_gemv_ksb_grouped(const gq_gemv_desc* mats, int count, int64_t K,
                                     const void* x, int x_dtype, int64_t B, int y_dtype,
                                     unsigned flags, int* dev_status, void* stream) {
  if (count > 0 && gq::grouped_groups(mats, count) >= gq::kManyGroupsPerSm * gq::sm_count())
    return gq::gemv_grouped_many(GQ_FMT_KSB, mats, count, K, x, x_dtype, B, y_dtype, flags,
                                 dev_status, gq::as_stream(stream));
  return gq::gemv_grouped_entry<GQ_FMT_KSB>(mats, count, K, x, x_dtype, B, y_dtype, flags,
                                            dev_status, stream);
}

// Allocation-free batch-1 Q4_0 GEMV: the integer tensor-core path of
// gq_gemv_q4_0 with its scratch in a static device array, for callers that
// cannot hand the library device memory -- a runtime that allocates nothing
// after start-up, or a C caller with no device allocator of its own.
GQ_API gq_status gq_gemv_q4_0_noalloc(const void* W, int64_t M, int64_t K, const void* x,
                                      void* y, int y_dtype, unsigned flags, int* dev_status,
                                      void* stream) {
  if (M < 0 || K < 0) return GQ_ERR_INVALID_ARG;
  if (!gq::valid_act_dtype(y_dtype)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (M == 0) return GQ_OK;
  if (!W || !x || !y) return GQ_ERR_INVALID_ARG;
  if (gq::misaligned16(W) || gq::misaligned16(x) || gq::misaligned16(y)) return GQ_ERR_ALIGNMENT;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return GQ_ERR_ALIGNMENT;
  if (!gq::i8_shape_ok(GQ_FMT_Q4_0, M, K, 1, GQ_F16, W)) return GQ_ERR_SHAPE;
  return gq::i8_gemv_noalloc(W, M, K, x, y, y_dtype, (flags & GQ_GEMV_PDL) != 0, dev_status,
                             gq::as_stream(stream));
}

// Bounded-wait self-test: a Q4_0 GEMV (fp16 x and y, batch 1) whose producer
// never fills its first stage; with a ~1 ms budget the consumers' wait runs
// out, the kernel ORs GQ_DEV_TIMEOUT into *dev_status, lets every copy it did
// issue land, and exits.  Nothing faults, traps or hangs.
GQ_API gq_status gq_selftest_gemv_timeout(const void* W, int64_t M, int64_t K, const void* x,
                                          void* y, int* dev_status, void* stream) {
  if (!dev_status) return GQ_ERR_INVALID_ARG;
  return gq::gemv_entry<GQ_FMT_Q4_0>(W, M, K, x, GQ_F16, 1, y, GQ_F16, nullptr, 0, 0u,
                                     dev_status, stream, 2000000LL, 1);
}

}  // extern "C"
#endif  // GQ_GEMV_MANY_TU
