// gq_gemv.cu -- dequantize-fused matrix-vector product for decode,
// y[b][m] = sum_k W_hat[m][k] * x[b][k], for 1..8 activation vectors.
//
// Operation: the matrix multiply that consumes decoded blocks ("GGUF 量化内幕
// 第4章" 4.3: w = d * (code - 8); "GGUF K-quants" 套娃: s~_j = S * q_j), in the
// memory-bound decode setting (TurboQuant W4A8 post, section 2.3).
//
// Design (sm_100a):
//  * One CTA owns 16 consecutive rows (one m16 MMA tile) over all of K.  Its
//    rows are contiguous in HBM, so the CTA reads one contiguous byte range.
//  * Warp 0 is the producer: for each K chunk of 1024 weights it issues one
//    1-D bulk async copy (cp.async.bulk, no multicast) per row into a 4-stage
//    shared-memory ring, completion tracked by mbarrier transaction counts.
//    Row pieces need not be 16-byte aligned (18-byte / 138-byte blocks): the
//    copy covers the enclosing 16-byte granules and consumers index from the
//    piece's offset inside its first granule.
//  * Warps 1..4 consume: each takes a quarter of the chunk, decodes 4-bit
//    codes straight into MMA A fragments (code - 8 exactly, by exponent-bias
//    tricks on packed halves), and runs warp MMA m16n8k16 with fp32
//    accumulation.  The batch columns are the MMA's N dimension (N = 8 covers
//    B <= 8; B = 1 replicates one column).  Because every block has its own
//    scale, the two MMAs of a 32-weight block accumulate into a fresh
//    fragment that is then scaled and added in fp32 -- products are exact
//    (4-bit integer x fp16/bf16), so no weight is ever rounded.
//  * fp32 activations are split exactly into three bfloat16 terms (three
//    MMAs per k-step); fp16 and bf16 activations use one.
//  * The activations live in shared memory in the fragment order of the MMA
//    B operand; a warp reads its B fragments with one 16-byte load per block.
//  * Programmatic dependent launch: the producer streams W immediately;
//    consumers wait for the preceding grid before reading x or writing y.
//  * Every mbarrier wait is bounded; on expiry the kernel sets
//    GQ_DEV_TIMEOUT, drains its own in-flight copies (bounded) and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_host.h"

namespace gq {
namespace {

constexpr int kRows = 16;                           // rows per CTA
constexpr int kConsumers = 4;                       // consumer warps
constexpr int kThreads = 32 * (1 + kConsumers);
constexpr int kChunkW = 1024;                       // weights per row per stage
constexpr int kPitch = 592;                         // bytes per row slot (>= 590)
constexpr int kStageBytes = kRows * kPitch + 16;    // +16: window-read slack
constexpr int kStages = 4;
constexpr int kXBlk = 64;                           // B-fragment bytes per 32 weights
constexpr int kXStride = (kChunkW / 32) * kXBlk + 64;  // per (chunk, batch row), padded
constexpr int kXSmemMax = 96 * 1024;                // activation window budget

enum { XT_F16 = 0, XT_BF16 = 1, XT_F32 = 2 };

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
  int B, ytype, nchunks, win;  // win: chunks per activation window
};

// ---- decode 8 codes (one 32-bit word = qs[4t..4t+3]) into four A registers
// holding (code - 8) as packed halves:
//   r0 = (w[4t],    w[4t+2])     r1 = (w[4t+16], w[4t+18])
//   r2 = (w[4t+1],  w[4t+3])     r3 = (w[4t+17], w[4t+19])
// fp16: 0x6400 | n is 1024 + n; 0x6400 | (n << 4) is 1024 + 16n.
__device__ __forceinline__ void decode_f16(uint32_t q, uint32_t r[4]) {
  const uint32_t q8 = q >> 8;
  __half2 h0, h1, h2, h3;
  uint32_t t0 = lop3_and_or(q, 0x000F000Fu, 0x64006400u);
  uint32_t t1 = lop3_and_or(q, 0x00F000F0u, 0x64006400u);
  uint32_t t2 = lop3_and_or(q8, 0x000F000Fu, 0x64006400u);
  uint32_t t3 = lop3_and_or(q8, 0x00F000F0u, 0x64006400u);
  const __half2 k1032 = __float2half2_rn(1032.0f);
  const __half2 k16th = __float2half2_rn(0.0625f);
  const __half2 km72 = __float2half2_rn(-72.0f);
  h0 = __hsub2(*reinterpret_cast<__half2*>(&t0), k1032);
  h1 = __hfma2(*reinterpret_cast<__half2*>(&t1), k16th, km72);
  h2 = __hsub2(*reinterpret_cast<__half2*>(&t2), k1032);
  h3 = __hfma2(*reinterpret_cast<__half2*>(&t3), k16th, km72);
  r[0] = *reinterpret_cast<uint32_t*>(&h0);
  r[1] = *reinterpret_cast<uint32_t*>(&h1);
  r[2] = *reinterpret_cast<uint32_t*>(&h2);
  r[3] = *reinterpret_cast<uint32_t*>(&h3);
}

// bf16: 0x4300 | n is 128 + n (7 mantissa bits, so nibbles are shifted down).
__device__ __forceinline__ void decode_bf16(uint32_t q, uint32_t r[4]) {
  const __nv_bfloat162 k136 = __float2bfloat162_rn(136.0f);
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

template <int XT>
__device__ __forceinline__ void decode(uint32_t q, uint32_t r[4]) {
  if constexpr (XT == XT_F16)
    decode_f16(q, r);
  else
    decode_bf16(q, r);
}

template <int XT>
__device__ __forceinline__ void mma(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                    uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (XT == XT_F16)
    mma_f16(c, a0, a1, a2, a3, b0, b1);
  else
    mma_bf16(c, a0, a1, a2, a3, b0, b1);
}

// One 32-weight block for rows r (codes qa) and r+8 (codes qb): the two k16
// MMAs of the block, over all activation terms, into c (zeroed by caller).
template <int XT>
__device__ __forceinline__ void block_mma(float c[4], uint32_t qa, uint32_t qb, uint32_t xaddr,
                                          uint32_t term_stride) {
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  uint32_t ra[4], rb[4];
  decode<XT>(qa, ra);
  decode<XT>(qb, rb);
#pragma unroll
  for (int tm = 0; tm < kTerms; ++tm) {
    const uint4 xv = lds128(xaddr + tm * term_stride);
    // A regs: (row r, k lo) (row r+8, k lo) (row r, k hi) (row r+8, k hi)
    mma<XT>(c, ra[0], rb[0], ra[2], rb[2], xv.x, xv.y);
    mma<XT>(c, ra[1], rb[1], ra[3], rb[3], xv.z, xv.w);
  }
}

// Load one window of activations into shared memory in B-fragment order.
// For 32 weights of batch row b, lane-group t (0..3) reads 16 bytes:
//   x[4t], x[4t+2], x[4t+1], x[4t+3], x[4t+16], x[4t+18], x[4t+17], x[4t+19]
template <int XT>
__device__ void load_x_window(uint8_t* xs, const void* x, int64_t K, int B, int c0, int nwin,
                              uint32_t term_stride, int tid) {
  const int64_t k_begin = static_cast<int64_t>(c0) * kChunkW;
  const int64_t k_end = i64min(K, k_begin + static_cast<int64_t>(nwin) * kChunkW);
  const int per_row = static_cast<int>((k_end - k_begin) / 8);
  for (int idx = tid; idx < B * per_row; idx += 32 * kConsumers) {
    const int b = idx / per_row;
    const int k8 = (idx - b * per_row) * 8;  // relative to the window
    const int64_t gk = k_begin + k8;
    float v[8];
    uint16_t bits[8];
    if constexpr (XT == XT_F32) {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + b * K + gk);
      const float4 u0 = p[0], u1 = p[1];
      v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
      v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
    } else {
      const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + b * K + gk);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        bits[2 * i] = static_cast<uint16_t>(w[i] & 0xFFFFu);
        bits[2 * i + 1] = static_cast<uint16_t>(w[i] >> 16);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int kk = k8 + i;
      const int cw = kk / kChunkW, blk = (kk % kChunkW) / 32, p = kk % 32;
      const int hi = p >> 4, pp = p & 15, t = pp >> 2, ii = pp & 3;
      const int slot = hi * 4 + ((ii & 1) << 1) + (ii >> 1);
      uint8_t* dst = xs + (cw * B + b) * kXStride + blk * kXBlk + t * 16 + slot * 2;
      if constexpr (XT == XT_F32) {
        // exact split v = b1 + b2 + b3 into bfloat16 terms
        const __nv_bfloat16 b1 = __float2bfloat16_rn(v[i]);
        const float r1 = __fsub_rn(v[i], __bfloat162float(b1));
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(b2));
        const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
        *reinterpret_cast<__nv_bfloat16*>(dst) = b1;
        *reinterpret_cast<__nv_bfloat16*>(dst + term_stride) = b2;
        *reinterpret_cast<__nv_bfloat16*>(dst + 2 * term_stride) = b3;
      } else {
        *reinterpret_cast<uint16_t*>(dst) = bits[i];
      }
    }
  }
}

template <int FMT, int XT>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kBlkW = Fmt<FMT>::kBlkW, kBlkB = Fmt<FMT>::kBlkB;
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;

  uint8_t* stages = smem;
  uint8_t* xs = smem + kStages * kStageBytes;
  const uint32_t term_stride = static_cast<uint32_t>(a.win * a.B * kXStride);
  float* red = reinterpret_cast<float*>(xs + kTerms * term_stride);  // [kConsumers][32][4]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kConsumers * 32 * 4);
  uint64_t* empty = full + kStages;
  uint64_t* cbar = empty + kStages;  // consumer-group barrier (bounded waits)
  int* abort_flag = reinterpret_cast<int*>(cbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kRows;
  const int64_t nblk_row = a.K / kBlkW;
  constexpr int kBlkPerChunk = kChunkW / kBlkW;

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
    int issued = 0;
    bool ok = true;
    for (int c = 0; c < a.nchunks && ok; ++c) {
      const int s = c % kStages;
      const uint32_t ph = static_cast<uint32_t>(c / kStages) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u, a.budget)) {
        ok = false;
        break;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) {
        ok = false;
        break;
      }
      const int64_t b0 = static_cast<int64_t>(c) * kBlkPerChunk;
      const int64_t nb = i64min(kBlkPerChunk, nblk_row - b0);
      uint32_t len = 0;
      const uint8_t* src_al = nullptr;
      if (lane < kRows && m0 + lane < a.M) {
        const uintptr_t src = reinterpret_cast<uintptr_t>(a.W) +
                              static_cast<uintptr_t>((m0 + lane) * a.rowbytes + b0 * kBlkB);
        const uintptr_t lo = src & ~static_cast<uintptr_t>(15);
        const uintptr_t hi = (src + static_cast<uintptr_t>(nb * kBlkB) + 15) & ~static_cast<uintptr_t>(15);
        src_al = reinterpret_cast<const uint8_t*>(lo);
        len = static_cast<uint32_t>(hi - lo);
      }
      uint32_t total = len;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xFFFFFFFFu, total, o);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], total);
      __syncwarp();
      if (len) bulk_g2s(stages + s * kStageBytes + lane * kPitch, src_al, len, &full[s], pol);
      issued = c + 1;
    }
    if (!ok) {
      if (lane == 0) {
        report(a.dev_status, GQ_DEV_TIMEOUT);
        *reinterpret_cast<volatile int*>(abort_flag) = 1;
      }
    }
    // Drain: every issued copy must land before this CTA's shared memory is
    // released, whatever the consumers did.
    if (lane == 0) {
      for (int c = max(0, issued - kStages); c < issued; ++c) {
        const int s = c % kStages;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(c / kStages) & 1u, a.budget)) {
          report(a.dev_status, GQ_DEV_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;                // consumer index 0..3
  const int ctid = threadIdx.x - 32;      // 0..127
  const int r = lane >> 2, t = lane & 3;  // fragment row group / thread in group
  const int bsel = min(r, a.B - 1);       // batch column this lane's B fragment reads
  const uint32_t stages_addr = smem_addr(stages);
  const uint32_t xs_addr = smem_addr(xs);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
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

  pdl_wait();  // the preceding grid has finished: x is ready, y may be written

  for (int c = 0; c < a.nchunks; ++c) {
    if (c % a.win == 0) {
      if (!group_sync()) {
        ok = false;
        break;
      }
      load_x_window<XT>(xs, a.x, a.K, a.B, c, a.win, term_stride, ctid);
      if (!group_sync()) {
        ok = false;
        break;
      }
    }
    const int s = c % kStages;
    if (!mbar_wait(&full[s], static_cast<uint32_t>(c / kStages) & 1u, a.budget) ||
        *reinterpret_cast<volatile int*>(abort_flag)) {
      ok = false;
      break;
    }
    const int64_t b0 = static_cast<int64_t>(c) * kBlkPerChunk;
    // byte offset of each row piece inside its first 16-byte granule
    const uintptr_t base0 = reinterpret_cast<uintptr_t>(a.W) +
                            static_cast<uintptr_t>((m0 + r) * a.rowbytes + b0 * kBlkB);
    const uintptr_t base1 = base0 + static_cast<uintptr_t>(8 * a.rowbytes);
    const uint32_t row0 = stages_addr + s * kStageBytes + r * kPitch + (base0 & 15u);
    const uint32_t row1 = stages_addr + s * kStageBytes + (r + 8) * kPitch + (base1 & 15u);
    const uint32_t xw = xs_addr + ((c % a.win) * a.B + bsel) * kXStride + t * 16;

    if constexpr (FMT == GQ_FMT_Q4_0) {
      // this warp's 8 blocks of the chunk
      const int jb0 = cw * 8;
      const int nvalid = static_cast<int>(i64min(8, nblk_row - b0 - jb0));
#pragma unroll 4
      for (int j = 0; j < 8; ++j) {
        if (j < nvalid) {
          const uint32_t off = (jb0 + j) * kBlkB;
          const float d0 = half_bits_to_float(lds16(row0 + off));
          const float d1 = half_bits_to_float(lds16(row1 + off));
          const uint32_t qa = lds32_even(row0 + off + 2 + 4 * t);
          const uint32_t qb = lds32_even(row1 + off + 2 + 4 * t);
          float cf[4] = {0.f, 0.f, 0.f, 0.f};
          block_mma<XT>(cf, qa, qb, xw + (jb0 + j) * kXBlk, term_stride);
          acc[0] = fmaf(d0, cf[0], acc[0]);
          acc[1] = fmaf(d0, cf[1], acc[1]);
          acc[2] = fmaf(d1, cf[2], acc[2]);
          acc[3] = fmaf(d1, cf[3], acc[3]);
        }
      }
    } else {
      // this warp's super-block of the chunk
      if (b0 + cw < nblk_row) {
        const uint32_t off = cw * kBlkB;
        const float S0 = half_bits_to_float(lds16(row0 + off));
        const float S1 = half_bits_to_float(lds16(row1 + off));
        const uint32_t qs0a = lds32_even(row0 + off + 2), qs0b = lds32_even(row0 + off + 6);
        const uint32_t qs1a = lds32_even(row1 + off + 2), qs1b = lds32_even(row1 + off + 6);
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t qa = lds32_even(row0 + off + 10 + 16 * j + 4 * t);
          const uint32_t qb = lds32_even(row1 + off + 10 + 16 * j + 4 * t);
          float cf[4] = {0.f, 0.f, 0.f, 0.f};
          block_mma<XT>(cf, qa, qb, xw + (cw * 8 + j) * kXBlk, term_stride);
          const uint32_t w0 = (j < 4) ? qs0a : qs0b, w1 = (j < 4) ? qs1a : qs1b;
          const float qj0 = static_cast<float>(static_cast<int8_t>((w0 >> (8 * (j & 3))) & 0xFFu));
          const float qj1 = static_cast<float>(static_cast<int8_t>((w1 >> (8 * (j & 3))) & 0xFFu));
          sacc[0] = fmaf(qj0, cf[0], sacc[0]);
          sacc[1] = fmaf(qj0, cf[1], sacc[1]);
          sacc[2] = fmaf(qj1, cf[2], sacc[2]);
          sacc[3] = fmaf(qj1, cf[3], sacc[3]);
        }
        acc[0] = fmaf(S0, sacc[0], acc[0]);
        acc[1] = fmaf(S0, sacc[1], acc[1]);
        acc[2] = fmaf(S1, sacc[2], acc[2]);
        acc[3] = fmaf(S1, sacc[3], acc[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  if (!ok) {
    if (lane == 0) {
      report(a.dev_status, GQ_DEV_TIMEOUT);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
    }
    return;
  }

  // reduce the four consumer warps' partial sums, then store
  float* my = red + (cw * 32 + lane) * 4;
  my[0] = acc[0];
  my[1] = acc[1];
  my[2] = acc[2];
  my[3] = acc[3];
  if (!group_sync()) {
    if (lane == 0) report(a.dev_status, GQ_DEV_TIMEOUT);
    return;
  }
  if (cw == 0) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float* p = red + (w * 32 + lane) * 4;
      s4[0] += p[0];
      s4[1] += p[1];
      s4[2] += p[2];
      s4[3] += p[3];
    }
    const int64_t ra = m0 + r, rb = m0 + r + 8;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int col = 2 * t + i;
      if (col < a.B) {
        if (ra < a.M) store_elem(a.y, col * a.M + ra, s4[i], a.ytype);
        if (rb < a.M) store_elem(a.y, col * a.M + rb, s4[2 + i], a.ytype);
      }
    }
  }
}

size_t gemv_smem_bytes(int B, int terms, int win) {
  return static_cast<size_t>(kStages) * kStageBytes +
         static_cast<size_t>(terms) * win * B * kXStride + kConsumers * 32 * 4 * sizeof(float) +
         (2 * kStages + 1) * sizeof(uint64_t) + 16;
}

template <int FMT, int XT>
gq_status launch_gemv(const GemvArgs& a, cudaStream_t stream, bool pdl) {
  constexpr int kTerms = (XT == XT_F32) ? 3 : 1;
  const size_t smem = gemv_smem_bytes(a.B, kTerms, a.win);
  static int configured_dev = -1;
  static size_t configured = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev || configured < smem) {
    const size_t want = static_cast<size_t>(kStages) * kStageBytes + kXSmemMax + 8192;
    if (cudaFuncSetAttribute(gemv_kernel<FMT, XT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(want)) != cudaSuccess)
      return GQ_ERR_CUDA;
    configured_dev = dev;
    configured = want;
  }
  const int64_t grid = (a.M + kRows - 1) / kRows;
  return launch(gemv_kernel<FMT, XT>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem,
                stream, pdl, a);
}

template <int FMT>
gq_status gemv_entry(const void* W, int64_t M, int64_t K, const void* x, int xt, int64_t B,
                     void* y, int yt, unsigned flags, int* dev_status, void* stream) {
  constexpr int kBlkW = Fmt<FMT>::kBlkW, kBlkB = Fmt<FMT>::kBlkB;
  if (M < 0 || K < 0 || B < 0) return GQ_ERR_INVALID_ARG;
  if (!valid_act_dtype(xt) || !valid_act_dtype(yt)) return GQ_ERR_DTYPE;
  if (flags & ~GQ_GEMV_PDL) return GQ_ERR_INVALID_ARG;
  if (K % kBlkW) return GQ_ERR_SHAPE;
  if (B > 8 || M > 0x7FFFFFFFLL || K > (1LL << 24)) return GQ_ERR_SHAPE;
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
  a.W = static_cast<const uint8_t*>(W);
  a.M = M;
  a.K = K;
  a.rowbytes = K / kBlkW * kBlkB;
  a.x = x;
  a.y = y;
  a.dev_status = dev_status;
  a.budget = kWaitBudget;
  a.B = static_cast<int>(B);
  a.ytype = yt;
  a.nchunks = static_cast<int>((K + kChunkW - 1) / kChunkW);
  const int terms = (xt == GQ_F32) ? 3 : 1;
  int win = kXSmemMax / (terms * a.B * kXStride);
  if (win < 1) win = 1;
  if (win > a.nchunks) win = a.nchunks;
  a.win = win;

  const bool pdl = (flags & GQ_GEMV_PDL) != 0;
  cudaStream_t s = as_stream(stream);
  switch (xt) {
    case GQ_F16: return launch_gemv<FMT, XT_F16>(a, s, pdl);
    case GQ_BF16: return launch_gemv<FMT, XT_BF16>(a, s, pdl);
    default: return launch_gemv<FMT, XT_F32>(a, s, pdl);
  }
}

}  // namespace
}  // namespace gq

extern "C" {

GQ_API gq_status gq_gemv_q4_0(const void* W, int64_t M, int64_t K, const void* x, int x_dtype,
                              int64_t B, void* y, int y_dtype, unsigned flags, int* dev_status,
                              void* stream) {
  return gq::gemv_entry<GQ_FMT_Q4_0>(W, M, K, x, x_dtype, B, y, y_dtype, flags, dev_status,
                                     stream);
}

GQ_API gq_status gq_gemv_ksb(const void* W, int64_t M, int64_t K, const void* x, int x_dtype,
                             int64_t B, void* y, int y_dtype, unsigned flags, int* dev_status,
                             void* stream) {
  return gq::gemv_entry<GQ_FMT_KSB>(W, M, K, x, x_dtype, B, y, y_dtype, flags, dev_status,
                                    stream);
}

}  // extern "C"
