// gq_quant.cu -- block quantizers and dequantizers for Q4_0 and the
// super-block K-quant ("ksb").
//
// Q4_0: "GGUF 量化内幕 第4章" 4.1.2 (18-byte block), 4.2.1 (lo/hi nibble split),
//   4.2.2-4.3 (w = d * (code - 8)); the scale/code rule is the one fixed in gq.h.
// ksb:  "GGUF K-quants" section "套娃": eight sub-block FP16 scales quantized
//   to INT8 against one FP16 super-scale S = max/127; 2 + 8 + 128 bytes.
//
// Both directions are HBM-bound streams (4 B of fp32 per weight against
// 0.5625 / 0.539 B packed).  Loads are 128-bit and coalesced; a quantizer CTA
// builds the packed bytes of 128 Q4_0 blocks (2304 B) or 16 super-blocks
// (2208 B) in shared memory and writes them with 16-byte stores.  Four lanes
// hold one 32-weight block; its absmax is a shuffle reduction over them.  The
// quantizers run near the SM issue rate as much as the HBM rate, so the
// per-weight work avoids divides and per-code branches (below).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_host.h"

namespace gq {
namespace {

constexpr int kQThreads = 256;

// Division without a divide.  Every divisor here has a short significand:
// the FP16 scales (11 bits), S * q_j (at most 18 bits), 7 and 127.  With
// rb = RN(1/b), q = RN(a * rb) is within 1.5 ulp of a/b, the residual
// a - q*b comes from one FMA, and RN(q + (a - q*b) * rb) is the correctly
// rounded quotient.  This is Markstein's FMA division step (Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; Muller et al., Handbook of
// Floating-Point Arithmetic, the chapter on division with an FMA); the short
// divisor is what makes one step enough:
//   * the exact value of the corrected sum differs from a/b by at most
//     (1.5 ulp) * 2^-24 from rb and the same again if the residual rounds,
//     under 2^-22 ulp;
//   * a/b is never a midpoint between floats (a 24-bit a over a b of p bits
//     cannot equal a 25-bit odd significand), and a/b - m for a midpoint m is
//     a nonzero multiple of 2^(e_m - 24 - p) divided by b, at least
//     2^-(p+1) ulp = 2^-19 ulp for p = 18;
//   so the final rounding sees a/b's own side of every midpoint.  Operands
// are finite, a >= 0 or of either sign with |a/b| bounded, b > 0 normal; a
// quotient that underflows fp32 is below every FP16 and code threshold and
// its last bits never matter.
__device__ __forceinline__ float div_short(float a, float b, float rb) {
  const float q = __fmul_rn(a, rb);
  return __fmaf_rn(__fmaf_rn(-q, b, a), rb, q);
}

// FP16(fl32(a / 7)) and FP16(fl32(a / 127)) for maxima a >= 0; a = +inf or
// NaN (a block of NaNs only) passes through as the IEEE quotient would.
constexpr float kInv7 = 1.0f / 7.0f;
constexpr float kInv127 = 1.0f / 127.0f;
__device__ __forceinline__ __half scale_over(float a, float b, float rb) {
  return __float2half_rn(a < INFINITY ? div_short(a, b, rb) : a);
}

// Two codes clamp(rint(fl32(v / d)) + 8, 0, 15) as the halves of an s16x2,
// the quotient correctly rounded (div_short's argument, with r = RN(1/d)) and
// rint half to even.  d is the block's own scale (absmax/7 in FP16, or
// S * q_j within a factor 1.5 of it), so |v/d| <= 16: adding 1.5 * 2^23 + 8
// rounds to an integer exactly and half-even (8 is even), and the low 16 bits
// of the sum's encoding are rint(v/d) + 8 as a signed 16-bit value.  A NaN v
// gives some code in range (its block is reported non-finite).
__device__ __forceinline__ uint32_t code_pair(float a, float b, float d, float r) {
  const float2 v = make_float2(a, b), r2 = make_float2(r, r);
  float2 q = __fmul2_rn(v, r2);
  const float2 e = __ffma2_rn(q, make_float2(-d, -d), v);
  q = __fadd2_rn(__ffma2_rn(e, r2, q), make_float2(12582920.0f, 12582920.0f));
  const uint32_t k = __byte_perm(__float_as_uint(q.x), __float_as_uint(q.y), 0x5410);
  return __vimin_s16x2_relu(k, 0x000F000Fu);  // max(min(k, 15), 0) per half
}

// The four qs bytes of one lane: byte i = code(lo[i]) | code(hi[i]) << 4, the
// lo/hi split of the Q4_0 chapter, section 4.2.1 (lo holds weights 4t..4t+3,
// hi weights 16+4t..19+4t).  A zero, infinite or NaN scale gives code 8.
__device__ __forceinline__ uint32_t qs_bytes(float4 lo, float4 hi, float d) {
  const float r = __frcp_rn(d);
  const uint32_t b01 = code_pair(lo.x, lo.y, d, r) | (code_pair(hi.x, hi.y, d, r) << 4);
  const uint32_t b23 = code_pair(lo.z, lo.w, d, r) | (code_pair(hi.z, hi.w, d, r) << 4);
  const bool special = !(d > 0.0f && d < INFINITY);
  return special ? 0x88888888u : __byte_perm(b01, b23, 0x6420);
}

// max |v| over a lane's eight values with NaN propagation (NaN if any value
// is NaN, else +inf if any is infinite), so one compare finds a non-finite
// input.  The xorsign form takes absolute values of its operands; the sign it
// leaves is dropped at the end.
__device__ __forceinline__ float amax_nan(float a, float b) {
  float r;
  asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float absmax8(float4 u, float4 v) {
  const float a = amax_nan(amax_nan(u.x, u.y), amax_nan(u.z, u.w));
  const float b = amax_nan(amax_nan(v.x, v.y), amax_nan(v.z, v.w));
  return fabsf(amax_nan(a, b));
}

// max over the 4 lanes of an aligned group of 4
__device__ __forceinline__ float group4_max(float a) {
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
  return a;
}

__device__ __forceinline__ void st_u16(uint8_t* p, uint32_t v) {
  *reinterpret_cast<unsigned short*>(p) = static_cast<unsigned short>(v);
}

// Write `nbytes` (even) staged bytes to global memory; whole tiles use 16-byte
// stores, a ragged tail 2-byte stores.
__device__ __forceinline__ void flush_tile(uint8_t* dst, const uint8_t* stage, int nbytes,
                                           int full_bytes) {
  if (nbytes == full_bytes) {
    for (int i = threadIdx.x; i < full_bytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(stage)[i];
  } else {
    for (int i = threadIdx.x; i < nbytes / 2; i += blockDim.x)
      reinterpret_cast<unsigned short*>(dst)[i] =
          reinterpret_cast<const unsigned short*>(stage)[i];
  }
}

// ------------------------------------------- the page's reference Q4_0 rule
// Q4_0 chapter 4.4 (its printed quantizer): the signed value of largest
// magnitude (the first such value of the block on ties) sets d = max / -8;
// with id = 1/d (0 when d is 0) code = min(15, trunc(x * id + 8.5)), the
// product and the sum each rounded to fp32.  Dividing by -8 is exact, so d is
// max * -0.125; a NaN value never becomes the max.

// 64-bit ordering key of value v at block position i: larger magnitude first,
// then the earlier position, the sign in bit 0; 0 for NaN and for zeros, so
// that a block of zeros takes max = +0 as the page's loop (which starts from
// 0 and only replaces it on a strictly larger magnitude) does.
__device__ __forceinline__ unsigned long long smax_key(float v, int i) {
  const uint32_t bits = __float_as_uint(v), mag = bits & 0x7FFFFFFFu;
  if (isnan(v) || mag == 0u) return 0ull;
  return (static_cast<unsigned long long>(mag) << 32) | (static_cast<uint32_t>(31 - i) << 1) |
         (bits >> 31);
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  const uint32_t mag = static_cast<uint32_t>(k >> 32), sign = static_cast<uint32_t>(k) & 1u;
  return __uint_as_float(mag | (sign << 31));
}

// The four qs bytes of one lane (weights 4t..4t+3 in lo, 16+4t.. in hi)
// under the reference rule, with id = 1/d.
__device__ __forceinline__ uint32_t ref_code(float v, float id) {
  const float tt = __fadd_rn(__fmul_rn(v, id), 8.5f);
  const int c = (tt >= 0.0f && tt < 1e9f) ? __float2int_rz(tt) : 0;
  return static_cast<uint32_t>(c < 15 ? c : 15);
}
__device__ __forceinline__ uint32_t ref_qs_bytes(float4 lo, float4 hi, float id) {
  return (ref_code(lo.x, id) | (ref_code(hi.x, id) << 4)) |
         ((ref_code(lo.y, id) | (ref_code(hi.y, id) << 4)) << 8) |
         ((ref_code(lo.z, id) | (ref_code(hi.z, id) << 4)) << 16) |
         ((ref_code(lo.w, id) | (ref_code(hi.w, id) << 4)) << 24);
}

// Scale of the reference rule for the block whose values this lane group of
// four holds (lane t: positions 4t..4t+3 and 16+4t..19+4t).
__device__ __forceinline__ float ref_scale(float4 lo, float4 hi, int t) {
  unsigned long long k = smax_key(lo.x, 4 * t);
  const float lv[4] = {lo.x, lo.y, lo.z, lo.w}, hv[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long a = smax_key(lv[i], 4 * t + i);
    const unsigned long long b = smax_key(hv[i], 16 + 4 * t + i);
    k = a > k ? a : k;
    k = b > k ? b : k;
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, k, o);
    k = other > k ? other : k;
  }
  return __fmul_rn(key_value(k), -0.125f);
}

// ---------------------------------------------------------------- Q4_0 quantize
// CTA tile: 128 blocks (4096 floats).  Four lanes share a block: lane t of a
// block holds weights 4t..4t+3 and 16+4t..19+4t, the two halves whose codes
// fill qs bytes 4t..4t+3, so a lane packs its bytes without a partner.  Warp w
// owns blocks 16w..16w+15, eight per pass.  A CTA walks its tiles with the
// next tile's loads issued before the current tile is packed, so each lane
// keeps 64 B of reads in flight while it computes.
constexpr int kQ0Tile = 128;

template <bool REF_RULE>
__global__ void __launch_bounds__(kQThreads)
    quantize_q4_0_kernel(const float* __restrict__ x, int64_t nblk, uint8_t* __restrict__ out,
                         int* dev_status) {
  __shared__ __align__(16) uint8_t stage[kQ0Tile * 18];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = lane & 3;
  int flags = 0;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kQ0Tile;
  // this lane's two float4 of pass h of the tile at `b`
  auto load = [&](int64_t b, float4 (&l)[2], float4 (&u)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t bl = b + warp * 16 + h * 8 + (lane >> 2);
      l[h] = u[h] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bl < nblk) {
        const float4* src = reinterpret_cast<const float4*>(x + bl * 32);
        l[h] = __ldcs(src + t);
        u[h] = __ldcs(src + 4 + t);
      }
    }
  };
  float4 lo[2], hi[2];
  load(static_cast<int64_t>(blockIdx.x) * kQ0Tile, lo, hi);
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kQ0Tile; base < nblk; base += step) {
    const int nb = static_cast<int>(i64min(kQ0Tile, nblk - base));
    float4 nlo[2], nhi[2];  // the next tile's values, in flight while this one is packed
    load(base + step, nlo, nhi);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int bl = warp * 16 + h * 8 + (lane >> 2);
      const float own = absmax8(lo[h], hi[h]);
      if (!(own < INFINITY)) flags |= GQ_DEV_NONFINITE;
      __half dh;
      uint32_t b;
      if constexpr (REF_RULE) {
        const float d = ref_scale(lo[h], hi[h], t);
        dh = __float2half_rn(d);
        b = ref_qs_bytes(lo[h], hi[h], d != 0.0f ? __frcp_rn(d) : 0.0f);
      } else {
        dh = scale_over(group4_max(own), 7.0f, kInv7);
        b = qs_bytes(lo[h], hi[h], __half2float(dh));
      }
      if (__hisinf(dh)) flags |= GQ_DEV_RANGE;
      if (bl < nb) {
        uint8_t* blk = stage + bl * 18;
        if (t == 0) st_u16(blk, __half_as_ushort(dh));
        st_u16(blk + 2 + 4 * t, b & 0xFFFFu);
        st_u16(blk + 4 + 4 * t, b >> 16);
      }
    }
    __syncthreads();
    flush_tile(out + base * 18, stage, nb * 18, kQ0Tile * 18);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lo[h] = nlo[h];
      hi[h] = nhi[h];
    }
  }
  if (flags) report(dev_status, flags);
}

// ----------------------------------------------------------------- ksb quantize
// CTA tile: 16 super-blocks; warp w owns super-blocks w and 8 + w, one per
// pass, with the next tile's loads in flight as in the Q4_0 kernel.  Lane
// 4j + t holds, of sub-block j, weights 4t..4t+3 and 16+4t..19+4t (the Q4_0
// lane split of one block).
constexpr int kKsbTile = 16;

__global__ void __launch_bounds__(kQThreads)
    quantize_ksb_kernel(const float* __restrict__ x, int64_t nsb, uint8_t* __restrict__ out,
                        int* dev_status) {
  __shared__ __align__(16) uint8_t stage[kKsbTile * 138];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = lane >> 2, t = lane & 3;
  int flags = 0;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kKsbTile;
  auto load = [&](int64_t b, float4 (&l)[2], float4 (&u)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t sb = b + warp + 8 * h;
      l[h] = u[h] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (sb < nsb) {
        const float4* src = reinterpret_cast<const float4*>(x + sb * 256 + 32 * j);
        l[h] = __ldcs(src + t);
        u[h] = __ldcs(src + 4 + t);
      }
    }
  };
  float4 lo[2], hi[2];
  load(static_cast<int64_t>(blockIdx.x) * kKsbTile, lo, hi);
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kKsbTile; base < nsb; base += step) {
    const int ns = static_cast<int>(i64min(kKsbTile, nsb - base));
    float4 nlo[2], nhi[2];  // the next tile's values, in flight while this one is packed
    load(base + step, nlo, nhi);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int sb = warp + 8 * h;
      const float own = absmax8(lo[h], hi[h]);
      if (!(own < INFINITY)) flags |= GQ_DEV_NONFINITE;
      // the sub-block's own FP16 scale, absmax / 7
      const __half dh = scale_over(group4_max(own), 7.0f, kInv7);
      if (__hisinf(dh)) flags |= GQ_DEV_RANGE;
      const float d = __half2float(dh);
      // super-scale S = FP16(max_j d_j / 127)
      float m = d;
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
      const __half sh = scale_over(m, 127.0f, kInv127);
      const float S = __half2float(sh);
      int q = 0;
      if (S != 0.0f && !__hisinf(sh))
        q = min(max(__float2int_rn(div_short(d, S, __frcp_rn(S))), 0), 127);
      // codes against the scale the decoder rebuilds, S * q_j
      const float st = __fmul_rn(S, static_cast<float>(q));
      const uint32_t b = qs_bytes(lo[h], hi[h], st);
      if (sb < ns) {
        uint8_t* blk = stage + sb * 138;
        if (lane == 0) st_u16(blk, __half_as_ushort(sh));
        if (t == 0) blk[2 + j] = static_cast<uint8_t>(q);
        uint8_t* qs = blk + 10 + 16 * j + 4 * t;
        st_u16(qs, b & 0xFFFFu);
        st_u16(qs + 2, b >> 16);
      }
    }
    __syncthreads();
    flush_tile(out + base * 138, stage, ns * 138, kKsbTile * 138);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lo[h] = nlo[h];
      hi[h] = nhi[h];
    }
  }
  if (flags) report(dev_status, flags);
}

// -------------------------------------------------------------- dequantizers
// Stage a tile of packed bytes (a whole number of 16-byte granules, the last
// one possibly running past the data up to its 16-byte boundary).
__device__ __forceinline__ void load_tile(uint8_t* stage, const uint8_t* src, int nbytes) {
  const int ng = (nbytes + 15) / 16;
  for (int i = threadIdx.x; i < ng; i += blockDim.x)
    reinterpret_cast<uint4*>(stage)[i] = __ldcs(reinterpret_cast<const uint4*>(src) + i);
}

// Q4_0 chapter 4.3: w[j] = d * (lo(qs[j]) - 8), w[j+16] = d * (hi(qs[j]) - 8).
// CTA tile: 64 blocks in, 512 float4 out (two per thread, coalesced).
__global__ void __launch_bounds__(kQThreads)
    dequantize_q4_0_kernel(const uint8_t* __restrict__ q, int64_t nblk, float* __restrict__ out) {
  __shared__ __align__(16) uint8_t stage[64 * 18 + 16];  // +16: slack for 8-byte window reads
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * 64; base < nblk;
       base += static_cast<int64_t>(gridDim.x) * 64) {
    const int nb = static_cast<int>(i64min(64, nblk - base));
    load_tile(stage, q + base * 18, nb * 18);
    __syncthreads();
    const uint32_t s0 = smem_addr(stage);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = threadIdx.x + h * kQThreads;  // float4 index in the tile
      const int bl = f >> 3, p = (f & 7) * 4;     // block, first weight
      if (bl < nb) {
        const uint32_t blk = s0 + bl * 18;
        const float d = half_bits_to_float(lds16(blk));
        const uint32_t w = lds32_even(blk + 2 + (p & 15));
        const uint32_t sh = (p >= 16) ? 4u : 0u;
        float4 o;
        o.x = __fmul_rn(d, static_cast<float>(static_cast<int>((w >> sh) & 15u) - 8));
        o.y = __fmul_rn(d, static_cast<float>(static_cast<int>((w >> (8 + sh)) & 15u) - 8));
        o.z = __fmul_rn(d, static_cast<float>(static_cast<int>((w >> (16 + sh)) & 15u) - 8));
        o.w = __fmul_rn(d, static_cast<float>(static_cast<int>((w >> (24 + sh)) & 15u) - 8));
        __stcs(reinterpret_cast<float4*>(out + (base + bl) * 32 + p), o);
      }
    }
    __syncthreads();
  }
}

// K-quants post, step 5: s~_j = S * q_j, then w = s~_j * (code - 8).
// CTA tile: 8 super-blocks in, 512 float4 out.
__global__ void __launch_bounds__(kQThreads)
    dequantize_ksb_kernel(const uint8_t* __restrict__ q, int64_t nsb, float* __restrict__ out) {
  __shared__ __align__(16) uint8_t stage[8 * 138 + 16];
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * 8; base < nsb;
       base += static_cast<int64_t>(gridDim.x) * 8) {
    const int ns = static_cast<int>(i64min(8, nsb - base));
    load_tile(stage, q + base * 138, ns * 138);
    __syncthreads();
    const uint32_t s0 = smem_addr(stage);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = threadIdx.x + h * kQThreads;  // float4 index in the tile
      const int sb = f >> 6, j = (f >> 3) & 7, p = (f & 7) * 4;
      if (sb < ns) {
        const uint32_t blk = s0 + sb * 138;
        const float S = half_bits_to_float(lds16(blk));
        const int qj = static_cast<int8_t>(stage[sb * 138 + 2 + j]);
        const float st = __fmul_rn(S, static_cast<float>(qj));
        const uint32_t w = lds32_even(blk + 10 + 16 * j + (p & 15));
        const uint32_t sh = (p >= 16) ? 4u : 0u;
        float4 o;
        o.x = __fmul_rn(st, static_cast<float>(static_cast<int>((w >> sh) & 15u) - 8));
        o.y = __fmul_rn(st, static_cast<float>(static_cast<int>((w >> (8 + sh)) & 15u) - 8));
        o.z = __fmul_rn(st, static_cast<float>(static_cast<int>((w >> (16 + sh)) & 15u) - 8));
        o.w = __fmul_rn(st, static_cast<float>(static_cast<int>((w >> (24 + sh)) & 15u) - 8));
        __stcs(reinterpret_cast<float4*>(out + (base + sb) * 256 + 32 * j + p), o);
      }
    }
    __syncthreads();
  }
}

int stream_grid(int64_t tiles) {
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(tiles < cap ? (tiles > 0 ? tiles : 1) : cap);
}

// One wave of resident CTAs (or fewer when there are fewer tiles): the
// quantizers prefetch across their own tiles, so a second wave would only
// add a tail.
template <typename Kernel>
int resident_grid(Kernel kernel, int64_t tiles) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQThreads, 0) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  return static_cast<int>(tiles < cap ? (tiles > 0 ? tiles : 1) : cap);
}

gq_status check_common(const void* in, int64_t n, int block, const void* out, const int* st) {
  if (n < 0) return GQ_ERR_INVALID_ARG;
  if (n % block) return GQ_ERR_SHAPE;
  if (n == 0) return GQ_OK;
  if (!in || !out) return GQ_ERR_INVALID_ARG;
  if (misaligned16(in) || misaligned16(out)) return GQ_ERR_ALIGNMENT;
  if (st && (reinterpret_cast<uintptr_t>(st) & 3u)) return GQ_ERR_ALIGNMENT;
  return GQ_OK;
}

}  // namespace
}  // namespace gq

using namespace gq;

extern "C" {

GQ_API gq_status gq_quantize_q4_0_ex(const float* x, int64_t n, void* out, unsigned flags,
                                     int* dev_status, void* stream) {
  if (flags & ~GQ_QUANT_REF_RULE) return GQ_ERR_INVALID_ARG;
  gq_status s = check_common(x, n, 32, out, dev_status);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nblk = n / 32;
  const int64_t tiles = (nblk + kQ0Tile - 1) / kQ0Tile;
  uint8_t* o = static_cast<uint8_t*>(out);
  if (flags & GQ_QUANT_REF_RULE) {
    const dim3 grid(resident_grid(quantize_q4_0_kernel<true>, tiles));
    return launch(quantize_q4_0_kernel<true>, grid, dim3(kQThreads), 0, as_stream(stream), false,
                  x, nblk, o, dev_status);
  }
  const dim3 grid(resident_grid(quantize_q4_0_kernel<false>, tiles));
  return launch(quantize_q4_0_kernel<false>, grid, dim3(kQThreads), 0, as_stream(stream), false, x,
                nblk, o, dev_status);
}

GQ_API gq_status gq_quantize_q4_0(const float* x, int64_t n, void* out, int* dev_status,
                                  void* stream) {
  return gq_quantize_q4_0_ex(x, n, out, 0u, dev_status, stream);
}

GQ_API gq_status gq_quantize_ksb(const float* x, int64_t n, void* out, int* dev_status,
                                 void* stream) {
  gq_status s = check_common(x, n, 256, out, dev_status);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nsb = n / 256;
  const dim3 grid(resident_grid(quantize_ksb_kernel, (nsb + kKsbTile - 1) / kKsbTile));
  return launch(quantize_ksb_kernel, grid, dim3(kQThreads), 0, as_stream(stream), false, x, nsb,
                static_cast<uint8_t*>(out), dev_status);
}

GQ_API gq_status gq_dequantize_q4_0(const void* q, int64_t n, float* out, void* stream) {
  gq_status s = check_common(q, n, 32, out, nullptr);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nblk = n / 32;
  return launch(dequantize_q4_0_kernel, dim3(stream_grid((nblk + 63) / 64)), dim3(kQThreads), 0,
                as_stream(stream), false, static_cast<const uint8_t*>(q), nblk, out);
}

GQ_API gq_status gq_dequantize_ksb(const void* q, int64_t n, float* out, void* stream) {
  gq_status s = check_common(q, n, 256, out, nullptr);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nsb = n / 256;
  return launch(dequantize_ksb_kernel, dim3(stream_grid((nsb + 7) / 8)), dim3(kQThreads), 0,
                as_stream(stream), false, static_cast<const uint8_t*>(q), nsb, out);
}

}  // extern "C"
