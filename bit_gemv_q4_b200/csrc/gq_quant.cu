// gq_quant.cu -- block quantizers and dequantizers for Q4_0 and the
// super-block K-quant ("ksb").
//
// Q4_0: "GGUF 量化内幕 第4章" 4.1.2 (18-byte block), 4.2.1 (lo/hi nibble split),
//   4.2.2-4.3 (w = d * (code - 8)); the scale/code rule is the one fixed in gq.h.
// ksb:  "GGUF K-quants" section "套娃": eight sub-block FP16 scales quantized
//   to INT8 against one FP16 super-scale S = max/127; 2 + 8 + 128 bytes.
//
// Both directions are HBM-bound streams (4 B of fp32 per weight against
// 0.5625 / 0.539 B packed).  Loads are 128-bit and coalesced; a CTA builds
// the packed bytes of 64 Q4_0 blocks (1152 B) or 8 super-blocks (1104 B) in
// shared memory and writes them with 16-byte stores.  Block absmax values are
// warp-shuffle reductions over the 8 lanes that hold one 32-weight block.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_device.cuh"
#include "gq_host.h"

namespace gq {
namespace {

constexpr int kQThreads = 256;

// Four codes clamp(rint(fl32(v / d)) + 8, 0, 15) as four nibbles (first value
// in bits 0-3), with the IEEE quotient and round-half-even; a zero, infinite
// or NaN scale gives code 8.
//
// The quotient needs no divide per value: with r = RN(1/d) (one IEEE
// reciprocal per block), q = RN(v * r) is within one ulp of v/d, e = v - d*q
// is exact as an FMA, and RN(q + e * r) is the correctly rounded quotient
// (Markstein's theorem for division with a fused multiply-add: Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; Muller et al., Handbook of
// Floating-Point Arithmetic, the chapter on division and square root with an
// FMA), provided nothing underflows or overflows.  Here d is the block's own
// scale (absmax/7 rounded to FP16, or S * q_j within a factor 1.5 of it), so
// |v/d| <= 10.5 and nothing overflows; a quotient small enough to underflow
// is far from +-0.5 and its code is 8 whatever its last bits.  rint is
// an add of 1.5 * 2^23, exact and round-half-even for |t| < 2^22.
__device__ __forceinline__ uint32_t codes4(float4 v, float d, float r) {
  const bool special = !(d > 0.0f && d < INFINITY);
  const float2 r2 = make_float2(r, r), nd2 = make_float2(-d, -d);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
  float2 q01 = __fmul2_rn(v01, r2), q23 = __fmul2_rn(v23, r2);
  const float2 e01 = __ffma2_rn(q01, nd2, v01), e23 = __ffma2_rn(q23, nd2, v23);
  q01 = __fadd2_rn(__ffma2_rn(e01, r2, q01), magic);
  q23 = __fadd2_rn(__ffma2_rn(e23, r2, q23), magic);
  // bits(1.5 * 2^23 + k) = 0x4B400000 + k for |k| < 2^22
  const int bias = static_cast<int>(0x4B400000u) - 8;
  const int c[4] = {__float_as_int(q01.x) - bias, __float_as_int(q01.y) - bias,
                    __float_as_int(q23.x) - bias, __float_as_int(q23.y) - bias};
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) out |= static_cast<uint32_t>(min(max(c[i], 0), 15)) << (4 * i);
  return special ? 0x8888u : out;
}

// The reciprocal the codes of a block use (any value for a special scale).
__device__ __forceinline__ float recip_of(float d) { return __frcp_rn(d); }

// Spread four nibbles into the low nibbles of four bytes.
__device__ __forceinline__ uint32_t spread4(uint32_t a) {
  return (a & 0xFu) | ((a & 0xF0u) << 4) | ((a & 0xF00u) << 8) | ((a & 0xF000u) << 12);
}

// qs bytes for weights j..j+3 (low nibbles, from `lo`) and j+16..j+19 (high
// nibbles, from `hi`): the lo/hi split of the Q4_0 chapter, section 4.2.1.
__device__ __forceinline__ uint32_t pack_lohi(uint32_t lo, uint32_t hi) {
  return spread4(lo) | (spread4(hi) << 4);
}

__device__ __forceinline__ float absmax4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__device__ __forceinline__ bool finite4(float4 v) {
  return isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
}

// max over the 8 lanes of an aligned group of 8
__device__ __forceinline__ float group8_max(float a) {
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 4));
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

// ---------------------------------------------------------------- Q4_0 quantize
// CTA tile: 64 blocks (2048 floats).  Warp w owns blocks 8w..8w+7; in each of
// two passes its lanes hold 4 blocks, 8 lanes (one float4 each) per block.
__global__ void __launch_bounds__(kQThreads)
    quantize_q4_0_kernel(const float* __restrict__ x, int64_t nblk, uint8_t* __restrict__ out,
                         int* dev_status) {
  __shared__ __align__(16) uint8_t stage[64 * 18];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, sub = lane & 7;
  int flags = 0;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * 64; base < nblk;
       base += static_cast<int64_t>(gridDim.x) * 64) {
    const int nb = static_cast<int>(i64min(64, nblk - base));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int bl = warp * 8 + h * 4 + g;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bl < nb) v = __ldcs(reinterpret_cast<const float4*>(x + (base + bl) * 32) + sub);
      if (!finite4(v)) flags |= GQ_DEV_NONFINITE;
      const float a = group8_max(absmax4(v));
      const __half dh = __float2half_rn(__fdiv_rn(a, 7.0f));
      const float d = __half2float(dh);
      if (__hisinf(dh)) flags |= GQ_DEV_RANGE;
      const uint32_t c = codes4(v, d, recip_of(d));
      const uint32_t partner = __shfl_xor_sync(0xFFFFFFFFu, c, 4);
      if (bl < nb) {
        uint8_t* blk = stage + bl * 18;
        if (sub == 0) st_u16(blk, __half_as_ushort(dh));
        if (sub < 4) {
          const uint32_t b = pack_lohi(c, partner);
          st_u16(blk + 2 + 4 * sub, b & 0xFFFFu);
          st_u16(blk + 4 + 4 * sub, b >> 16);
        }
      }
    }
    __syncthreads();
    flush_tile(out + base * 18, stage, nb * 18, 64 * 18);
    __syncthreads();
  }
  if (flags) report(dev_status, flags);
}

// ----------------------------------------------------------------- ksb quantize
// CTA tile: 8 super-blocks; warp w owns super-block w.  Lane l holds float4 l
// (sub-block l/8) and float4 32+l (sub-block 4+l/8).
__global__ void __launch_bounds__(kQThreads)
    quantize_ksb_kernel(const float* __restrict__ x, int64_t nsb, uint8_t* __restrict__ out,
                        int* dev_status) {
  __shared__ __align__(16) uint8_t stage[8 * 138];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, sub = lane & 7;
  int flags = 0;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * 8; base < nsb;
       base += static_cast<int64_t>(gridDim.x) * 8) {
    const int ns = static_cast<int>(i64min(8, nsb - base));
    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
    if (warp < ns) {
      const float4* p = reinterpret_cast<const float4*>(x + (base + warp) * 256);
      v0 = __ldcs(p + lane);
      v1 = __ldcs(p + 32 + lane);
    }
    if (!finite4(v0) || !finite4(v1)) flags |= GQ_DEV_NONFINITE;
    // each sub-block's own FP16 scale, absmax / 7
    const __half d0h = __float2half_rn(__fdiv_rn(group8_max(absmax4(v0)), 7.0f));
    const __half d1h = __float2half_rn(__fdiv_rn(group8_max(absmax4(v1)), 7.0f));
    if (__hisinf(d0h) || __hisinf(d1h)) flags |= GQ_DEV_RANGE;
    const float d0 = __half2float(d0h), d1 = __half2float(d1h);
    // super-scale S = FP16(max_j d_j / 127)
    float m = fmaxf(d0, d1);
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
    const __half sh = __float2half_rn(__fdiv_rn(m, 127.0f));
    const float S = __half2float(sh);
    int q0 = 0, q1 = 0;
    if (S != 0.0f && !__hisinf(sh)) {
      q0 = min(max(__float2int_rn(__fdiv_rn(d0, S)), 0), 127);
      q1 = min(max(__float2int_rn(__fdiv_rn(d1, S)), 0), 127);
    }
    // codes against the scale the decoder rebuilds, S * q_j
    const float st0 = __fmul_rn(S, static_cast<float>(q0));
    const float st1 = __fmul_rn(S, static_cast<float>(q1));
    const uint32_t c0 = codes4(v0, st0, recip_of(st0)), c1 = codes4(v1, st1, recip_of(st1));
    const uint32_t p0 = __shfl_xor_sync(0xFFFFFFFFu, c0, 4);
    const uint32_t p1 = __shfl_xor_sync(0xFFFFFFFFu, c1, 4);
    if (warp < ns) {
      uint8_t* sb = stage + warp * 138;
      if (lane == 0) st_u16(sb, __half_as_ushort(sh));
      if (sub == 0) {
        sb[2 + g] = static_cast<uint8_t>(q0);
        sb[6 + g] = static_cast<uint8_t>(q1);
      }
      if (sub < 4) {
        const uint32_t b0 = pack_lohi(c0, p0), b1 = pack_lohi(c1, p1);
        uint8_t* s0 = sb + 10 + 16 * g + 4 * sub;
        uint8_t* s1 = sb + 10 + 16 * (4 + g) + 4 * sub;
        st_u16(s0, b0 & 0xFFFFu);
        st_u16(s0 + 2, b0 >> 16);
        st_u16(s1, b1 & 0xFFFFu);
        st_u16(s1 + 2, b1 >> 16);
      }
    }
    __syncthreads();
    flush_tile(out + base * 138, stage, ns * 138, 8 * 138);
    __syncthreads();
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

GQ_API gq_status gq_quantize_q4_0(const float* x, int64_t n, void* out, int* dev_status,
                                  void* stream) {
  gq_status s = check_common(x, n, 32, out, dev_status);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nblk = n / 32;
  return launch(quantize_q4_0_kernel, dim3(stream_grid((nblk + 63) / 64)), dim3(kQThreads), 0,
                as_stream(stream), false, x, nblk, static_cast<uint8_t*>(out), dev_status);
}

GQ_API gq_status gq_quantize_ksb(const float* x, int64_t n, void* out, int* dev_status,
                                 void* stream) {
  gq_status s = check_common(x, n, 256, out, dev_status);
  if (s != GQ_OK || n == 0) return s;
  const int64_t nsb = n / 256;
  return launch(quantize_ksb_kernel, dim3(stream_grid((nsb + 7) / 8)), dim3(kQThreads), 0,
                as_stream(stream), false, x, nsb, static_cast<uint8_t*>(out), dev_status);
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
