// gq_stream_read.cu -- a plain streaming read of a buffer: the practical
// ceiling of one launch that reads a given number of bytes once.
//
// The GEMV streams each weight byte from HBM exactly once; how fast a single
// launch of that size can read its bytes at all (launch, ramp-up and drain
// included) is the reference its measured time is compared with, beside the
// long-copy peak.  This kernel does nothing but read: 16-byte streaming loads
// (evict-first), a grid of eight 256-thread CTAs per SM striding over the
// buffer, and an XOR fold of every 32-bit word so that the loads have a
// checkable result (one atomic per CTA).
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"
#include "gq_host.h"

namespace gq {
namespace {

constexpr int kThreads = 256;
constexpr int kCtasPerSm = 8;

__global__ void __launch_bounds__(kThreads) stream_read_kernel(const uint4* __restrict__ p,
                                                               size_t n16, uint32_t* sink) {
  uint32_t acc = 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * kThreads;
  size_t i = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x;
  // four independent loads in flight per thread
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = __ldcs(p + i), b = __ldcs(p + i + stride);
    const uint4 c = __ldcs(p + i + 2 * stride), d = __ldcs(p + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w;
    acc ^= c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n16; i += stride) {
    const uint4 a = __ldcs(p + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  // one atomic per CTA: the folds of its warps meet in shared memory first
  __shared__ uint32_t part[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t v = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v ^= part[w];
    if (v != 0) atomicXor(sink, v);
  }
}

}  // namespace
}  // namespace gq

extern "C" {

GQ_API gq_status gq_stream_read(const void* p, size_t bytes, uint32_t* sink, void* stream) {
  using namespace gq;
  if (!sink || (bytes && !p)) return GQ_ERR_INVALID_ARG;
  if (misaligned16(p) || (reinterpret_cast<uintptr_t>(sink) & 3u)) return GQ_ERR_ALIGNMENT;
  if (bytes % 16) return GQ_ERR_SHAPE;
  if (bytes == 0) return GQ_OK;
  const size_t n16 = bytes / 16;
  const size_t want = (n16 + kThreads - 1) / kThreads;
  const int grid = static_cast<int>(want < static_cast<size_t>(kCtasPerSm) * sm_count()
                                        ? want
                                        : static_cast<size_t>(kCtasPerSm) * sm_count());
  return launch(stream_read_kernel, dim3(grid), dim3(kThreads), 0, as_stream(stream), false,
                static_cast<const uint4*>(p), n16, sink);
}

}  // extern "C"
