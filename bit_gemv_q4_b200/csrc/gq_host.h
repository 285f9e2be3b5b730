// gq_host.h -- host-side helpers shared by the entry points of libgq:
// argument checks that run before any launch, device property caching and
// the launch wrapper.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"

namespace gq {

inline bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool valid_act_dtype(int t) { return t == GQ_F32 || t == GQ_F16 || t == GQ_BF16; }

inline int dtype_size(int t) { return t == GQ_F32 ? 4 : 2; }

// Number of SMs of the current device (looked up once per device).
int sm_count();

// Process-unique ID of the calling thread's current CUDA context (0 if there
// is none yet, or the driver cannot say).  Per-context state -- function
// attributes, symbol addresses -- is keyed by it, so that it is set up again
// when a context is destroyed and another one created.
unsigned long long context_id();

// cuTensorMapEncodeTiled from the driver (looked up once; null if missing).
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiled tensor_map_encoder();

// cudaLaunchKernelEx wrapper; `pdl` adds programmatic stream serialization.
template <typename... KArgs, typename... Args>
gq_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                 cudaStream_t stream, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  return e == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

// As launch(), as clusters of `cluster` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
gq_status launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t stream, bool pdl, unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.numAttrs = 1;
  if (pdl) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  cfg.attrs = attr;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  return e == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

}  // namespace gq
