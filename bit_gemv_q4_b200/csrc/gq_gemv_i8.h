// gq_gemv_i8.h -- the batch-1 integer tensor-core GEMV (gq_gemv_i8.cu), as
// seen by the gq_gemv_* entry points.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gq.h"

namespace gq {

// Whether a call with these arguments takes the integer path when given a
// workspace: Q4_0, batch 1, fp16 x, K a multiple of 256 (rows of whole
// 16-byte granules), W 16-byte aligned, and K short enough for the plan.
bool i8_eligible(int fmt, int64_t M, int64_t K, int64_t B, int xt, const void* W);
// The same test without the device's SM count (which only bounds the
// scratch of gq_gemv_q4_0_noalloc, checked there).
bool i8_shape_ok(int fmt, int64_t M, int64_t K, int64_t B, int xt, const void* W);

// Workspace bytes of that path for an M x K matrix on the current device.
size_t i8_workspace_bytes(int64_t M, int64_t K);

// Launches the GEMV (it splits x itself) on `stream`.
gq_status i8_gemv(const void* W, int64_t M, int64_t K, const void* x, void* y, int yt,
                  void* workspace, size_t ws_bytes, bool pdl, int* dev_status,
                  cudaStream_t stream);

// The same path with static device scratch instead of a workspace (the
// counts are cleared in stream order before each launch).
gq_status i8_gemv_noalloc(const void* W, int64_t M, int64_t K, const void* x, void* y, int yt,
                          bool pdl, int* dev_status, cudaStream_t stream);

}  // namespace gq
