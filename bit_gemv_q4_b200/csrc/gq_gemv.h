// gq_gemv.h -- the warp-MMA dequantize-fused product of gq_gemv.cu as seen by
// the other entry points of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gq.h"

namespace gq {

// Largest batch the warp-MMA product takes (two n8 tiles of the MMA's N).
constexpr int64_t kWarpMmaMaxB = 16;

// Y[B][M] = W_hat[M][K] * x[B][K]^T for 1 <= B <= kWarpMmaMaxB on the warp-MMA
// path of gq_gemv_* (fmt GQ_FMT_Q4_0 or GQ_FMT_KSB), launched on `stream`.
// Arguments, validation and status as for gq_gemv_q4_0 with no workspace and
// no flags, except the larger batch.  Small-batch GEMMs use it: below about
// 16 columns a tcgen05 MMA spends most of its fixed cost on empty columns.
gq_status gemv_batched(int fmt, const void* W, int64_t M, int64_t K, const void* x, int xt,
                       int64_t B, void* y, int yt, int* dev_status, cudaStream_t stream);

// gq_gemv_*_grouped on the large-table configuration (gq_gemv_grouped.cu:
// four small CTAs per SM, 1024-weight chunks), for tables with many row
// groups per SM.  Arguments, validation and status as for the grouped entry
// points; results differ from the single-matrix product only in the order
// of fp32 additions.
gq_status gemv_grouped_many(int fmt, const gq_gemv_desc* mats, int count, int64_t K,
                            const void* x, int xt, int64_t B, int yt, unsigned flags,
                            int* dev_status, cudaStream_t stream);

}  // namespace gq
