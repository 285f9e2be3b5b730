// gq_gemv_grouped.cu -- the grouped GEMV for large tables: gq_gemv.cu's
// kernel compiled with a pipeline of four small CTAs per SM (1024-weight
// chunks, four stages, four consumer warps each) instead of two wide ones.
// A grouped call with many row groups per SM streams without launch gaps,
// and there more independent pipelines per SM keep the consumer warps busier
// (measured on the 224-matrix decoder stream: 3.94 against 3.74 TB/s);
// single launches and short tables keep the wide configuration.  Only
// gq::gemv_grouped_many is defined here; everything else of gq_gemv.cu sits
// in this unit's anonymous namespace.
#undef GQ_GEMV_CHUNK
#undef GQ_GEMV_STAGES
#undef GQ_GEMV_CONSUMERS
#undef GQ_GEMV_MINB
#define GQ_GEMV_CHUNK 1024
#define GQ_GEMV_STAGES 4
#define GQ_GEMV_CONSUMERS 4
#define GQ_GEMV_MINB 4
#define GQ_GEMV_MANY_TU 1
#include "gq_gemv.cu"
