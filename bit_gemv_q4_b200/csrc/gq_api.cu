// gq_api.cu -- entry points of libgq that launch nothing: version, status
// strings, device-status decoding and packed sizes.
#include <cuda_runtime.h>

#include <atomic>

#include "gq.h"
#include "gq_host.h"

namespace gq {

int sm_count() {
  static std::atomic<int> cached[64];  // zero-initialized; same value from every thread
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

unsigned long long context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static const GetCurrent cur = []() -> GetCurrent {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<GetCurrent>(p);
    return nullptr;
  }();
  static const GetId id = []() -> GetId {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<GetId>(p);
    return nullptr;
  }();
  CUcontext c = nullptr;
  unsigned long long v = 0;
  if (!cur || !id || cur(&c) != CUDA_SUCCESS || !c || id(c, &v) != CUDA_SUCCESS) return 0;
  return v;
}

EncodeTiled tensor_map_encoder() {
  // looked up once (a function-local static is initialized exactly once,
  // also when several threads arrive together)
  static const EncodeTiled fn = []() -> EncodeTiled {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiled>(p);
    return nullptr;
  }();
  return fn;
}

}  // namespace gq

extern "C" {

GQ_API int gq_abi_version(void) { return GQ_ABI_VERSION; }

GQ_API const char* gq_status_string(int status) {
  switch (status) {
    case GQ_OK: return "ok";
    case GQ_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative size or bad enum)";
    case GQ_ERR_SHAPE: return "shape error (size not a whole number of blocks, or batch out of range)";
    case GQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case GQ_ERR_DTYPE: return "unsupported element type";
    case GQ_ERR_NONFINITE: return "NaN or infinity in quantizer input";
    case GQ_ERR_RANGE: return "scale overflowed FP16";
    case GQ_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
    case GQ_ERR_CUDA: return "CUDA launch or runtime error";
    case GQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

GQ_API gq_status gq_status_from_dev(int f) {
  if (f & GQ_DEV_TIMEOUT) return GQ_ERR_TIMEOUT;
  if (f & GQ_DEV_NONFINITE) return GQ_ERR_NONFINITE;
  if (f & GQ_DEV_RANGE) return GQ_ERR_RANGE;
  return GQ_OK;
}

// Q4_0 chapter 4.1.2: 2 + 16 bytes per 32 weights.
GQ_API size_t gq_q4_0_bytes(int64_t n) {
  if (n < 0 || n % 32) return 0;
  return static_cast<size_t>(n / 32) * 18u;
}

// K-quants bits table: 16 + 8 x 8 bits of scales and 128 bytes of codes per 256 weights.
GQ_API size_t gq_ksb_bytes(int64_t n) {
  if (n < 0 || n % 256) return 0;
  return static_cast<size_t>(n / 256) * 138u;
}

}  // extern "C"
