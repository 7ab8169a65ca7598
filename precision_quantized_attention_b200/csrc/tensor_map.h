// tensor_map.h -- the driver's cuTensorMapEncodeTiled, looked up once per process through the
// runtime (no link against libcuda), for the TMA descriptors of the attention and GEMM kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

namespace qattn {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// nullptr when the driver does not provide it (the callers then fail the launch).
inline EncodeTiledFn encode_tiled_fn() {
  static const EncodeTiledFn fn = [] {          // initialised once, thread-safe
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace qattn
