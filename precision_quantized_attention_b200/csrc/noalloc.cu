// noalloc.cu -- qattn_calibrate_quantize_fp8_noalloc: the fused calibrate + FP8 quantize with its
// grid workspace in library-owned static device memory instead of a caller buffer.
//
// For callers that cannot hand the library a scratch buffer: C code with no device allocator at
// the call site, or a runtime whose device memory is planned ahead of time and that must not
// allocate on the hot path.  The call itself allocates nothing (no cudaMalloc/cudaFree, no
// allocating library call): the workspace is the file-scope array below, which the CUDA module
// loader places (zero-filled) in device memory of every device that loads the library.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "qattn.h"

namespace {

// Size of the static workspace: the fused kernel's workspace bound.  The kernel uses its first
// few words (an amax word and two grid counters) whatever n is, so no input size can need more.
constexpr size_t kNoallocScratchBytes = QATTN_FUSED_WORKSPACE_BYTES;
static_assert(kNoallocScratchBytes >= 16 && kNoallocScratchBytes % 16 == 0,
              "the fused calibrate+quantize workspace must fit the static scratch");
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct ScratchSlot {
  bool ready = false;
  void* ptr = nullptr;
};
ScratchSlot g_slot[kMaxDevices];
std::mutex g_slot_mutex;

// Set-up, once per device, with that device current: the device address of the array.
qattn_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_slot_mutex);
  ScratchSlot& s = g_slot[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return QATTN_ERR_CUDA;
    s.ptr = p;
    s.ready = true;
  }
  *out = s.ptr;
  return QATTN_OK;
}

}  // namespace

extern "C" QATTN_API qattn_status qattn_calibrate_quantize_fp8_noalloc(const void* x_bf16,
                                                                       size_t n, float* amax_dev,
                                                                       uint8_t* out_e4m3,
                                                                       float* scale_dev,
                                                                       qattn_stream_t stream) {
  // the argument checks of qattn_calibrate_quantize_fp8, before any device call
  if (!x_bf16 || !amax_dev || !out_e4m3 || !scale_dev || n == 0) return QATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x_bf16) % 16 || reinterpret_cast<uintptr_t>(out_e4m3) % 8 ||
      reinterpret_cast<uintptr_t>(amax_dev) % 4 || reinterpret_cast<uintptr_t>(scale_dev) % 4)
    return QATTN_ERR_INVALID_ARG;
  void* scratch = nullptr;
  qattn_status st = scratch_for_current_device(&scratch);
  if (st != QATTN_OK) return st;
  // The kernel expects a zero-filled workspace; clear it on the stream (no allocation), so a
  // previous call that gave up on a wait cannot leave stale counters behind.
  if (cudaMemsetAsync(scratch, 0, kNoallocScratchBytes, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return QATTN_ERR_CUDA;
  return qattn_calibrate_quantize_fp8(x_bf16, n, amax_dev, out_e4m3, scale_dev, scratch,
                                      kNoallocScratchBytes, stream);
}
