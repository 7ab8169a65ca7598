// device_once.h -- per-device values the host launchers compute once (occupancy, the
// dynamic-shared-memory attribute of a kernel): thread-safe on first use (std::call_once per
// device), so host threads making their first calls at the same moment on the same or on
// different devices neither race nor read a half-written value.  Internal to the library.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace qattn {

constexpr int kMaxCachedDevices = 64;

class DeviceOnce {
 public:
  // The value `init()` returned on the first call made with the current device; later calls
  // on that device return it without calling init again.  Devices beyond the cache are not
  // cached (init runs every time).
  template <class F>
  int get(F&& init) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxCachedDevices) return init();
    std::call_once(flag_[dev], [&] { val_[dev] = init(); });
    return val_[dev];
  }

 private:
  std::once_flag flag_[kMaxCachedDevices];
  int val_[kMaxCachedDevices] = {};
};

}  // namespace qattn
