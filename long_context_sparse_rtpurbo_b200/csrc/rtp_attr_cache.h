// Host-side cache of a kernel attribute that must be set per device: the largest dynamic
// shared-memory size set so far for each (kernel instance, device), under a lock. The setter
// runs only when the (instance, device) entry is below the requested size, so a second device
// (or a larger layer) sets its own attribute while repeated calls cost one locked compare.
// Host-only C++ (no CUDA types), so it is unit-tested on the CPU with a fake setter.
#pragma once

#include <mutex>

namespace rtp {

template <int kInstances, int kDevices>
class AttrCache {
 public:
  // set(dev, bytes) -> 0 on success; returns set's status, 0 when nothing had to be set, or
  // -1 for an instance or device index out of range.
  template <class Setter>
  int ensure(int inst, int dev, int bytes, Setter&& set) {
    if (inst < 0 || inst >= kInstances || dev < 0 || dev >= kDevices) return -1;
    std::lock_guard<std::mutex> lock(mu_);
    if (have_[inst][dev] >= bytes) return 0;
    const int rc = set(dev, bytes);
    if (rc == 0) have_[inst][dev] = bytes;
    return rc;
  }

 private:
  std::mutex mu_;
  int have_[kInstances][kDevices] = {};   // 0: never set on that device
};

}  // namespace rtp
