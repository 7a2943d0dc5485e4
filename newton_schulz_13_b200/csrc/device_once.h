// Per-device "done once" flags for settings that belong to one device's context, such as a
// kernel's dynamic shared-memory limit (cudaFuncSetAttribute applies to the current device only):
// a process that runs the library on several devices must apply them on each. Header-only and
// free of CUDA types, so that the bookkeeping can be unit-tested on a machine without a GPU.
#pragma once

#include <atomic>
#include <cstdint>

namespace muon {

class PerDeviceOnce {
 public:
  static constexpr int kTracked = 128;   // device indices [0, kTracked) are remembered

  // Runs fn() (returning 0 on success, anything else on failure) unless it has already succeeded
  // for device `dev`; returns fn's result, or 0 when it was skipped. A failure is not remembered,
  // so the next call retries. Devices outside the tracked range run fn() every time.
  template <class F>
  int run(int dev, F&& fn) {
    if (dev < 0 || dev >= kTracked) return fn();
    std::atomic<uint64_t>& word = done_[dev / 64];
    const uint64_t bit = uint64_t(1) << (dev % 64);
    if (word.load(std::memory_order_acquire) & bit) return 0;
    const int rc = fn();
    if (rc == 0) word.fetch_or(bit, std::memory_order_acq_rel);
    return rc;
  }

  bool done(int dev) const {
    if (dev < 0 || dev >= kTracked) return false;
    return (done_[dev / 64].load(std::memory_order_acquire) >> (dev % 64)) & 1u;
  }

 private:
  std::atomic<uint64_t> done_[kTracked / 64] = {};
};

}  // namespace muon
