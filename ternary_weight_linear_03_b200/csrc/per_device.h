// Per-device, thread-safe one-time set-up values of the library's host code (a kernel's
// shared-memory limit applied with cudaFuncSetAttribute, its occupancy, the SM count).
// Such settings belong to one device's context, so each value is computed once per
// device ordinal; concurrent callers on any mix of devices see it computed exactly once.
// Plain C++ (no CUDA types), so the logic is testable on a machine without a GPU.
#pragma once

#include <atomic>
#include <mutex>

namespace bl {

constexpr int kMaxDevices = 64;

class PerDevice {
 public:
  // The cached value for `dev`, running init(dev) under the lock the first time. init
  // returns a positive value on success; zero or negative means failure, which is
  // returned but not cached (the next call tries again). Returns -1 for an ordinal
  // outside [0, kMaxDevices).
  template <class F>
  int get(int dev, F init) {
    if (dev < 0 || dev >= kMaxDevices) return -1;
    int v = val_[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    std::lock_guard<std::mutex> lock(mu_);
    v = val_[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    v = init(dev);
    if (v > 0) val_[dev].store(v, std::memory_order_release);
    return v;
  }

 private:
  std::mutex mu_;
  std::atomic<int> val_[kMaxDevices] = {};
};

}  // namespace bl
