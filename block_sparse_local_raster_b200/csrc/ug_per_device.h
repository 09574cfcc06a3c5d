// Per-device set-up done once: a kernel's shared-memory opt-in and a static
// symbol's device address are properties of one device (one context), so a
// process that drives several devices needs them once per device, and host
// threads may race to do them.  PerDevice<T> keeps one slot per device
// ordinal: the first caller for a device runs the set-up under the table's
// mutex and stores its result; later callers read the slot.  A failed set-up
// leaves the slot empty, so the next call tries again.
//
// Plain C++ (no CUDA types), so that the bookkeeping itself is testable on a
// machine without a GPU.
#pragma once

#include <atomic>
#include <mutex>

#include "ug.h"

namespace ug {

constexpr int kMaxDevices = 64;

template <class T>
class PerDevice {
 public:
  PerDevice() {
    for (auto& r : ready_) r.store(false, std::memory_order_relaxed);
  }

  // Runs setup(T&) -> status once for `device` (0 <= device < kMaxDevices)
  // and returns its status; on UG_OK, *out (if not null) receives the value
  // stored for that device.
  template <class F>
  int get(int device, F&& setup, T* out = nullptr) {
    if (device < 0 || device >= kMaxDevices) return UG_ERR_UNSUPPORTED;
    if (!ready_[device].load(std::memory_order_acquire)) {
      std::lock_guard<std::mutex> lock(mu_);
      if (!ready_[device].load(std::memory_order_relaxed)) {
        T v{};
        const int st = setup(v);
        if (st != UG_OK) return st;
        value_[device] = v;
        ready_[device].store(true, std::memory_order_release);
      }
    }
    if (out) *out = value_[device];
    return UG_OK;
  }

  bool ready(int device) const {
    return device >= 0 && device < kMaxDevices && ready_[device].load(std::memory_order_acquire);
  }

 private:
  std::mutex mu_;
  std::atomic<bool> ready_[kMaxDevices];
  T value_[kMaxDevices] = {};
};

}  // namespace ug
