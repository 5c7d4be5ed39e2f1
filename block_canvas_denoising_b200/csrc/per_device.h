// per_device.h -- a value computed once per CUDA device and kept for the
// life of the process (host code only, no CUDA calls of its own).
//
// The head kernel's launch set-up -- raising its dynamic shared-memory limit
// and asking how many CTA pairs fit at once -- is state of the device current
// when it is done, not of the process.  A process that drives several GPUs
// (one after another, or from several threads) must therefore do it once for
// each device it launches on; PerDevice<T> keeps one slot per device ordinal
// and runs the set-up for a device the first time that device asks for it.
// A set-up that fails is not remembered, so a later call retries it.
#pragma once

#include <mutex>

namespace dg {

template <typename T, int kMaxDevices = 64>
class PerDevice {
 public:
  // The value for device `dev`: make(&value) runs, under the lock, only the
  // first time `dev` asks (and again after a failed attempt).  Returns false
  // for an out-of-range ordinal or when make() returns false.
  template <typename Make>
  bool get(int dev, Make&& make, T* out) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(mu_);
    if (!ready_[dev]) {
      T v{};
      if (!make(&v)) return false;
      val_[dev] = v;
      ready_[dev] = true;
    }
    *out = val_[dev];
    return true;
  }

 private:
  std::mutex mu_;
  T val_[kMaxDevices] = {};
  bool ready_[kMaxDevices] = {};
};

}  // namespace dg
