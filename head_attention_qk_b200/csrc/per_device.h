// per_device.h -- one-time setup per CUDA device ordinal (plain C++, no CUDA).
//
// Kernel attributes set with cudaFuncSetAttribute (the dynamic shared-memory
// limit) and the checks made with cudaFuncGetAttributes belong to one device:
// a process that drives several GPUs must make them on each device before its
// first launch there.  PerDeviceOnce runs a setup function the first time a
// device ordinal asks and remembers success for the rest of the process; a
// failed setup is not remembered, so the next call on that device tries again.
// Concurrent first calls (several host threads) run the setup once.
#pragma once

#include <atomic>
#include <mutex>

namespace hattn {

class PerDeviceOnce {
 public:
  static constexpr int kMaxDevices = 64;

  // True if `setup` has succeeded for `device` (running it now if it has not
  // run yet, or failed before); false for an ordinal outside [0, kMaxDevices)
  // or a failed setup.
  template <class F>
  bool ensure(int device, F&& setup) {
    if (device < 0 || device >= kMaxDevices) return false;
    if (done_[device].load(std::memory_order_acquire)) return true;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[device].load(std::memory_order_relaxed)) return true;
    if (!setup()) return false;
    done_[device].store(true, std::memory_order_release);
    return true;
  }

 private:
  std::atomic<bool> done_[kMaxDevices] = {};
  std::mutex mu_;
};

}  // namespace hattn
