// Per-device memos for host code that may run on several devices and from
// several host threads at once: kernel attributes are set per device, and
// device properties differ per device.  Plain C++ (no CUDA), so the logic is
// tested on its own.
#pragma once

#include <atomic>

namespace i8lt {

constexpr int kMaxDevices = 64;

// A step that has to succeed once per device (setting a kernel attribute, say).
// run() calls it until it has succeeded on that device and then returns true
// without calling it; threads that race on the first calls may each run it, so
// the step must be idempotent.  Device ids outside [0, kMaxDevices) are not
// memoised: the step runs every time.
class PerDeviceOnce {
 public:
  template <class Step>
  bool run(int dev, Step&& step) {
    if (dev < 0 || dev >= kMaxDevices) return step();
    if (done_[dev].load(std::memory_order_acquire)) return true;
    const bool ok = step();
    if (ok) done_[dev].store(true, std::memory_order_release);
    return ok;
  }

 private:
  std::atomic<bool> done_[kMaxDevices]{};
};

// A non-zero int computed once per device (0 stands for "not known yet", so a
// computation that fails by returning 0 is tried again on the next call).
class PerDeviceInt {
 public:
  template <class Compute>
  int get(int dev, Compute&& compute) {
    if (dev < 0 || dev >= kMaxDevices) return compute();
    int v = slot_[dev].load(std::memory_order_acquire);
    if (v != 0) return v;
    v = compute();
    if (v != 0) slot_[dev].store(v, std::memory_order_release);
    return v;
  }

 private:
  std::atomic<int> slot_[kMaxDevices]{};
};

}  // namespace i8lt
