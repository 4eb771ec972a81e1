// Per-device one-time setup of a kernel launch site (host code only).
//
// A kernel's function attributes (the dynamic shared-memory limit above
// 48 KB) belong to one device's context, and so do the occupancy figures that
// depend on them: a process that launches a kernel on several devices must
// set them on each device.  Each launch site keeps one DeviceOnce (or one
// DeviceValue) as a function-local static and passes the current device.
//
// Ordinals 0..63 are remembered; for higher ordinals the setup runs on every
// call.  Threads that reach a device's first call together may each run the
// setup, so it must be idempotent (cudaFuncSetAttribute and the occupancy
// queries are).
#pragma once

#include <atomic>
#include <cstdint>

namespace qnf4 {

constexpr int kDeviceOnceSlots = 64;

// run(dev, setup): calls `setup` (which returns an error code, 0 = success)
// until it has succeeded once for device `dev`; afterwards returns 0 without
// calling it.  A failed setup is returned and tried again on the next call.
class DeviceOnce {
 public:
  template <typename Setup>
  auto run(int dev, Setup&& setup) -> decltype(setup()) {
    using Err = decltype(setup());
    const uint64_t bit = (dev >= 0 && dev < kDeviceOnceSlots) ? (uint64_t{1} << dev) : 0;
    if (bit != 0 && (done_.load(std::memory_order_acquire) & bit) != 0) return static_cast<Err>(0);
    const Err e = setup();
    if (e == static_cast<Err>(0) && bit != 0) done_.fetch_or(bit, std::memory_order_acq_rel);
    return e;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// get(dev, compute): an int computed once per device (how many CTAs or
// clusters fit at once, say).  A value >= 0 from `compute` is remembered for
// the device; a negative one reports a failure: it is returned, not
// remembered, and the next call computes again.
class DeviceValue {
 public:
  DeviceValue() {
    for (auto& s : slots_) s.store(-1, std::memory_order_relaxed);
  }

  template <typename Compute>
  int get(int dev, Compute&& compute) {
    if (dev < 0 || dev >= kDeviceOnceSlots) return compute();
    int v = slots_[dev].load(std::memory_order_acquire);
    if (v >= 0) return v;
    v = compute();
    if (v >= 0) slots_[dev].store(v, std::memory_order_release);
    return v;
  }

 private:
  std::atomic<int> slots_[kDeviceOnceSlots];
};

}  // namespace qnf4
