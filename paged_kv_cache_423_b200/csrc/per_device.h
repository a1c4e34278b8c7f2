// Once-per-device set-up for kernel launchers.
//
// Kernel attributes set with cudaFuncSetAttribute (the dynamic shared-memory limit) and the
// occupancy derived from them belong to one device's context, so a process that launches on
// several GPUs has to set them up on each device the first time it launches there.  This is
// plain host C++ (no CUDA types), so the bookkeeping can be compiled and tested without a GPU.
#pragma once

#include <atomic>
#include <mutex>

namespace pkv {

constexpr int kMaxDevices = 64;

// Holds one Value per device.  get(device, setup, &value) runs setup(value) the first time it
// sees `device` and keeps the value if setup returns 0; later calls on that device return 0 and
// the kept value without running setup.  A setup that fails (non-zero status) is not kept and is
// run again on the next call.  A device index outside [0, kMaxDevices) returns `bad_device`.
// Safe to call from several threads; setup runs under a lock, at most once per device at a time.
template <class Value>
class PerDevice {
 public:
  template <class F>
  int get(int device, F&& setup, Value* out, int bad_device) {
    if (device < 0 || device >= kMaxDevices) return bad_device;
    if (!done_[device].load(std::memory_order_acquire)) {
      std::lock_guard<std::mutex> lock(mu_);
      if (!done_[device].load(std::memory_order_relaxed)) {
        Value v{};
        const int st = setup(v);
        if (st != 0) return st;
        value_[device] = v;
        done_[device].store(true, std::memory_order_release);
      }
    }
    if (out) *out = value_[device];
    return 0;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
  Value value_[kMaxDevices] = {};
};

}  // namespace pkv
