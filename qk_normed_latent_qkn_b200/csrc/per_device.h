// One-time host-side set-up that belongs to one device: a kernel's launch
// attributes (maximum dynamic shared memory, carveout) are recorded per device
// by the runtime, so a process that drives several GPUs must set them once on
// each.  PerDeviceOnce keeps a bitmask of the devices on which the set-up
// succeeded.  The mask is read without a lock on the fast path and written
// under a mutex, so concurrent first calls from several threads run the set-up
// once per device, and a set-up that fails is tried again on the next call.
// Host-only C++ (no CUDA types), so that the bookkeeping can be tested on a
// machine without a GPU.
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>

namespace qkn {

class PerDeviceOnce {
 public:
  static constexpr int kTracked = 64;

  // Run setup() on device `dev` unless it already succeeded there.  `ok` is the
  // success value of setup's result type; it is also what a skipped call
  // returns.  Devices outside [0, kTracked) are not tracked: setup runs on
  // every call for them.
  template <typename R, typename F>
  R run(int dev, R ok, F&& setup) {
    if (dev < 0 || dev >= kTracked) return setup();
    const uint64_t bit = uint64_t{1} << dev;
    if (done_.load(std::memory_order_acquire) & bit) return ok;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_.load(std::memory_order_relaxed) & bit) return ok;
    R r = setup();
    if (r == ok) done_.fetch_or(bit, std::memory_order_release);
    return r;
  }

  bool done(int dev) const {
    return dev >= 0 && dev < kTracked && (done_.load(std::memory_order_acquire) >> dev) & 1u;
  }

 private:
  std::atomic<uint64_t> done_{0};
  std::mutex mu_;
};

}  // namespace qkn
