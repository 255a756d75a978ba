// Per-device launch facts of the library's kernels, for a process that drives several GPUs
// from any number of host threads.  Kernel attributes (the dynamic shared-memory limit) and
// occupancy belong to one device's context, so every fact is kept per device index; the
// caches are safe for concurrent host threads.  Nothing here calls CUDA: the callers pass
// the current device and a callable that performs the CUDA step, which also lets a plain
// C++ test drive the keying.
#pragma once

#include <atomic>
#include <mutex>

namespace rmsk {

constexpr int kMaxDevices = 64;

// The dynamic shared-memory bytes a kernel may use, granted per device.  grant(dev, bytes,
// set) calls set(bytes) -- which must raise the kernel's limit on device `dev`, the current
// one -- unless that device already granted at least `bytes`.  A device's grant only grows,
// and set() runs under a lock, so a smaller grant never overwrites a larger one that another
// thread made.  Returns set()'s code, or 0 when nothing had to be set.  Devices outside
// [0, kMaxDevices) are not cached: set() runs every time.
class SmemGrant {
  public:
    template <typename Set>
    int grant(int dev, int bytes, Set set) {
        if (dev < 0 || dev >= kMaxDevices) return set(bytes);
        if (granted_[dev].load(std::memory_order_acquire) >= bytes) return 0;
        std::lock_guard<std::mutex> lock(mu_);
        if (granted_[dev].load(std::memory_order_relaxed) >= bytes) return 0;
        const int rc = set(bytes);
        if (rc == 0) granted_[dev].store(bytes, std::memory_order_release);
        return rc;
    }
    int granted(int dev) const {
        return dev >= 0 && dev < kMaxDevices ? granted_[dev].load(std::memory_order_acquire) : 0;
    }

  private:
    std::atomic<int> granted_[kMaxDevices] = {};
    std::mutex mu_;
};

// A positive value computed once per device and key in [0, N) (e.g. resident CTAs per SM of
// one kernel at one block size).  compute() may run more than once when threads race; every
// run gives the same value, and a stored value is never torn.  A non-positive result is
// returned but not stored.  Devices or keys out of range are not cached.
template <int N = 1>
class PerDevice {
  public:
    template <typename F>
    int get(int dev, int key, F compute) {
        if (dev < 0 || dev >= kMaxDevices || key < 0 || key >= N) return compute();
        int v = v_[dev][key].load(std::memory_order_acquire);
        if (v > 0) return v;
        v = compute();
        if (v > 0) v_[dev][key].store(v, std::memory_order_release);
        return v;
    }

  private:
    std::atomic<int> v_[kMaxDevices][N] = {};
};

}  // namespace rmsk
