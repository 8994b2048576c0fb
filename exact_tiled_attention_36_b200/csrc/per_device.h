// per_device.h: values the library computes once per GPU and then reuses.
//
// State that belongs to one device (the address of a __device__ variable, a
// kernel's shared-memory attribute, its register count, the SM count) must be
// looked up with that device current and kept apart from the other devices'
// copies, or a process that drives several GPUs would hand one GPU's address
// to another GPU's kernels. PerDevice<T> keeps one slot per device index: the
// first get() for a device runs `make` under a lock and stores the result if
// `make` succeeded; later calls read the slot without locking. A failed
// `make` stores nothing, so the next call tries again.
//
// Plain C++ (no CUDA types): the caller passes the device index, which lets
// the cache be tested on a host without a GPU.
#pragma once

#include <atomic>
#include <mutex>

namespace fa {

constexpr int kMaxDevices = 64;

template <typename T>
class PerDevice {
  public:
    // The value of device `dev`, made by `make(T&) -> bool` on first use.
    // Returns false for a device index outside [0, kMaxDevices) or when `make`
    // fails (then *out is left unchanged).
    template <typename Make>
    bool get(int dev, Make&& make, T* out) {
        if (dev < 0 || dev >= kMaxDevices) return false;
        if (!ready_[dev].load(std::memory_order_acquire)) {
            std::lock_guard<std::mutex> lock(mu_);
            if (!ready_[dev].load(std::memory_order_relaxed)) {
                T v{};
                if (!make(v)) return false;
                vals_[dev] = v;
                ready_[dev].store(true, std::memory_order_release);
            }
        }
        *out = vals_[dev];
        return true;
    }

  private:
    std::mutex mu_;
    std::atomic<bool> ready_[kMaxDevices] = {};
    T vals_[kMaxDevices] = {};
};

}  // namespace fa
