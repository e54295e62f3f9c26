// device_once.h -- per-device, per-context one-time set-up for the host
// code of the library (kernel attributes, device constants, symbol
// addresses), safe under concurrent first calls from several host threads.
//
// A value cached for a device belongs to the CUDA context it was taken in:
// after cudaDeviceReset the primary context is a new one, with a fresh
// module (new symbol addresses, default kernel attributes).  So each cache
// entry stores the id of the context it was filled in (cuCtxGetId, reached
// through cudaGetDriverEntryPoint so that the library does not link
// libcuda) and is filled again when the current context's id differs.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

namespace moe {

constexpr int kMaxDevices = 64;

// Id of the calling thread's current context (never 0 once a context
// exists); 0 if it cannot be read, which only disables the reset check.
uint64_t current_context_id();

// SM count of the current device (cached per device and context; 148 if it
// cannot be read).
int num_sms();

// One cached value per device.  get() returns the value, running fill(&v)
// (a cudaError_t-returning callable) under a lock the first time for the
// current device and context; a failed fill is not cached.
template <typename T>
class DeviceOnce {
 public:
  template <typename F>
  cudaError_t get(int dev, T* out, F&& fill) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const uint64_t ctx = current_context_id();
    Slot& s = slots_[dev];
    if (s.ready.load(std::memory_order_acquire) &&
        s.ctx.load(std::memory_order_acquire) == ctx) {
      *out = s.value.load(std::memory_order_acquire);
      return cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(mu_);
    if (!(s.ready.load(std::memory_order_relaxed) &&
          s.ctx.load(std::memory_order_relaxed) == ctx)) {
      s.ready.store(false, std::memory_order_release);
      T v{};
      const cudaError_t e = fill(&v);
      if (e != cudaSuccess) return e;
      s.value.store(v, std::memory_order_release);
      s.ctx.store(ctx, std::memory_order_release);
      s.ready.store(true, std::memory_order_release);
    }
    *out = s.value.load(std::memory_order_acquire);
    return cudaSuccess;
  }

 private:
  struct Slot {
    std::atomic<bool> ready{false};
    std::atomic<uint64_t> ctx{0};
    std::atomic<T> value{};
  };
  Slot slots_[kMaxDevices];
  std::mutex mu_;
};

}  // namespace moe
