// Host-side caches of launch plans (per-device kernel attributes, launch
// shapes and encoded TMA descriptors), safe to use from any number of host
// threads.  Each cache is a small mutex-guarded table: a lookup copies the
// whole entry out under the lock, so a caller never sees a key from one
// insertion paired with a value from another.  Values are computed outside
// the lock (two threads missing on the same key both compute it; the values
// are equal, and the second insertion overwrites the first).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <stdint.h>
#include <string.h>

namespace w4a4 {

template <class Key, class Val, int kSlots>
class PlanCache {
 public:
  // Copy the value stored under `key` into `out`; false when absent.
  bool find(const Key& key, Val& out) {
    std::lock_guard<std::mutex> g(mu_);
    for (int i = 0; i < used_; ++i) {
      if (memcmp(&slots_[i].key, &key, sizeof(Key)) == 0) {
        out = slots_[i].val;
        slots_[i].stamp = ++clock_;
        return true;
      }
    }
    return false;
  }

  // Store (key, val), replacing the least recently used entry when full.
  void insert(const Key& key, const Val& val) {
    std::lock_guard<std::mutex> g(mu_);
    int victim = -1;
    for (int i = 0; i < used_; ++i)
      if (memcmp(&slots_[i].key, &key, sizeof(Key)) == 0) victim = i;
    if (victim < 0) {
      if (used_ < kSlots) {
        victim = used_++;
      } else {
        victim = 0;
        for (int i = 1; i < kSlots; ++i)
          if (slots_[i].stamp < slots_[victim].stamp) victim = i;
      }
    }
    slots_[victim].key = key;
    slots_[victim].val = val;
    slots_[victim].stamp = ++clock_;
  }

  // find(), else make(val) outside the lock and insert.  Returns false when
  // make() fails (nothing is cached then).
  template <class F>
  bool get(const Key& key, Val& out, F&& make) {
    if (find(key, out)) return true;
    Val v;
    if (!make(v)) return false;
    insert(key, v);
    out = v;
    return true;
  }

 private:
  struct Slot {
    Key key;
    Val val;
    uint64_t stamp;
  };
  std::mutex mu_;
  Slot slots_[kSlots];
  int used_ = 0;
  uint64_t clock_ = 0;
};

// One flag per device for one-time work such as cudaFuncSetAttribute: set
// only after the work succeeded, so a failure is retried by the next call
// (repeating the attribute call from two threads at once is harmless).
struct DeviceFlags {
  std::atomic<int> f[64];
  bool done(int dev) const { return dev >= 0 && dev < 64 && f[dev].load(std::memory_order_acquire) != 0; }
  void set(int dev) {
    if (dev >= 0 && dev < 64) f[dev].store(1, std::memory_order_release);
  }
};

// Unique id of the calling thread's current CUDA context (0 when there is
// none or the driver cannot say).  Device addresses of module globals are
// cached per context id, so a context recreated after cudaDeviceReset gets
// its own lookup instead of a stale address.
unsigned long long current_context_id();

// Device address of a module global (__device__ variable) in the current
// context, looked up once per context.
cudaError_t symbol_address_cached(const void* symbol, void** out);

// Number of SMs of a device, looked up once per device.
inline cudaError_t device_sm_count(int dev, int* out) {
  static std::atomic<int> cached[64];
  if (dev >= 0 && dev < 64) {
    const int n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) {
      *out = n;
      return cudaSuccess;
    }
  }
  int n = 0;
  const cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  *out = n;
  return cudaSuccess;
}

}  // namespace w4a4
