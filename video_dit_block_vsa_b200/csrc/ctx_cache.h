// Per-context cache of values that belong to a CUDA context: the device
// address of a file-scope __device__ variable, a kernel attribute that was
// raised, a stream the library created.  Such a value is only valid in the
// context it was made in.  A caller may make a context of its own current
// (a plugin inside an application that manages contexts with the driver API)
// or destroy the primary context (cudaDeviceReset) and get a new one, so the
// cache key is the context's unique id (cuCtxGetId), which the driver never
// hands out twice in one process: an entry made in a context that no longer
// exists can never match a later one.
//
// Plain C++ (no CUDA types), so the host-side logic is testable without a GPU.
#pragma once

#include <cstdint>
#include <mutex>

namespace vsa {

template <typename T, int kEntries = 8>
class CtxCache {
 public:
  // Looks up the value of context `id` (non-zero).  On a miss, make(&value)
  // is called under the cache's lock; if it returns true the value is stored
  // (replacing the oldest entry when full) and returned.  Returns make's
  // verdict on a miss, true on a hit.
  template <typename Make>
  bool get(uint64_t id, Make make, T* out) {
    if (id == 0) return false;
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < kEntries; ++i) {
      if (ids_[i] == id) {
        *out = vals_[i];
        return true;
      }
    }
    T v{};
    if (!make(&v)) return false;
    ids_[next_] = id;
    vals_[next_] = v;
    next_ = (next_ + 1) % kEntries;
    *out = v;
    return true;
  }

  // Number of stored entries (tests).
  int size() {
    std::lock_guard<std::mutex> lock(mu_);
    int n = 0;
    for (int i = 0; i < kEntries; ++i) n += ids_[i] != 0;
    return n;
  }

 private:
  std::mutex mu_;
  uint64_t ids_[kEntries] = {};
  T vals_[kEntries] = {};
  int next_ = 0;
};

}  // namespace vsa
