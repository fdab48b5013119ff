// Launch state that belongs to one device's context.
//
// The SM count and the dynamic shared-memory limit that cudaFuncSetAttribute raises for a kernel
// are properties of a device (the attribute is set in the current device's context).  A process
// that drives several devices, or several threads that call the library, must therefore keep them
// per device: this table holds, per device index, the SM count and, per kernel, the largest
// dynamic shared-memory size already allowed, all under one mutex.  The table is plain C++ (no
// CUDA types): the callers pass in the query and the setter, so the keying logic can be checked
// on a machine without a GPU.
#pragma once
#include <stddef.h>

#include <mutex>

#define DC_MAX_DEVICES 64

enum DcKernelId {
  DC_K_SEGMENTS = 0,
  DC_K_VSTAGE,
  DC_K_VPRE,
  DC_K_UDELTA,
  DC_K_UPRE,
  DC_K_BASE_TC,
  DC_K_BASE,
  DC_K_COUNT
};

class DcDevState {
 public:
  // SM count of device `dev`: `query(dev)` is called once per device and its value kept; a
  // value <= 0 (a failed query) is not kept and falls back to `fallback`.
  template <class Query>
  int sm_count(int dev, Query query, int fallback = 148) {
    if (dev < 0 || dev >= DC_MAX_DEVICES) return fallback;
    std::lock_guard<std::mutex> lock(mu_);
    if (n_sm_[dev] <= 0) {
      const int n = query(dev);
      if (n <= 0) return fallback;
      n_sm_[dev] = n;
    }
    return n_sm_[dev];
  }

  // Make sure kernel `kid` may use `need` bytes of dynamic shared memory on device `dev`:
  // `set(need)` (returns 0 on success, an error code otherwise) is called when `need` is above
  // what was already allowed there, and the new limit is kept only if it succeeded.  Returns 0 or
  // the setter's error code; -1 for a device or kernel index out of range.
  template <class Setter>
  int ensure_smem(int dev, int kid, size_t need, Setter set) {
    if (dev < 0 || dev >= DC_MAX_DEVICES || kid < 0 || kid >= DC_K_COUNT) return -1;
    std::lock_guard<std::mutex> lock(mu_);
    if (need <= smem_[dev][kid]) return 0;
    const int e = set(need);
    if (e == 0) smem_[dev][kid] = need;
    return e;
  }

  // The limit currently recorded for (dev, kid) (0 if none).
  size_t smem_limit(int dev, int kid) {
    if (dev < 0 || dev >= DC_MAX_DEVICES || kid < 0 || kid >= DC_K_COUNT) return 0;
    std::lock_guard<std::mutex> lock(mu_);
    return smem_[dev][kid];
  }

 private:
  std::mutex mu_;
  int n_sm_[DC_MAX_DEVICES] = {};
  size_t smem_[DC_MAX_DEVICES][DC_K_COUNT] = {};
};
