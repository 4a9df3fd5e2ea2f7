// kda_once.h -- per-device one-time setup for the kernel launchers, safe when several host
// threads launch at once, on one device or on several.
//
// A launcher raises its kernels' dynamic shared-memory limit (cudaFuncSetAttribute) once per
// device and may cache a device property next to it (the SM count).  Plain statics for this
// race between threads and go stale when a thread switches devices; this keeps one record per
// device ordinal under a mutex.
#pragma once

#include <mutex>

namespace kda {

constexpr int kMaxDevices = 64;

struct PerDevice {
  std::mutex mu;
  bool ready[kMaxDevices] = {};
  int value[kMaxDevices] = {};
};

// The first call for device `dev` runs setup(dev, &v) under the lock and, if it succeeds (the
// error type's zero value), records v; later calls return the recorded v.  A failed setup is not
// recorded, so the next call runs it again.  Ordinals outside [0, kMaxDevices) run setup on every
// call.  Returns setup's error, or zero.
template <class Setup>
auto once_per_device(PerDevice& st, int dev, int* value, Setup&& setup)
    -> decltype(setup(dev, value)) {
  using Err = decltype(setup(dev, value));
  const bool cached = dev >= 0 && dev < kMaxDevices;
  std::lock_guard<std::mutex> lock(st.mu);
  if (cached && st.ready[dev]) {
    *value = st.value[dev];
    return Err{};
  }
  int v = 0;
  const Err e = setup(dev, &v);
  if (e != Err{}) return e;
  if (cached) {
    st.value[dev] = v;
    st.ready[dev] = true;
  }
  *value = v;
  return e;
}

}  // namespace kda
