// Per-device caches for host-side set-up that the CUDA runtime keeps per
// device context: kernel attributes (cudaFuncSetAttribute), queried device
// properties, device addresses of library symbols.  Plain C++ (no CUDA
// headers), so the host tests compile and check it with a C++ compiler.
//
// A value set while device 0 was current says nothing about device 1: every
// entry is keyed by the device index.  Entries are atomics, so host threads
// that make their first calls at the same time do not race; at worst both run
// the set-up, which is idempotent for every use in this library.
#pragma once

#include <atomic>

namespace mbok {

constexpr int kMaxDevices = 64;

// One flag per device index: "the set-up for this device has succeeded".
struct PerDeviceOnce {
  std::atomic<bool> done[kMaxDevices];
  PerDeviceOnce() {
    for (int i = 0; i < kMaxDevices; ++i) done[i].store(false, std::memory_order_relaxed);
  }
};

// Runs setup() unless it has already succeeded for device `dev`.  setup()
// returns 0 on success, else an error code that is passed back (and the next
// call tries again).  Devices outside [0, kMaxDevices) are set up every time.
template <class Setup>
int run_once_for_device(PerDeviceOnce& once, int dev, Setup setup) {
  if (dev < 0 || dev >= kMaxDevices) return setup();
  if (once.done[dev].load(std::memory_order_acquire)) return 0;
  const int e = setup();
  if (e == 0) once.done[dev].store(true, std::memory_order_release);
  return e;
}

// One cached value per device index (0 / nullptr = not yet known).
template <class T>
struct PerDeviceValue {
  std::atomic<T> value[kMaxDevices];
  PerDeviceValue() {
    for (int i = 0; i < kMaxDevices; ++i) value[i].store(T(), std::memory_order_relaxed);
  }
  // The cached value for `dev`, or compute() stored for it when none is
  // cached yet; compute() returns T() on failure, which is not cached.
  template <class Compute>
  T get(int dev, Compute compute) {
    if (dev < 0 || dev >= kMaxDevices) return compute();
    T v = value[dev].load(std::memory_order_acquire);
    if (v != T()) return v;
    v = compute();
    if (v != T()) value[dev].store(v, std::memory_order_release);
    return v;
  }
};

}  // namespace mbok
