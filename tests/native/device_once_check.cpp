// Host check of the per-device set-up caches (device_once.h): a kernel
// attribute or cached value recorded for one device index must not be taken
// as set for another, a failed set-up must be retried, and device indices
// outside the table are set up on every call.  Exits 0 when every check holds.
#include <cstdio>
#include <thread>
#include <vector>

#include "device_once.h"

static int failures = 0;
#define CHECK(c)                                               \
  do {                                                         \
    if (!(c)) {                                                \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);       \
      ++failures;                                              \
    }                                                          \
  } while (0)

int main() {
  using namespace mbok;
  {
    PerDeviceOnce once;
    int calls = 0;
    auto ok = [&]() { ++calls; return 0; };
    CHECK(run_once_for_device(once, 0, ok) == 0 && calls == 1);
    CHECK(run_once_for_device(once, 0, ok) == 0 && calls == 1);   // cached for device 0
    CHECK(run_once_for_device(once, 1, ok) == 0 && calls == 2);   // device 1 is set up on its own
    CHECK(run_once_for_device(once, 1, ok) == 0 && calls == 2);
    CHECK(run_once_for_device(once, 63, ok) == 0 && calls == 3);
    CHECK(run_once_for_device(once, 64, ok) == 0 && calls == 4);  // outside the table: every time
    CHECK(run_once_for_device(once, 64, ok) == 0 && calls == 5);
    CHECK(run_once_for_device(once, -1, ok) == 0 && calls == 6);
  }
  {
    PerDeviceOnce once;
    int calls = 0;
    auto fail = [&]() { ++calls; return 7; };
    auto ok = [&]() { ++calls; return 0; };
    CHECK(run_once_for_device(once, 2, fail) == 7 && calls == 1);
    CHECK(run_once_for_device(once, 2, ok) == 0 && calls == 2);   // a failure is not cached
    CHECK(run_once_for_device(once, 2, ok) == 0 && calls == 2);
  }
  {
    PerDeviceValue<int> v;
    int calls = 0;
    CHECK(v.get(0, [&]() { ++calls; return 148; }) == 148 && calls == 1);
    CHECK(v.get(0, [&]() { ++calls; return 132; }) == 148 && calls == 1);
    CHECK(v.get(1, [&]() { ++calls; return 132; }) == 132 && calls == 2);
    CHECK(v.get(3, [&]() { ++calls; return 0; }) == 0 && calls == 3);   // failure not cached
    CHECK(v.get(3, [&]() { ++calls; return 5; }) == 5 && calls == 4);
  }
  {
    // Several host threads making their first call on several devices at once.
    PerDeviceValue<void*> v;
    static int cells[8];
    std::vector<std::thread> th;
    std::vector<void*> got(32, nullptr);
    for (int t = 0; t < 32; ++t)
      th.emplace_back([&, t]() { got[t] = v.get(t % 8, [t]() -> void* { return &cells[t % 8]; }); });
    for (auto& x : th) x.join();
    for (int t = 0; t < 32; ++t) CHECK(got[t] == &cells[t % 8]);
  }
  if (failures == 0) std::printf("device_once: all checks passed\n");
  return failures == 0 ? 0 : 1;
}
