// Host-only checks of ug::PerDevice, the once-per-device set-up table that
// the library uses for kernel attributes and the static scratch's address.
// Built and run by tests/test_per_device_host.py; prints "ok" on success.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "ug_per_device.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);           \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main() {
  ug::PerDevice<long> table;
  std::atomic<int> runs[ug::kMaxDevices];
  for (auto& r : runs) r = 0;

  // 16 threads race on devices 0..3: each device's set-up runs exactly once,
  // and every caller sees that device's value.
  std::vector<std::thread> th;
  std::atomic<int> bad{0};
  for (int t = 0; t < 16; ++t)
    th.emplace_back([&, t] {
      for (int rep = 0; rep < 200; ++rep) {
        const int dev = (t + rep) % 4;
        long v = -1;
        const int st = table.get(dev, [&](long& out) {
          runs[dev]++;
          std::this_thread::yield();
          out = 1000 + dev;
          return (int)UG_OK;
        }, &v);
        if (st != UG_OK || v != 1000 + dev) bad++;
      }
    });
  for (auto& x : th) x.join();
  CHECK(bad == 0);
  for (int d = 0; d < 4; ++d) CHECK(runs[d] == 1);
  for (int d = 4; d < ug::kMaxDevices; ++d) CHECK(runs[d] == 0 && !table.ready(d));

  // A failed set-up is not cached: the next call runs it again.
  int tries = 0;
  auto flaky = [&](long& out) {
    ++tries;
    out = 7;
    return tries == 1 ? (int)UG_ERR_CUDA : (int)UG_OK;
  };
  long v = 0;
  CHECK(table.get(9, flaky, &v) == UG_ERR_CUDA);
  CHECK(!table.ready(9));
  CHECK(table.get(9, flaky, &v) == UG_OK && v == 7 && tries == 2);
  CHECK(table.get(9, flaky, &v) == UG_OK && tries == 2 && table.ready(9));

  // Device ordinals outside the table are refused without running set-up.
  int called = 0;
  auto count = [&](long&) { ++called; return (int)UG_OK; };
  CHECK(table.get(-1, count) == UG_ERR_UNSUPPORTED);
  CHECK(table.get(ug::kMaxDevices, count) == UG_ERR_UNSUPPORTED);
  CHECK(called == 0);
  std::printf("ok\n");
  return 0;
}
