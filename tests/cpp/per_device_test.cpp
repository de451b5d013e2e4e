// Host-side test of the per-device memos (int8_mixed_precision_vectorwise_b200/csrc/per_device.h):
// several threads, several device ids, failing and succeeding steps.  Prints "ok" or
// the first failed check and exits non-zero.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "per_device.h"

static int fails = 0;
#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      std::printf("check failed, line %d: %s\n", __LINE__, #c); \
      ++fails;                                                \
    }                                                         \
  } while (0)

int main() {
  using i8lt::PerDeviceInt;
  using i8lt::PerDeviceOnce;
  {  // a step that succeeds runs until it succeeded on that device, then never again
    PerDeviceOnce once;
    std::atomic<int> calls[8] = {};
    std::vector<std::thread> ts;
    for (int t = 0; t < 16; ++t)
      ts.emplace_back([&, t] {
        for (int i = 0; i < 1000; ++i) {
          const int dev = (t + i) % 8;
          CHECK(once.run(dev, [&] { calls[dev]++; return true; }));
        }
      });
    for (auto& th : ts) th.join();
    for (int d = 0; d < 8; ++d) {
      CHECK(calls[d] >= 1 && calls[d] <= 16);   // at most the threads that raced on the first call
      const int before = calls[d];
      CHECK(once.run(d, [&] { calls[d]++; return true; }));
      CHECK(calls[d] == before);
    }
  }
  {  // a failing step is retried, and only on its own device
    PerDeviceOnce once;
    int a = 0, b = 0;
    CHECK(!once.run(2, [&] { ++a; return false; }));
    CHECK(once.run(3, [&] { ++b; return true; }));
    CHECK(!once.run(2, [&] { ++a; return false; }));
    CHECK(once.run(2, [&] { ++a; return true; }));
    CHECK(once.run(2, [&] { ++a; return true; }));
    CHECK(a == 3 && b == 1);
  }
  {  // device ids outside the table are never memoised
    PerDeviceOnce once;
    int n = 0;
    for (int i = 0; i < 3; ++i) once.run(-1, [&] { ++n; return true; });
    for (int i = 0; i < 3; ++i) once.run(i8lt::kMaxDevices, [&] { ++n; return true; });
    CHECK(n == 6);
  }
  {  // per-device values: computed once, kept apart per device, 0 means "try again"
    PerDeviceInt memo;
    std::atomic<int> computes[4] = {};
    std::vector<std::thread> ts;
    for (int t = 0; t < 8; ++t)
      ts.emplace_back([&] {
        for (int i = 0; i < 500; ++i) {
          const int dev = i % 4;
          const int v = memo.get(dev, [&] { computes[dev]++; return 100 + dev; });
          CHECK(v == 100 + dev);
        }
      });
    for (auto& th : ts) th.join();
    for (int d = 0; d < 4; ++d) CHECK(computes[d] >= 1 && computes[d] <= 8);
    int tries = 0;
    CHECK(memo.get(9, [&] { ++tries; return 0; }) == 0);
    CHECK(memo.get(9, [&] { ++tries; return 7; }) == 7);
    CHECK(memo.get(9, [&] { ++tries; return 8; }) == 7);
    CHECK(tries == 2);
    CHECK(memo.get(-5, [] { return 3; }) == 3 && memo.get(-5, [] { return 4; }) == 4);
  }
  std::printf(fails ? "FAILED\n" : "ok\n");
  return fails ? 1 : 0;
}
