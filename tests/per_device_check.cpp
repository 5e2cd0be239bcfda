// Host-only check of PerDeviceOnce (the per-device bookkeeping behind the
// kernels' one-time launch attributes): compiled with g++ and run by
// tests/test_per_device.py.  Prints "ok" and exits 0 when every check holds.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "per_device.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      std::printf("failed: %s (line %d)\n", #c, __LINE__);        \
      return 1;                                                   \
    }                                                             \
  } while (0)

int main() {
  using qkn::PerDeviceOnce;
  {  // once per device, not once per process
    PerDeviceOnce once;
    int calls[4] = {0, 0, 0, 0};
    for (int rep = 0; rep < 3; ++rep)
      for (int dev = 0; dev < 4; ++dev) CHECK(once.run(dev, 0, [&] { ++calls[dev]; return 0; }) == 0);
    for (int dev = 0; dev < 4; ++dev) CHECK(calls[dev] == 1 && once.done(dev));
    CHECK(!once.done(4));
  }
  {  // a failed set-up is not recorded and runs again
    PerDeviceOnce once;
    int calls = 0;
    CHECK(once.run(2, 0, [&] { ++calls; return 7; }) == 7);
    CHECK(!once.done(2));
    CHECK(once.run(2, 0, [&] { ++calls; return 0; }) == 0);
    CHECK(once.run(2, 0, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 2 && once.done(2));
  }
  {  // devices outside the tracked range run the set-up every time
    PerDeviceOnce once;
    int calls = 0;
    for (int rep = 0; rep < 3; ++rep) CHECK(once.run(64, 0, [&] { ++calls; return 0; }) == 0);
    CHECK(once.run(-1, 0, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 4 && !once.done(64));
    CHECK(once.run(63, 0, [&] { ++calls; return 0; }) == 0 && once.done(63));
  }
  {  // concurrent first calls from many threads run it once per device
    PerDeviceOnce once;
    std::atomic<int> calls[8];
    for (auto& c : calls) c = 0;
    std::vector<std::thread> ts;
    for (int t = 0; t < 16; ++t)
      ts.emplace_back([&, t] {
        for (int rep = 0; rep < 200; ++rep) {
          const int dev = (t + rep) % 8;
          once.run(dev, 0, [&] {
            calls[dev].fetch_add(1);
            std::this_thread::yield();
            return 0;
          });
        }
      });
    for (auto& th : ts) th.join();
    for (int dev = 0; dev < 8; ++dev) CHECK(calls[dev].load() == 1);
  }
  std::printf("ok\n");
  return 0;
}
