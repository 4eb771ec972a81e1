// Host-side checks of the per-device launch setup helpers (device_once.h):
// setup runs once per device ordinal, failures are returned and retried,
// ordinals beyond the remembered range set up on every call, and concurrent
// first calls leave every device set up.
#include "device_once.h"

#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#define CHECK(c)                                         \
  do {                                                   \
    if (!(c)) {                                          \
      std::printf("FAIL line %d: %s\n", __LINE__, #c);   \
      return 1;                                          \
    }                                                    \
  } while (0)

int main() {
  using qnf4::DeviceOnce;
  using qnf4::DeviceValue;
  {
    DeviceOnce once;
    int calls = 0;
    auto ok = [&] {
      ++calls;
      return 0;
    };
    CHECK(once.run(0, ok) == 0 && calls == 1);
    CHECK(once.run(0, ok) == 0 && calls == 1);  // remembered for device 0
    CHECK(once.run(1, ok) == 0 && calls == 2);  // device 1 is set up on its own
    CHECK(once.run(63, ok) == 0 && calls == 3);
    CHECK(once.run(63, ok) == 0 && calls == 3);
    CHECK(once.run(64, ok) == 0 && calls == 4);  // beyond the slots: every call
    CHECK(once.run(64, ok) == 0 && calls == 5);
    CHECK(once.run(-1, ok) == 0 && calls == 6);
    CHECK(once.run(1, ok) == 0 && calls == 6);
  }
  {
    DeviceOnce once;
    int calls = 0, failures_left = 2;
    auto flaky = [&] {
      ++calls;
      return failures_left-- > 0 ? 7 : 0;
    };
    CHECK(once.run(3, flaky) == 7);  // a failure is returned ...
    CHECK(once.run(3, flaky) == 7);  // ... and the setup tried again
    CHECK(once.run(3, flaky) == 0 && calls == 3);
    CHECK(once.run(3, flaky) == 0 && calls == 3);
    CHECK(once.run(4, flaky) == 0 && calls == 4);
  }
  {
    DeviceValue val;
    int calls = 0;
    CHECK(val.get(0, [&] { return ++calls, 148; }) == 148);
    CHECK(val.get(0, [&] { return ++calls, 5; }) == 148 && calls == 1);
    CHECK(val.get(2, [&] { return ++calls, 0; }) == 0 && calls == 2);  // 0 is a value
    CHECK(val.get(2, [&] { return ++calls, 9; }) == 0 && calls == 2);
    CHECK(val.get(5, [&] { return ++calls, -1; }) == -1);  // a failure is not remembered
    CHECK(val.get(5, [&] { return ++calls, 74; }) == 74 && calls == 4);
    CHECK(val.get(5, [&] { return ++calls, 1; }) == 74 && calls == 4);
    CHECK(val.get(99, [&] { return ++calls, 1; }) == 1 && calls == 5);  // not remembered
    CHECK(val.get(99, [&] { return ++calls, 2; }) == 2 && calls == 6);
  }
  {
    // Eight threads race through the first calls of eight devices: each
    // device is set up at least once and at most once per thread.
    DeviceOnce once;
    std::atomic<int> calls[8];
    for (auto& c : calls) c.store(0);
    std::vector<std::thread> threads;
    for (int t = 0; t < 8; ++t)
      threads.emplace_back([&] {
        for (int i = 0; i < 1000; ++i) {
          const int d = i % 8;
          once.run(d, [&] {
            calls[d].fetch_add(1);
            return 0;
          });
        }
      });
    for (auto& t : threads) t.join();
    for (int d = 0; d < 8; ++d) CHECK(calls[d].load() >= 1 && calls[d].load() <= 8);
  }
  std::printf("ok\n");
  return 0;
}
