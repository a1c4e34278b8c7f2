// Host test of the once-per-device launcher set-up (paged_kv_cache_423_b200/csrc/per_device.h):
// compiled with g++ and run by tests/test_abi.py, no GPU involved.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "per_device.h"

static int failures = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      std::printf("FAILED line %d: %s\n", __LINE__, #cond);      \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main() {
  constexpr int kBad = -7;
  // Each device is set up on its first use only, and keeps its own value.
  {
    pkv::PerDevice<int> pd;
    int calls[pkv::kMaxDevices] = {};
    auto setup_for = [&calls](int dev) {
      return [&calls, dev](int& v) {
        ++calls[dev];
        v = 100 + dev;
        return 0;
      };
    };
    int v = -1;
    CHECK(pd.get(0, setup_for(0), &v, kBad) == 0 && v == 100 && calls[0] == 1);
    CHECK(pd.get(1, setup_for(1), &v, kBad) == 0 && v == 101 && calls[1] == 1);
    CHECK(pd.get(0, setup_for(0), &v, kBad) == 0 && v == 100 && calls[0] == 1);
    CHECK(pd.get(1, setup_for(1), nullptr, kBad) == 0 && calls[1] == 1);
    CHECK(pd.get(pkv::kMaxDevices - 1, setup_for(pkv::kMaxDevices - 1), &v, kBad) == 0 &&
          v == 100 + pkv::kMaxDevices - 1);
    // indices outside the table are refused without running the set-up
    CHECK(pd.get(-1, setup_for(0), &v, kBad) == kBad);
    CHECK(pd.get(pkv::kMaxDevices, setup_for(0), &v, kBad) == kBad);
    CHECK(calls[0] == 1);
  }
  // A failed set-up returns its status, is not kept, and runs again on the next call.
  {
    pkv::PerDevice<int> pd;
    int tries = 0, v = -1;
    CHECK(pd.get(3, [&](int&) { ++tries; return 98; }, &v, kBad) == 98 && v == -1);
    CHECK(pd.get(3, [&](int& x) { ++tries; x = 5; return 0; }, &v, kBad) == 0 && v == 5 && tries == 2);
    CHECK(pd.get(3, [&](int&) { ++tries; return 98; }, &v, kBad) == 0 && v == 5 && tries == 2);
  }
  // Many threads on many devices: one set-up per device, every caller sees its value.
  {
    pkv::PerDevice<int> pd;
    std::atomic<int> calls[8];
    for (auto& c : calls) c = 0;
    std::atomic<int> wrong{0};
    std::vector<std::thread> threads;
    for (int t = 0; t < 16; ++t) {
      threads.emplace_back([&, t] {
        for (int i = 0; i < 2000; ++i) {
          const int dev = (i + t) % 8;
          int v = -1;
          const int st = pd.get(dev, [&, dev](int& x) { calls[dev]++; x = 3 * dev + 1; return 0; }, &v, kBad);
          if (st != 0 || v != 3 * dev + 1) wrong++;
        }
      });
    }
    for (auto& th : threads) th.join();
    CHECK(wrong.load() == 0);
    for (int d = 0; d < 8; ++d) CHECK(calls[d].load() == 1);
  }
  if (failures == 0) std::puts("ok");
  return failures == 0 ? 0 : 1;
}
