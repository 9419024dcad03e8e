// Host-only check of bl::PerDevice (the per-device, thread-safe set-up cache of the
// library's launch code): many threads on several device ordinals at once must run each
// device's initialiser exactly once and all see its value; a failing initialiser is
// retried, not cached; ordinals out of range are refused. Prints "ok" on success.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "../../ternary_weight_linear_03_b200/csrc/per_device.h"

int main() {
  bl::PerDevice cache;
  constexpr int kDevices = 8, kThreads = 32, kCalls = 2000;
  std::atomic<int> inits[kDevices];
  for (auto& a : inits) a = 0;
  std::atomic<int> wrong{0};
  std::vector<std::thread> pool;
  for (int t = 0; t < kThreads; ++t) {
    pool.emplace_back([&, t] {
      for (int i = 0; i < kCalls; ++i) {
        const int dev = (t + i) % kDevices;
        const int v = cache.get(dev, [&](int d) {
          inits[d].fetch_add(1);
          std::this_thread::yield();
          return 100 + d;
        });
        if (v != 100 + dev) wrong.fetch_add(1);
      }
    });
  }
  for (auto& th : pool) th.join();
  for (int d = 0; d < kDevices; ++d)
    if (inits[d].load() != 1) {
      std::printf("device %d initialised %d times\n", d, inits[d].load());
      return 1;
    }
  if (wrong.load() != 0) {
    std::printf("%d calls saw a wrong value\n", wrong.load());
    return 1;
  }
  // failures are returned and retried
  bl::PerDevice flaky;
  int calls = 0;
  if (flaky.get(3, [&](int) { ++calls; return 0; }) != 0) return 1;
  if (flaky.get(3, [&](int) { ++calls; return 7; }) != 7) return 1;
  if (flaky.get(3, [&](int) { ++calls; return 9; }) != 7) return 1;
  if (calls != 2) return 1;
  // ordinals out of range
  if (flaky.get(-1, [](int) { return 1; }) != -1) return 1;
  if (flaky.get(bl::kMaxDevices, [](int) { return 1; }) != -1) return 1;
  std::printf("ok\n");
  return 0;
}
