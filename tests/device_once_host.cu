// Host-only check of enc::DeviceOnce (the per-device one-time set-up of the
// kernel launchers): many threads race for the first launch on a few device
// ordinals. No CUDA call is made; nvcc is used only because the header is CUDA C++.
#include <cstdio>
#include <thread>
#include <vector>

#include "internal.h"

int main() {
  constexpr int kDevices = 4, kThreads = 32, kRounds = 200;
  int failures = 0;
  for (int round = 0; round < kRounds; ++round) {
    enc::DeviceOnce once;
    std::atomic<int> inits[kDevices];
    int published[kDevices];
    for (int d = 0; d < kDevices; ++d) { inits[d] = 0; published[d] = 0; }
    std::atomic<int> go{0}, bad{0};
    std::vector<std::thread> pool;
    for (int i = 0; i < kThreads; ++i) {
      pool.emplace_back([&, i] {
        const int dev = i % kDevices;
        while (!go.load()) {
        }
        const bool ok = once.run(dev, [&] {
          inits[dev].fetch_add(1);
          published[dev] = 1000 + dev;   // plain store, published by run()
          return true;
        });
        if (!ok || published[dev] != 1000 + dev) bad.fetch_add(1);
      });
    }
    go.store(1);
    for (auto& t : pool) t.join();
    for (int d = 0; d < kDevices; ++d)
      if (inits[d].load() != 1) ++failures;
    if (bad.load()) ++failures;
  }
  // a failed init leaves the device unset, and the next call tries again
  enc::DeviceOnce once;
  int calls = 0;
  const bool first = once.run(3, [&] { ++calls; return false; });
  const bool second = once.run(3, [&] { ++calls; return true; });
  const bool third = once.run(3, [&] { ++calls; return true; });
  if (first || !second || !third || calls != 2) ++failures;
  // ordinals 64 apart share a bit
  int calls64 = 0;
  once.run(67, [&] { ++calls64; return true; });
  if (calls64 != 0) ++failures;
  std::printf("%d failures\n", failures);
  return failures == 0 ? 0 : 1;
}
