// Host-only check of the per-device setup helpers in csrc/common.cuh: many
// threads, several devices, each setup runs once per device (failures are
// retried), each cached value is computed at most a few times and then
// returned unchanged.  No kernel is launched; runs without a GPU.
#include <cstdio>
#include <thread>
#include <vector>

#include "../../token_dispatch_combine_b200/csrc/common.cuh"

int main() {
  moe::PerDeviceOnce once;
  moe::PerDeviceInt cache;
  std::atomic<int> runs[4] = {}, fails_left{3}, computes{0};
  std::vector<std::thread> pool;
  for (int t = 0; t < 16; ++t) {
    pool.emplace_back([&, t] {
      for (int i = 0; i < 2000; ++i) {
        const int dev = (t + i) % 4;
        once.run(dev, [&] {
          if (dev == 3 && fails_left.fetch_sub(1) > 0) return cudaErrorInvalidValue;  // retried later
          runs[dev].fetch_add(1);
          return cudaSuccess;
        });
        const int v = cache.get(dev, [&] {
          computes.fetch_add(1);
          return 100 + dev;
        });
        if (v != 100 + dev) {
          std::printf("bad cached value %d for device %d\n", v, dev);
          std::exit(1);
        }
      }
    });
  }
  for (auto& th : pool) th.join();
  for (int d = 0; d < 4; ++d) {
    if (runs[d].load() != 1) {
      std::printf("device %d: setup ran %d times\n", d, runs[d].load());
      return 1;
    }
  }
  // an out-of-range device index bypasses the cache
  int direct = 0;
  once.run(moe::kMaxDevices, [&] {
    ++direct;
    return cudaSuccess;
  });
  if (direct != 1) return 1;
  std::printf("ok %d\n", computes.load());
  return 0;
}
