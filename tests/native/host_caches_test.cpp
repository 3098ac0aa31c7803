// Host-side caches of libfp8bq under many threads (no GPU needed):
//  - DeviceOnce runs each device's set-up exactly once and every caller sees
//    its result, even when 32 threads ask at the same time;
//  - a set-up that fails with a CUDA error is not cached (the next call
//    retries), UNSUPPORTED and OK are;
//  - device ordinals outside [0, kMaxDevices) are refused without a set-up;
//  - TensorMapCache returns exactly what was inserted under the same key while
//    other threads insert and look up other keys, and empties at capacity.
// Prints "ok" and exits 0 on success.
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <thread>
#include <vector>

#include "../../fp8_block_scaled_fp8bq_b200/csrc/internal.h"

using namespace fp8bq;

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

static TensorMapKey key_for(int i) {
  TensorMapKey k;
  memset(&k, 0, sizeof(k));
  k.base = reinterpret_cast<const void *>(uintptr_t(0x100000) + 256u * (uintptr_t)i);
  k.dims[0] = 4096 + i;
  k.dims[1] = 128;
  k.strides[0] = 4096;
  k.box[0] = 128;
  k.box[1] = 128;
  k.box[2] = 0;
  k.rank = 2;
  return k;
}

static CUtensorMap map_for(int i) {
  CUtensorMap m;
  memset(&m, 0, sizeof(m));
  memcpy(&m, &i, sizeof(i));
  return m;
}

static bool same(const CUtensorMap &a, const CUtensorMap &b) { return memcmp(&a, &b, sizeof(a)) == 0; }

int main() {
  constexpr int kThreads = 32, kIters = 2000, kDevs = 8;
  {
    DeviceOnce once;
    std::atomic<int> runs[kDevs];
    for (auto &r : runs) r = 0;
    std::atomic<int> bad{0};
    std::vector<std::thread> ts;
    for (int t = 0; t < kThreads; ++t)
      ts.emplace_back([&, t] {
        for (int i = 0; i < kIters; ++i) {
          const int dev = (t + i) % kDevs;
          const fp8bq_status st = once.get_for(dev, [&](int d) {
            runs[d].fetch_add(1);
            std::this_thread::yield();
            return d % 2 ? FP8BQ_ERR_UNSUPPORTED : FP8BQ_OK;
          });
          if (st != (dev % 2 ? FP8BQ_ERR_UNSUPPORTED : FP8BQ_OK)) bad.fetch_add(1);
        }
      });
    for (auto &th : ts) th.join();
    CHECK(bad.load() == 0);
    for (int d = 0; d < kDevs; ++d) CHECK(runs[d].load() == 1);
    int calls = 0;
    CHECK(once.get_for(-1, [&](int) { ++calls; return FP8BQ_OK; }) == FP8BQ_ERR_UNSUPPORTED);
    CHECK(once.get_for(kMaxDevices, [&](int) { ++calls; return FP8BQ_OK; }) == FP8BQ_ERR_UNSUPPORTED);
    CHECK(calls == 0);
  }
  {
    DeviceOnce once;  // a CUDA failure is retried, then the success sticks
    int calls = 0;
    CHECK(once.get_for(3, [&](int) { ++calls; return FP8BQ_ERR_CUDA; }) == FP8BQ_ERR_CUDA);
    CHECK(once.get_for(3, [&](int) { ++calls; return FP8BQ_OK; }) == FP8BQ_OK);
    CHECK(once.get_for(3, [&](int) { ++calls; return FP8BQ_ERR_CUDA; }) == FP8BQ_OK);
    CHECK(calls == 2);
  }
  {
    TensorMapCache cache;
    std::atomic<int> bad{0};
    std::vector<std::thread> ts;
    for (int t = 0; t < kThreads; ++t)
      ts.emplace_back([&, t] {
        for (int i = 0; i < kIters; ++i) {
          const int id = t * 64 + i % 64;  // each thread owns 64 keys
          CUtensorMap m;
          if (cache.find(key_for(id), &m)) {
            if (!same(m, map_for(id))) bad.fetch_add(1);
          } else {
            cache.insert(key_for(id), map_for(id));
          }
        }
      });
    for (auto &th : ts) th.join();
    CHECK(bad.load() == 0);
    CHECK(cache.size() == (size_t)kThreads * 64);
    for (int i = 0; i < (int)TensorMapCache::kCapacity + 10; ++i) cache.insert(key_for(100000 + i), map_for(i));
    CHECK(cache.size() <= TensorMapCache::kCapacity);
    CUtensorMap m;
    CHECK(cache.find(key_for(100000 + (int)TensorMapCache::kCapacity + 9), &m));
    CHECK(same(m, map_for((int)TensorMapCache::kCapacity + 9)));
    TensorMapKey other = key_for(100000 + (int)TensorMapCache::kCapacity + 9);
    other.box[1] = 64;  // any field of the key distinguishes entries
    CHECK(!cache.find(other, &m));
  }
  printf("ok\n");
  return 0;
}
