// Host-side unit test of dg::PerDevice (the per-device launch set-up cache
// of the head kernel), with fake "devices": two devices used alternately by
// one process, several threads racing on one device, and a set-up that fails
// once and is retried.  Prints "ok" and exits 0 on success.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "per_device.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      std::printf("FAILED %s at line %d\n", #c, __LINE__);       \
      return 1;                                                   \
    }                                                             \
  } while (0)

int main() {
  // two devices with different capacities (a 148-SM part: 74 pairs; a
  // smaller one: 66): each is set up once, on first use, with its own value
  dg::PerDevice<int> cache;
  int calls[2] = {0, 0};
  auto make_for = [&](int dev) {
    return [&, dev](int* v) {
      ++calls[dev];
      *v = dev == 0 ? 74 : 66;
      return true;
    };
  };
  int v = 0;
  CHECK(cache.get(0, make_for(0), &v) && v == 74);
  CHECK(cache.get(1, make_for(1), &v) && v == 66);
  for (int i = 0; i < 10; ++i) {
    CHECK(cache.get(i & 1, make_for(i & 1), &v) && v == ((i & 1) ? 66 : 74));
  }
  CHECK(calls[0] == 1 && calls[1] == 1);

  // a failed set-up is not remembered: the next call retries it
  dg::PerDevice<int> flaky;
  int attempts = 0;
  auto fail_once = [&](int* out) {
    ++attempts;
    if (attempts == 1) return false;
    *out = 7;
    return true;
  };
  CHECK(!flaky.get(3, fail_once, &v));
  CHECK(flaky.get(3, fail_once, &v) && v == 7);
  CHECK(flaky.get(3, fail_once, &v) && v == 7 && attempts == 2);

  // out-of-range ordinals are refused without running the set-up
  int ran = 0;
  auto count = [&](int* out) { ++ran; *out = 1; return true; };
  CHECK(!flaky.get(-1, count, &v) && !flaky.get(64, count, &v) && ran == 0);

  // eight threads racing on one device: the set-up runs exactly once
  dg::PerDevice<int> shared;
  std::atomic<int> made{0};
  std::vector<std::thread> th;
  std::atomic<int> bad{0};
  for (int t = 0; t < 8; ++t)
    th.emplace_back([&] {
      for (int i = 0; i < 1000; ++i) {
        int x = 0;
        if (!shared.get(5, [&](int* out) { ++made; *out = 42; return true; }, &x) || x != 42) ++bad;
      }
    });
  for (auto& t : th) t.join();
  CHECK(made == 1 && bad == 0);
  std::printf("ok\n");
  return 0;
}
