// CPU check of the per-device attribute cache (rtp_attr_cache.h) with a fake setter: every
// (instance, device) is set once, on its own, and again only for a larger size.
#include <cstdio>
#include <map>
#include <utility>

#include "../long_context_sparse_rtpurbo_b200/csrc/rtp_attr_cache.h"

int main() {
  rtp::AttrCache<4, 64> cache;
  std::map<std::pair<int, int>, int> calls;          // (device, bytes) -> calls
  auto set = [&](int dev, int bytes) { ++calls[{dev, bytes}]; return 0; };
  int bad = 0;
  auto expect = [&](bool ok, const char* what) {
    if (!ok) { std::printf("FAIL %s\n", what); ++bad; }
  };
  expect(cache.ensure(2, 0, 200000, set) == 0, "set on device 0");
  expect(cache.ensure(2, 0, 200000, set) == 0, "repeat on device 0");
  expect(calls[{0, 200000}] == 1, "device 0 set once");
  expect(cache.ensure(2, 1, 200000, set) == 0, "set on device 1");
  expect(calls[{1, 200000}] == 1, "device 1 set on its own (not skipped after device 0)");
  expect(cache.ensure(2, 1, 150000, set) == 0 && calls[{1, 150000}] == 0, "smaller size: no set");
  expect(cache.ensure(2, 1, 230000, set) == 0 && calls[{1, 230000}] == 1, "larger size: set again");
  expect(cache.ensure(3, 1, 200000, set) == 0 && calls[{1, 200000}] == 2, "other instance: own entry");
  expect(cache.ensure(2, 64, 1000, set) == -1 && cache.ensure(4, 0, 1000, set) == -1,
         "out-of-range index");
  int fails = 0;
  auto failing = [&](int, int) { ++fails; return 7; };
  expect(cache.ensure(1, 5, 1000, failing) == 7, "setter error returned");
  expect(cache.ensure(1, 5, 1000, failing) == 7 && fails == 2, "failed set is not cached");
  std::printf(bad ? "attr cache: %d failures\n" : "attr cache: ok\n", bad);
  return bad ? 1 : 0;
}
