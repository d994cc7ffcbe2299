// Host-side checks of the per-context cache the library keys its
// context-bound values with (device addresses of __device__ variables,
// raised kernel attributes, internal streams).  Built with g++ by
// tests/test_ctx_cache_cpu.py; exits non-zero on the first failure.
#include <cstdio>

#include "ctx_cache.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);          \
      return 1;                                                   \
    }                                                             \
  } while (0)

int main() {
  vsa::CtxCache<int, 4> cache;
  int calls = 0, v = 0;
  auto make = [&](int value) {
    return [&, value](int* out) { ++calls; *out = value; return true; };
  };
  // a miss looks the value up, a hit does not
  CHECK(cache.get(7, make(70), &v) && v == 70 && calls == 1);
  CHECK(cache.get(7, make(99), &v) && v == 70 && calls == 1);
  // a second context gets its own value; the first keeps its own
  CHECK(cache.get(8, make(80), &v) && v == 80 && calls == 2);
  CHECK(cache.get(7, make(99), &v) && v == 70 && calls == 2);
  // id 0 (context unknown) is never cached or looked up
  CHECK(!cache.get(0, make(1), &v) && calls == 2);
  // a failed lookup is not stored: the next call tries again
  CHECK(!cache.get(9, [&](int*) { ++calls; return false; }, &v) && calls == 3);
  CHECK(cache.get(9, make(90), &v) && v == 90 && calls == 4);
  CHECK(cache.size() == 3);
  // a destroyed context's entry never answers for a new context: ids are
  // unique, so a new id misses even when the old entry is still stored
  CHECK(cache.get(10, make(100), &v) && v == 100 && calls == 5);
  // full: the oldest entry (7) is replaced, later lookups of 7 look up again
  CHECK(cache.get(11, make(110), &v) && v == 110 && calls == 6);
  CHECK(cache.size() == 4);
  CHECK(cache.get(7, make(71), &v) && v == 71 && calls == 7);
  CHECK(cache.get(11, make(0), &v) && v == 110 && calls == 7);
  std::printf("ok\n");
  return 0;
}
