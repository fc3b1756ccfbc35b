// Host check of ScratchAddressCache (expert_ffn_execution_b200/csrc/
// scratch_cache.h) with fake contexts and a fake symbol lookup: the address
// is looked up once per (device, context), again when the current context
// changes, never cached when the lookup fails or no context handle exists,
// and an out-of-range device gives nullptr.
#include <cstdio>

#include "scratch_cache.h"

static int fails = 0;
#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      std::printf("FAIL line %d: %s\n", __LINE__, #c);        \
      ++fails;                                                \
    }                                                         \
  } while (0)

int main() {
  strata::ScratchAddressCache<4> cache;
  int ctxA = 0, ctxB = 0, addr1 = 0, addr2 = 0;
  void* cur = &ctxA;
  void* next_addr = &addr1;
  int lookups = 0;
  auto ctx_of = [&] { return cur; };
  auto lookup = [&] {
    ++lookups;
    return next_addr;
  };
  // first call in a context looks up; the next ones hit the cache
  CHECK(cache.get(0, ctx_of, lookup) == &addr1 && lookups == 1);
  CHECK(cache.get(0, ctx_of, lookup) == &addr1 && lookups == 1);
  // another device has its own slot
  CHECK(cache.get(1, ctx_of, lookup) == &addr1 && lookups == 2);
  // a new context on device 0 (e.g. after a device reset): looked up again
  cur = &ctxB;
  next_addr = &addr2;
  CHECK(cache.get(0, ctx_of, lookup) == &addr2 && lookups == 3);
  CHECK(cache.get(0, ctx_of, lookup) == &addr2 && lookups == 3);
  // a failed lookup returns nullptr and caches nothing
  cur = &ctxA;
  next_addr = nullptr;
  CHECK(cache.get(0, ctx_of, lookup) == nullptr && lookups == 4);
  next_addr = &addr1;
  CHECK(cache.get(0, ctx_of, lookup) == &addr1 && lookups == 5);
  CHECK(cache.get(0, ctx_of, lookup) == &addr1 && lookups == 5);
  // no context handle: every call looks up
  cur = nullptr;
  CHECK(cache.get(2, ctx_of, lookup) == &addr1 && lookups == 6);
  CHECK(cache.get(2, ctx_of, lookup) == &addr1 && lookups == 7);
  // out-of-range devices
  CHECK(cache.get(-1, ctx_of, lookup) == nullptr && lookups == 7);
  CHECK(cache.get(4, ctx_of, lookup) == nullptr && lookups == 7);
  if (fails) return 1;
  std::printf("ok scratch cache\n");
  return 0;
}
