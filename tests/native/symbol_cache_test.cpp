// Host-only test of the policy of SymbolAddressCache (quantized_kv_cache_19_b200/csrc/symbol_cache.h):
// an address is reused only in the context it was looked up in, looked up again from any other
// context or when the context id is unknown, kept per device, left unchanged by a failed lookup,
// and safe to use from several host threads. Built and run by tests/test_capi_host.py with g++.
#include <cstdio>
#include <thread>
#include <vector>

#include "symbol_cache.h"

#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);      \
      return 1;                                               \
    }                                                         \
  } while (0)

int main() {
  qkv::SymbolAddressCache cache;
  char a[4], b[4], c[4];
  void* next = a;
  auto lookup = [&](void** p) { *p = next; return 0; };
  void* out = nullptr;

  // first lookup on device 0 in context 11
  CHECK(cache.get(0, 11, lookup, &out) == 0 && out == a && cache.lookups() == 1);
  // same device and context: the remembered address, no new lookup
  next = b;
  CHECK(cache.get(0, 11, lookup, &out) == 0 && out == a && cache.lookups() == 1);
  // a re-created context (new id) on the same device: looked up again
  CHECK(cache.get(0, 12, lookup, &out) == 0 && out == b && cache.lookups() == 2);
  // another device has its own entry
  next = c;
  CHECK(cache.get(3, 12, lookup, &out) == 0 && out == c && cache.lookups() == 3);
  CHECK(cache.get(0, 12, lookup, &out) == 0 && out == b && cache.lookups() == 3);
  // unknown context id: never trusted, always looked up
  CHECK(cache.get(0, 0, lookup, &out) == 0 && out == c && cache.lookups() == 4);
  CHECK(cache.get(0, 0, lookup, &out) == 0 && cache.lookups() == 5);
  // a failed lookup passes its code on and leaves the entry as it was
  auto failing = [&](void** p) { *p = nullptr; return 7; };
  out = nullptr;
  CHECK(cache.get(3, 99, failing, &out) == 7 && out == nullptr);
  CHECK(cache.get(3, 12, lookup, &out) == 0 && out == c);
  // device index out of range
  CHECK(cache.get(-1, 1, lookup, &out) == -1 && cache.get(64, 1, lookup, &out) == -1);

  // many threads, contexts alternating: every result is the address of the context asked for
  qkv::SymbolAddressCache shared;
  static char slots[8][4];
  std::vector<std::thread> threads;
  std::vector<int> bad(8, 0);
  for (int t = 0; t < 8; ++t) {
    threads.emplace_back([&, t] {
      for (int i = 0; i < 20000; ++i) {
        const unsigned long long ctx = 1 + ((i + t) & 1);
        void* got = nullptr;
        const int rc = shared.get(t & 1, ctx, [&](void** p) { *p = slots[ctx]; return 0; }, &got);
        if (rc != 0 || got != slots[ctx]) bad[t] = 1;
      }
    });
  }
  for (auto& th : threads) th.join();
  for (int t = 0; t < 8; ++t) CHECK(bad[t] == 0);
  std::printf("ok\n");
  return 0;
}
