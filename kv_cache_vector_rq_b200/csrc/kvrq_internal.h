// Internal helpers shared by the library's translation units (host side).
#pragma once

#include <cstdint>
#include <new>

#include "kvrq.h"

namespace kvrq {

// Records `msg` as this thread's last error and returns `st`.
kvrq_status set_error(kvrq_status st, const char* msg);

// Same, formatted (printf style).
kvrq_status set_errorf(kvrq_status st, const char* fmt, ...);

// Normal number i of the counter-based stream `seed` (splitmix64 + Box-Muller).
double stream_normal(uint64_t seed, uint64_t i);

// Called where a host entry point is about to allocate: throws std::bad_alloc while the
// allocation-failure test hook (kvrq_test_fail_allocations) has failures left to inject.
void alloc_check();

// Runs f() (an entry point's body); a host allocation that fails inside it (or one the test hook
// injects) returns KVRQ_ENOMEM instead of letting an exception cross the C ABI.
template <typename F>
kvrq_status guarded(const char* name, F&& f) {
  try {
    return f();
  } catch (const std::bad_alloc&) {
    return set_errorf(KVRQ_ENOMEM, "%s: host memory could not be allocated (nothing was changed)", name);
  } catch (...) {
    return set_errorf(KVRQ_ENOMEM, "%s: host resources could not be obtained (nothing was changed)", name);
  }
}

}  // namespace kvrq
