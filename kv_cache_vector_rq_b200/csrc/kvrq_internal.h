// Internal helpers shared by the library's translation units (host side).
#pragma once

#include <cstdint>

#include "kvrq.h"

namespace kvrq {

// Records `msg` as this thread's last error and returns `st`.
kvrq_status set_error(kvrq_status st, const char* msg);

// Same, formatted (printf style).
kvrq_status set_errorf(kvrq_status st, const char* fmt, ...);

// Normal number i of the counter-based stream `seed` (splitmix64 + Box-Muller).
double stream_normal(uint64_t seed, uint64_t i);

}  // namespace kvrq
