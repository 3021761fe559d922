// Host-side status helpers shared by every translation unit of libpagedkv.
#pragma once

#include <cstdarg>
#include <cstdint>

#include "pagedkv.h"

namespace pagedkv {

// Record a thread-local description of a failure and return its status.
pa_status fail(pa_status s, const char* fmt, ...)
    __attribute__((format(printf, 2, 3)));

// Count one kernel launch issued by the library.
void count_launch();

// Clear the thread-local description (called on entry of each API call).
void clear_error();

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

}  // namespace pagedkv
