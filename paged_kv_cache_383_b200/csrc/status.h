// Host-side helpers shared by every translation unit of libpagedkv: the
// status and error text of the C ABI, the launch count, and device queries.
#pragma once

#include <cudaTypedefs.h>

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

// SM count of the current device, looked up once per device ordinal (the
// launch paths ask on every call).
int device_sm_count();

// The driver's cuTensorMapEncodeTiled, or nullptr if it is unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

}  // namespace pagedkv
