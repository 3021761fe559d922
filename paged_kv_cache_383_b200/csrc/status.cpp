// Version, status strings and the thread-local error text of the C ABI;
// the launch count and the device queries the launch paths share.
#include "status.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>

namespace pagedkv {

namespace {
thread_local char g_last_error[512] = {0};
std::atomic<int64_t> g_launches{0};
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

pa_status fail(pa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

void clear_error() { g_last_error[0] = 0; }

const char* last_error() { return g_last_error; }

int device_sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int count = 148;
  cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev].store(count, std::memory_order_relaxed);
  return count;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cached{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 fn =
      cached.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

}  // namespace pagedkv

extern "C" {

const char* pa_version(void) { return "pagedkv 0.1.0 (sm_100a)"; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape";
    case PA_ERR_NO_FREE_BLOCKS: return "no free blocks";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_DEVICE_OOB: return "device-side index out of range";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* pa_last_error(void) { return pagedkv::last_error(); }

int64_t pa_launch_count(void) {
  return pagedkv::g_launches.load(std::memory_order_relaxed);
}

}  // extern "C"
