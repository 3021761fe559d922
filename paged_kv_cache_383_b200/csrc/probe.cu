// pa_read_probe: read a device buffer once with streaming 128-bit loads.
//
// A measurement helper with no counterpart in the pages: the bench times it
// on a buffer much larger than L2 to get the read bandwidth this GPU actually
// sustains, the roofline the decode kernel's bandwidth is compared with.
#include <cuda_runtime.h>

#include <cstdint>

#include "device_utils.cuh"
#include "pagedkv.h"
#include "status.h"

namespace pagedkv {
namespace {

__global__ void __launch_bounds__(512)
    read_probe_kernel(const uint4* __restrict__ p, size_t n,
                      uint32_t* __restrict__ sink) {
  uint32_t acc = 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
#pragma unroll 8
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
       i < n; i += stride) {
    const uint4 v = __ldcs(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  // The xor keeps the loads alive; the store almost never happens.
  if (acc == 0x9e3779b9u) sink[0] = acc;
}

}  // namespace
}  // namespace pagedkv

extern "C" pa_status pa_read_probe(const void* buf, size_t bytes,
                                   uint32_t* sink, void* stream) {
  pagedkv::clear_error();
  if (!buf || !sink || bytes < 16 || !pagedkv::aligned16(buf))
    return pagedkv::fail(PA_ERR_INVALID_ARG,
                         "pa_read_probe: need a 16-byte aligned buffer of at "
                         "least 16 bytes and a sink word");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  pagedkv::read_probe_kernel<<<sms * 8, 512, 0,
                               static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(buf), bytes / 16, sink);
  pagedkv::count_launch();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return pagedkv::fail(PA_ERR_CUDA, "pa_read_probe: launch failed: %s",
                         cudaGetErrorString(e));
  return PA_OK;
}
