// pa_read_probe: read a device buffer once with streaming 128-bit loads.
// pa_wait_probe: make one bounded mbarrier wait run out.
//
// Helpers with no counterpart in the pages.  The bench times the read probe
// on a buffer much larger than L2 to get the read bandwidth this GPU actually
// sustains, the roofline the decode kernel's bandwidth is compared with.  The
// wait probe lets a test see the kernels' failure path (a wait that gives up,
// an error word, tensor memory freed, the context still usable) without a
// copy that really fails.
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

// One warp, set up the way the prefill's MMA warp is: it allocates tensor
// memory, then waits on an mbarrier that nothing ever arrives at.  The
// bounded wait gives up after its limit; the warp reports
// PA_ERR_DEVICE_TIMEOUT, frees the tensor memory and returns, as the
// kernels do when a copy never lands.
__global__ void __launch_bounds__(32) wait_probe_kernel(int32_t* dev_err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const uint32_t b = dev::smem_u32(&bar);
  if (threadIdx.x == 0) {
    dev::mbar_init(b, 1);
    dev::fence_mbar_init();
  }
  __syncwarp();
  dev::tmem_alloc(dev::smem_u32(&tmem_slot), 32);
  dev::tmem_relinquish();
  dev::tc_fence_before();
  __syncwarp();
  dev::tc_fence_after();
  const uint32_t tbase = tmem_slot;
  int ok = 1;
  if (threadIdx.x == 0) ok = dev::mbar_wait(b, 0) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok && threadIdx.x == 0) dev::set_error(dev_err, PA_ERR_DEVICE_TIMEOUT);
  __syncwarp();
  dev::tc_fence_after();
  dev::tmem_dealloc(tbase, 32);
}

}  // namespace
}  // namespace pagedkv

extern "C" pa_status pa_wait_probe(int32_t* dev_err, void* stream) {
  pagedkv::clear_error();
  if (!dev_err)
    return pagedkv::fail(PA_ERR_INVALID_ARG,
                         "pa_wait_probe: needs a device error word");
  pagedkv::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_err);
  pagedkv::count_launch();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return pagedkv::fail(PA_ERR_CUDA, "pa_wait_probe: launch failed: %s",
                         cudaGetErrorString(e));
  return PA_OK;
}

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
