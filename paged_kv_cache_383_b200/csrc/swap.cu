// pa_swap_blocks: move whole KV blocks between two pools, either of which may
// sit in page-locked host memory, for preemption by swapping a request's KV
// cache to CPU RAM and back ([Taming the Tail] "Infrastructure Scale").
//
// One launch covers every (source, destination) pair the block manager's
// swap returned: CTA (pair, K|V) streams one block (num_kv_heads x
// block_size x head_dim elements, contiguous in the [blocks, heads, tokens,
// dim] layout) with 16-byte loads, kUnroll of them in flight per thread
// before the stores, so the link to host memory sees many outstanding
// requests.  Host pages are reached through the device-side address of the
// mapped, page-locked allocation (zero-copy); pageable host memory is
// refused on the host before any launch.  Block ids are checked on the
// device: a pair outside either pool records PA_ERR_DEVICE_OOB and is
// skipped.
#include <cuda_runtime.h>

#include <cstdint>

#include "device_utils.cuh"
#include "pagedkv.h"
#include "status.h"

namespace pagedkv {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads)
    swap_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                       const uint4* __restrict__ src_k,
                       const uint4* __restrict__ src_v,
                       const int32_t* __restrict__ pairs, int64_t block_chunks,
                       int num_src, int num_dst, int32_t* dev_err) {
  const int pair = blockIdx.x;
  const int32_t s = pairs[2 * pair];
  const int32_t d = pairs[2 * pair + 1];
  if (s < 0 || s >= num_src || d < 0 || d >= num_dst) {
    if (threadIdx.x == 0 && blockIdx.y == 0)
      dev::set_error(dev_err, PA_ERR_DEVICE_OOB);
    return;
  }
  const uint4* src = (blockIdx.y ? src_v : src_k) + s * block_chunks;
  uint4* dst = (blockIdx.y ? dst_v : dst_k) + d * block_chunks;
  for (int64_t base = threadIdx.x; base < block_chunks;
       base += static_cast<int64_t>(kThreads) * kUnroll) {
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads;
      if (i < block_chunks) r[u] = __ldcs(src + i);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads;
      if (i < block_chunks) __stcs(dst + i, r[u]);
    }
  }
}

// Address at which the current device reaches `p`: device memory of this
// device, or mapped page-locked host memory.  nullptr for anything else
// (pageable host memory, another device's memory).
void* device_view(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // the failed query's error is not sticky: clear it
    return nullptr;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      return a.device == dev ? const_cast<void*>(p) : nullptr;
    case cudaMemoryTypeHost:
      return a.devicePointer;  // NULL if the allocation is not mapped
    default:
      return nullptr;
  }
}

}  // namespace
}  // namespace pagedkv

using pagedkv::fail;

extern "C" pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache,
                                    const void* src_k_cache,
                                    const void* src_v_cache,
                                    const int32_t* pairs, int num_pairs,
                                    int num_kv_heads, int head_dim,
                                    int block_size, int num_src_blocks,
                                    int num_dst_blocks, pa_dtype dtype,
                                    int32_t* dev_err, void* stream) {
  pagedkv::clear_error();
  if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_src_blocks < 0 || num_dst_blocks < 0 || num_pairs < 0 ||
      (dtype != PA_F16 && dtype != PA_BF16))
    return fail(PA_ERR_INVALID_ARG,
                "pa_swap_blocks: num_kv_heads=%d head_dim=%d block_size=%d "
                "num_src_blocks=%d num_dst_blocks=%d num_pairs=%d dtype=%d",
                num_kv_heads, head_dim, block_size, num_src_blocks,
                num_dst_blocks, num_pairs, static_cast<int>(dtype));
  if ((head_dim * 2) % 16 != 0)
    return fail(PA_ERR_UNSUPPORTED,
                "pa_swap_blocks: head_dim*2 bytes (%d) must be a multiple of "
                "16", head_dim * 2);
  if (num_pairs == 0) return PA_OK;
  const void* ptrs[5] = {dst_k_cache, dst_v_cache, src_k_cache, src_v_cache,
                         pairs};
  const char* names[5] = {"dst_k_cache", "dst_v_cache", "src_k_cache",
                          "src_v_cache", "pairs"};
  void* view[5];
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i])
      return fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: %s is NULL",
                  names[i]);
    view[i] = pagedkv::device_view(ptrs[i]);
    if (!view[i])
      return fail(PA_ERR_INVALID_ARG,
                  "pa_swap_blocks: %s is neither memory of the current device "
                  "nor mapped page-locked host memory", names[i]);
    if (i < 4 && !pagedkv::aligned16(view[i]))
      return fail(PA_ERR_INVALID_ARG,
                  "pa_swap_blocks: %s must be 16-byte aligned", names[i]);
  }
  int32_t* err_view = nullptr;
  if (dev_err) {
    err_view = static_cast<int32_t*>(pagedkv::device_view(dev_err));
    if (!err_view)
      return fail(PA_ERR_INVALID_ARG,
                  "pa_swap_blocks: dev_err is not reachable from the device");
  }
  const int64_t block_chunks =
      static_cast<int64_t>(num_kv_heads) * block_size * head_dim * 2 / 16;
  pagedkv::swap_blocks_kernel<<<dim3(num_pairs, 2), pagedkv::kThreads, 0,
                                static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(view[0]), static_cast<uint4*>(view[1]),
      static_cast<const uint4*>(view[2]), static_cast<const uint4*>(view[3]),
      static_cast<const int32_t*>(view[4]), block_chunks, num_src_blocks,
      num_dst_blocks, err_view);
  pagedkv::count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_swap_blocks: launch failed: %s",
                cudaGetErrorString(e));
  return PA_OK;
}
