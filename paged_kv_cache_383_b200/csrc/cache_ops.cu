// pa_cache_write (scatter new tokens' K/V into their slots) and
// pa_copy_blocks (whole-block copies for copy-on-write).
//
// Both are byte moves bound by HBM bandwidth: every thread moves 16-byte
// chunks, consecutive threads take consecutive chunks of one token row (or of
// one block), so reads and writes are fully coalesced.  Indices are checked
// on the device; a bad slot or block id records PA_ERR_DEVICE_OOB and the
// chunk is skipped, so no access ever leaves the caller's buffers.
#include <cuda_runtime.h>

#include <cstdint>

#include "device_utils.cuh"
#include "pagedkv.h"
#include "status.h"

namespace pagedkv {
namespace {

// Grid-stride over groups of kTok tokens; thread c moves 16-byte chunk c of
// each token's K row and V row (num_kv_heads * head_dim elements each), all
// kTok loads issued before the stores so each thread keeps several chunks in
// flight.  Chunk c of head h lands in the (block, h, offset) page.
constexpr int kTok = 4;

__global__ void cache_write_kernel(uint4* __restrict__ k_cache,
                                   uint4* __restrict__ v_cache,
                                   const uint4* __restrict__ k,
                                   const uint4* __restrict__ v,
                                   const int64_t* __restrict__ slot_mapping,
                                   int num_tokens, int head_chunks,
                                   int num_kv_heads, int block_size,
                                   int64_t num_slots, int32_t* dev_err) {
  dev::pdl_trigger();  // a following decode may run its prologue now
  const int row_chunks = head_chunks * num_kv_heads;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTok; t0 < num_tokens;
       t0 += static_cast<int64_t>(gridDim.x) * kTok) {
    int64_t base[kTok];  // first chunk of (block, head 0, offset), -1 = skip
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      base[u] = -1;
      const int64_t t = t0 + u;
      if (t < num_tokens) {
        const int64_t slot = slot_mapping[t];
        if (slot >= num_slots) {
          if (threadIdx.x == 0) dev::set_error(dev_err, PA_ERR_DEVICE_OOB);
        } else if (slot >= 0) {  // negative: padding token
          const int64_t blk = slot / block_size;
          const int64_t off = slot - blk * block_size;
          base[u] = (blk * num_kv_heads * block_size + off) * head_chunks;
        }
      }
    }
    for (int c = threadIdx.x; c < 2 * row_chunks; c += blockDim.x) {
      const int which = c >= row_chunks;  // 0 = K, 1 = V
      const int cc = c - which * row_chunks;
      const int h = cc / head_chunks;
      const int hc = cc - h * head_chunks;
      const uint4* src = which ? v : k;
      uint4* dst = which ? v_cache : k_cache;
      const int64_t head_off =
          static_cast<int64_t>(h) * block_size * head_chunks + hc;
      uint4 val[kTok];
#pragma unroll
      for (int u = 0; u < kTok; ++u)
        if (base[u] >= 0) val[u] = src[(t0 + u) * row_chunks + cc];
#pragma unroll
      for (int u = 0; u < kTok; ++u)
        if (base[u] >= 0) dst[base[u] + head_off] = val[u];
    }
  }
}

// grid.x = pair, grid.y = K|V; the block copies one whole physical block
// (num_kv_heads * block_size * head_dim elements, contiguous in the cache).
__global__ void copy_blocks_kernel(uint4* __restrict__ k_cache,
                                   uint4* __restrict__ v_cache,
                                   const int32_t* __restrict__ pairs,
                                   int64_t block_chunks, int num_blocks,
                                   int32_t* dev_err) {
  dev::pdl_trigger();
  const int pair = blockIdx.x;
  const int32_t src = pairs[2 * pair];
  const int32_t dst = pairs[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0)
      dev::set_error(dev_err, PA_ERR_DEVICE_OOB);
    return;
  }
  uint4* cache = blockIdx.y == 0 ? k_cache : v_cache;
  const uint4* s = cache + static_cast<int64_t>(src) * block_chunks;
  uint4* d = cache + static_cast<int64_t>(dst) * block_chunks;
  // Eight 16-byte loads in flight per thread before their stores: the
  // source and destination share one array, so the compiler may not hoist a
  // load above an earlier store, and a load-store loop would pay one memory
  // round trip per chunk (a 32 KB block is then a single round of loads).
  constexpr int kInFlight = 8;
  const int64_t stride = blockDim.x;
  for (int64_t i0 = threadIdx.x; i0 < block_chunks; i0 += stride * kInFlight) {
    uint4 v[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < block_chunks) v[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < block_chunks) d[i] = v[u];
    }
  }
}

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess)
      count = 148;
  }
  return count;
}

pa_status check_cache_shape(const char* fn, int num_kv_heads, int head_dim,
                            int block_size, int num_blocks, pa_dtype dtype) {
  if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks < 0 || (dtype != PA_F16 && dtype != PA_BF16))
    return fail(PA_ERR_INVALID_ARG,
                "%s: num_kv_heads=%d head_dim=%d block_size=%d num_blocks=%d "
                "dtype=%d", fn, num_kv_heads, head_dim, block_size, num_blocks,
                static_cast<int>(dtype));
  if ((head_dim * 2) % 16 != 0)
    return fail(PA_ERR_UNSUPPORTED,
                "%s: head_dim*2 bytes (%d) must be a multiple of 16", fn,
                head_dim * 2);
  return PA_OK;
}

}  // namespace
}  // namespace pagedkv

using pagedkv::fail;

extern "C" {

pa_status pa_cache_write(void* k_cache, void* v_cache, const void* k,
                         const void* v, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err, void* stream) {
  pagedkv::clear_error();
  pa_status st = pagedkv::check_cache_shape("pa_cache_write", num_kv_heads,
                                            head_dim, block_size, num_blocks,
                                            dtype);
  if (st != PA_OK) return st;
  if (num_tokens < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_cache_write: num_tokens=%d",
                num_tokens);
  if (num_tokens == 0) return PA_OK;
  if (!k_cache || !v_cache || !k || !v || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "pa_cache_write: NULL pointer");
  if (!pagedkv::aligned16(k_cache) || !pagedkv::aligned16(v_cache) ||
      !pagedkv::aligned16(k) || !pagedkv::aligned16(v))
    return fail(PA_ERR_INVALID_ARG,
                "pa_cache_write: tensors must be 16-byte aligned");
  const int head_chunks = head_dim * 2 / 16;
  const int row2 = 2 * num_kv_heads * head_chunks;  // chunks per token (K+V)
  const int threads = row2 >= 256 ? 256 : ((row2 + 31) / 32) * 32;
  int64_t blocks = (num_tokens + pagedkv::kTok - 1) / pagedkv::kTok;
  const int64_t cap = static_cast<int64_t>(pagedkv::sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  pagedkv::cache_write_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                                static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
      num_tokens, head_chunks, num_kv_heads, block_size,
      static_cast<int64_t>(num_blocks) * block_size, dev_err);
  pagedkv::count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_cache_write: launch failed: %s",
                cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs,
                         int num_pairs, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err, void* stream) {
  pagedkv::clear_error();
  pa_status st = pagedkv::check_cache_shape("pa_copy_blocks", num_kv_heads,
                                            head_dim, block_size, num_blocks,
                                            dtype);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || num_pairs > 0x7fffffff / 2)
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: num_pairs=%d", num_pairs);
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !pairs)
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: NULL pointer");
  if (!pagedkv::aligned16(k_cache) || !pagedkv::aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG,
                "pa_copy_blocks: caches must be 16-byte aligned");
  const int64_t block_chunks =
      static_cast<int64_t>(num_kv_heads) * block_size * head_dim * 2 / 16;
  pagedkv::copy_blocks_kernel<<<dim3(num_pairs, 2), 256, 0,
                                static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs,
      block_chunks, num_blocks, dev_err);
  pagedkv::count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_copy_blocks: launch failed: %s",
                cudaGetErrorString(e));
  return PA_OK;
}

}  // extern "C"
