// Longest-first order of sequences by context length, for grids whose row z
// serves sequence order[z]: the last CTAs to start then hold short work, so
// the grid's tail is short.  A counting sort on context_len >> shift over
// 1024 buckets, descending, run by one CTA of kOrderThreads threads.  Within
// a bucket the order follows the atomics; callers' results do not depend on
// it (each sequence is computed on its own).
#pragma once

#include <cstdint>

namespace pagedkv {
namespace {

constexpr int kOrderThreads = 1024;
constexpr int kOrderBuckets = 1024;

// Bucket shift for lengths up to max_ctx: max_ctx >> shift < 1024.
inline int order_shift(int max_ctx) {
  int shift = 0;
  while ((max_ctx >> shift) >= kOrderBuckets) ++shift;
  return shift;
}

// Called by all kOrderThreads threads of the CTA.  Counts and scans, then
// calls before_write() (e.g. a wait for the previous kernel that may still
// read `order`), then writes order[0 .. num_seqs).
template <typename BeforeWrite>
__device__ __forceinline__ void sort_longest_first(
    const int32_t* __restrict__ context_lens, int num_seqs, int shift,
    int32_t* __restrict__ order, BeforeWrite before_write) {
  __shared__ int hist[kOrderBuckets];
  __shared__ int warp_sum[kOrderThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto bucket = [&](int i) {
    const int L = context_lens[i];
    const int k = L <= 0 ? 0 : min(L >> shift, kOrderBuckets - 1);
    return kOrderBuckets - 1 - k;  // longest first
  };
  hist[tid] = 0;
  __syncthreads();
  for (int i = tid; i < num_seqs; i += kOrderThreads)
    atomicAdd(&hist[bucket(i)], 1);
  __syncthreads();
  // Exclusive scan of the 1024 bucket counts (one per thread).
  const int c = hist[tid];
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  hist[tid] = x - c + (warp > 0 ? warp_sum[warp - 1] : 0);
  __syncthreads();
  before_write();
  for (int i = tid; i < num_seqs; i += kOrderThreads)
    order[atomicAdd(&hist[bucket(i)], 1)] = i;
}

}  // namespace
}  // namespace pagedkv
