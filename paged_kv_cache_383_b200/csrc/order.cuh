// Longest-first orders for grids whose rows serve the entries of a sorted
// list (sequences by context length, or partitions by their token count): the
// last CTAs to start then hold short work, so the grid's tail is short.  A
// counting sort over 1024 buckets, descending, run by one CTA of
// kOrderThreads threads.  Within a bucket the order follows the atomics;
// callers' results do not depend on it (each unit is computed on its own).
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

// Called by all kOrderThreads threads of the CTA.  A counting sort of items
// 0 .. n-1 by key_of(i) (a non-negative int, clipped to 1023), largest key
// first: counts and scans, then calls before_write() (e.g. a wait for the
// previous kernel that may still read the output), then place(pos, i) for
// every item, pos being its rank; thread t places items t, t + kOrderThreads,
// ...
template <typename KeyOf, typename Place, typename BeforeWrite>
__device__ __forceinline__ void counting_sort_desc_place(
    int n, KeyOf key_of, Place place, BeforeWrite before_write) {
  __shared__ int hist[kOrderBuckets];
  __shared__ int warp_sum[kOrderThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto bucket = [&](int i) {
    return kOrderBuckets - 1 - min(key_of(i), kOrderBuckets - 1);
  };
  hist[tid] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kOrderThreads) atomicAdd(&hist[bucket(i)], 1);
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
  for (int i = tid; i < n; i += kOrderThreads)
    place(atomicAdd(&hist[bucket(i)], 1), i);
}

// The same, writing out[rank] = i.
template <typename KeyOf, typename BeforeWrite>
__device__ __forceinline__ void counting_sort_desc(int n, KeyOf key_of,
                                                   int32_t* __restrict__ out,
                                                   BeforeWrite before_write) {
  counting_sort_desc_place(
      n, key_of, [&](int pos, int i) { out[pos] = i; }, before_write);
}

// The sequences by context_len >> shift over 1024 buckets, longest first.
template <typename BeforeWrite>
__device__ __forceinline__ void sort_longest_first(
    const int32_t* __restrict__ context_lens, int num_seqs, int shift,
    int32_t* __restrict__ order, BeforeWrite before_write) {
  counting_sort_desc(
      num_seqs,
      [&](int i) {
        const int L = context_lens[i];
        return L <= 0 ? 0 : (L >> shift);
      },
      order, before_write);
}

}  // namespace
}  // namespace pagedkv
