// Paged decode attention for sm_100a: pa_decode and its partition reduce.
//
// What is computed ([Taming the Tail] "Under the Hood: The CUDA Kernel
// Engineering"; [KV-cache chapter] "PagedAttention: borrowing virtual memory
// ..." and "Common misconception..."): for each sequence b and query head h,
// softmax(scale * K_b q) V_b over the sequence's tokens, K_b / V_b gathered
// block by block through the block table.  The pages ask three things of the
// kernel: look the physical block up in the table, keep the accesses
// coalesced despite the scattered blocks, and handle a partly filled last
// block.  Their sketch (one fp32 element per thread) is prior art only.
//
// B200 design.
//  * Work unit = (partition of <= partition_size tokens, KV head, sequence):
//    one CTA.  All G = Hq/Hkv query heads of the KV head are served by the
//    same CTA, so each K/V byte leaves HBM once.
//  * Warp 0, lane 0 is the producer.  It stages the unit's slice of the block
//    table in shared memory and issues 2-D TMA tile loads of whole pages
//    (block_size rows x 128 B, 128-byte swizzle, no multicast) into an
//    S-stage ring, each stage one K page + one V page, signalled by mbarriers
//    with transaction counts.  Waits are bounded (1 s) and report
//    PA_ERR_DEVICE_TIMEOUT instead of hanging.
//  * Warps 1..4 are consumers; consumer w takes pages w, w+4, ... and keeps
//    its own online-softmax state (running max m, sum l, accumulator o) for
//    all G heads.  At the end the four states are merged through shared
//    memory.
//  * Compute variant MMA (default): S^T = K_page . Q^T and O^T += V^T . P^T as
//    m16n8k16 tensor-core MMAs, N = 8 = the (padded) query-head group.  K
//    fragments come from ldmatrix, V fragments from ldmatrix.trans, P moves
//    from the score accumulator layout to the B-operand layout with
//    movmatrix.  P is split into a rounded part and its residual (two
//    16-bit operands) so PV keeps ~16 mantissa bits; accumulation is fp32.
//  * Compute variant SIMT: fp32 FMA dot products on the CUDA cores (kept to
//    show what the tensor-core mapping buys).
//  * A sequence that needs more than one partition writes (m, l, o/l) per
//    partition to the workspace.  With at most 16 partitions the partition
//    CTA that finishes last combines them (fence + ticket, nobody waits);
//    otherwise, or on request, a separate reduce kernel does.  A sequence
//    that fits one partition is written straight to `out`.
//  * With the reduce kernel and partitions of <= 1024 tokens, a CTA serves
//    four consecutive partitions, one per consumer warp (pages interleaved
//    so each warp still owns its ring stages): no cross-warp merge.
//  * A one-CTA prep kernel runs first: it orders the sequences longest
//    first (grid row z serves order[z], so the grid ends on short work) and
//    resets the partition counters.  Kernels are chained by programmatic
//    dependent launch.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "device_utils.cuh"
#include "order.cuh"
#include "pagedkv.h"
#include "status.h"

// Built-in scratch for pa_decode_noalloc: a fixed device array that lives in
// this library's module on every GPU that loads it, for callers that cannot
// allocate device memory.  In host code this name is only a stand-in, not a
// device address: scratch_address() below asks the runtime for the address,
// once per CUDA context.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace pagedkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kConsumers = 4;                      // consumer warps per CTA
constexpr int kThreads = (kConsumers + 1) * 32;    // + one producer warp
constexpr int kMaxGroup = 8;                       // query heads per KV head
constexpr int kMaxPartition = 8192;
constexpr int kMaxParts = 16384;                   // partitions per sequence
constexpr int kFusedMaxParts = 16;  // up to this many: combine in the decode
constexpr int kWarpPartsMaxPartition = 1024;  // warp_parts up to this size

struct DecodeArgs {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;   // [num_seqs, num_q_heads, max_parts, head_dim]
  float* ws_ml;  // [num_seqs, num_q_heads, max_parts, 2] = (max, sum), log2 units
  int* counters; // [num_seqs, num_kv_heads] finished partitions (fused mode)
  const int32_t* order;  // [num_seqs] sequence served by grid row z
  // [num_seqs * max_parts] partition units longest first (entry u: sequence
  // u / max_parts, partition u % max_parts); non-null when the grid is
  // (KV head, unit) rather than (partition, KV head, sequence)
  const int32_t* units;
  int fused;     // 1: the last partition CTA combines; 0: the reduce kernel
  int warp_parts;  // 1: a CTA serves kConsumers consecutive partitions, one
                   // per consumer warp (reduce kernel path, short partitions)
  int32_t* dev_err;
  float scale_log2;  // scale * log2(e): scores are kept in base-2 units
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int partition_size;
  int max_parts;
  int max_context_len;
  int out_f32;   // 1: out is float32 (the value before the cast to T)
};

// Shared-memory geometry of one (block_size, head_dim, stages) instance.
// A page (one block, one KV head) is head_dim/64 TMA boxes of block_size
// rows x 128 bytes; within a box, 16-byte chunk c of row r sits at chunk
// c ^ (r % 8) (the TMA 128-byte swizzle), so eight consecutive rows read at
// the same logical chunk hit eight different bank groups.
template <int BS, int D, int S>
struct Geometry {
  // Consumer warp w takes pages w, w+4, ... and page i sits in stage i % S.
  // With S a multiple of the consumer count a warp owns its stages, so it
  // waits on every use of them in order and a parity wait can never run two
  // phases ahead (a parity test cannot tell phase m from m-2).
  static_assert(S % kConsumers == 0, "stages must be a multiple of consumers");
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = BS * 128;
  static constexpr int kPageBytes = kBoxes * kBoxBytes;
  static constexpr int kStageBytes = 2 * kPageBytes;  // K page then V page
  static constexpr int kRingBytes = S * kStageBytes;
  static constexpr int kBarBytes = 2 * S * 8;         // full[S], empty[S]
  // Per consumer warp: o[8][kORow], m[8], l[8] (fp32); aliases the ring.
  // Rows are padded by 4 floats so the four head pairs a warp writes at
  // once land in different banks.
  static constexpr int kORow = D + 4;
  static constexpr int kEpiWarpFloats = kMaxGroup * kORow + 2 * kMaxGroup;
  static_assert(kConsumers * kEpiWarpFloats * 4 <= kRingBytes,
                "epilogue must fit in the ring");
  // SIMT scratch: q in fp32 with a 4-float skew between the two halves of a
  // row (bank spread), then per warp scores[BS][8], alpha[8], m_new[8].
  static constexpr int kQRow = D + 8;
  static constexpr int kSimtQFloats = kMaxGroup * kQRow;
  static constexpr int kSimtWarpFloats = BS * kMaxGroup + 2 * kMaxGroup;
  static constexpr int kSimtBytes =
      (kSimtQFloats + kConsumers * kSimtWarpFloats) * 4;

  // Byte offset of element (row, col) inside a page.
  static __device__ __forceinline__ uint32_t offset(int row, int col) {
    return (col >> 6) * kBoxBytes + row * 128 +
           ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
  }
};

// Bytes of the staged block-table slice, rounded to 16.
__host__ __device__ constexpr int bt_bytes(int pages_per_part) {
  return (pages_per_part * 4 + 15) & ~15;
}

// Dynamic shared memory of one CTA: alignment slack, ring, barriers, the
// block-table slice and (SIMT only) the fp32 scratch.
template <int BS, int D, int S, bool kMma>
constexpr size_t smem_bytes_for(int pages_per_part) {
  using G = Geometry<BS, D, S>;
  return 1024 + G::kRingBytes + G::kBarBytes + bt_bytes(pages_per_part) +
         (kMma ? 0 : G::kSimtBytes);
}

template <typename T>
__device__ __forceinline__ T from_float(float x);
template <>
__device__ __forceinline__ __nv_bfloat16 from_float(float x) {
  return __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ __half from_float(float x) {
  return __float2half_rn(x);
}

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float to_float(__half x) {
  return __half2float(x);
}

__device__ __forceinline__ float warp_max_xor(float v, int lo_mask,
                                              int hi_mask) {
  for (int m = lo_mask; m <= hi_mask; m <<= 1)
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Final store of one output element: rounded once to the output dtype, or,
// on request, the fp32 value itself (lets tests separate the kernel's error
// from the output rounding).
template <typename T>
__device__ __forceinline__ void store_out(const DecodeArgs& a, int64_t idx,
                                          float v) {
  if (a.out_f32)
    static_cast<float*>(a.out)[idx] = v;
  else
    static_cast<T*>(a.out)[idx] = from_float<T>(v);
}

// ---------------------------------------------------------------------------
// Fused combine of one (sequence, KV head)'s partitions, run by threads
// [t, ...) step nt of the partition CTA that finished last:
//   out = sum_j w_j o_j / sum_j w_j,  w_j = l_j 2^(m_j - M),  M = max_j m_j.
// Thread item = (query head g, 16-lane slice of head_dim); four partitions
// are loaded before they are folded.
template <typename T, int D>
__device__ __forceinline__ void combine_partials(const DecodeArgs& a, int b,
                                                 int kvh, int n_parts, int t,
                                                 int nt) {
  constexpr int kDT = D / 16;  // dims per thread: 8 or 4
  const int G = a.group;
  const float2* ml2 = reinterpret_cast<const float2*>(a.ws_ml);
  for (int item = t; item < G * 16; item += nt) {
    const int g = item >> 4;
    const int d0 = (item & 15) * kDT;
    const int64_t row0 =
        (static_cast<int64_t>(b) * a.num_q_heads + kvh * G + g) * a.max_parts;
    float M = -INFINITY, W = 0.f;
    float acc[kDT];
#pragma unroll
    for (int e = 0; e < kDT; ++e) acc[e] = 0.f;
    for (int j0 = 0; j0 < n_parts; j0 += 4) {
      float2 mlj[4];
      float oj[4][kDT];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u;
        mlj[u] = j < n_parts ? __ldcg(ml2 + row0 + j)
                             : make_float2(-INFINITY, 0.f);
        const float4* src =
            reinterpret_cast<const float4*>(a.ws_o + (row0 + j) * D + d0);
#pragma unroll
        for (int v = 0; v < kDT / 4; ++v) {
          const float4 x = j < n_parts ? __ldcg(src + v)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
          oj[u][4 * v] = x.x;
          oj[u][4 * v + 1] = x.y;
          oj[u][4 * v + 2] = x.z;
          oj[u][4 * v + 3] = x.w;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (mlj[u].x == -INFINITY) continue;  // empty or skipped partition
        if (mlj[u].x > M) {
          const float sc = dev::fast_exp2(M - mlj[u].x);  // 0 when M = -inf
          W *= sc;
#pragma unroll
          for (int e = 0; e < kDT; ++e) acc[e] *= sc;
          M = mlj[u].x;
        }
        const float w = mlj[u].y * dev::fast_exp2(mlj[u].x - M);
        W += w;
#pragma unroll
        for (int e = 0; e < kDT; ++e) acc[e] += w * oj[u][e];
      }
    }
    const int64_t dst =
        (static_cast<int64_t>(b) * a.num_q_heads + kvh * G + g) * D + d0;
#pragma unroll
    for (int e = 0; e < kDT; ++e)
      store_out<T>(a, dst + e, W > 0.f ? acc[e] / W : 0.f);
  }
}

// ---------------------------------------------------------------------------
// The decode kernel.
template <typename T, int BS, int D, int S, bool kMma>
__global__ void __launch_bounds__(kThreads)
    decode_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap,
                  const DecodeArgs a) {
  using Geo = Geometry<BS, D, S>;
  extern __shared__ uint8_t smem_dyn[];
  // The TMA swizzle is a function of shared-memory address bits, so the ring
  // must start on a 1024-byte boundary of the shared window.
  uint8_t* smem = smem_dyn + ((1024u - (dev::smem_u32(smem_dyn) & 1023u)) & 1023u);

  // Partitions this CTA serves: one, or (warp_parts) kConsumers consecutive
  // ones, consumer warp w taking partition part + w.
  const int nsub = a.warp_parts ? kConsumers : 1;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  dev::pdl_trigger();  // the reduce may start its prologue early
  // Grid rows are handed out longest first (the order the prep kernel wrote,
  // which this grid may only read after waiting for it), so the last CTAs
  // to start are short ones and the tail of the grid is short: partition
  // units by their token count (all KV heads of a unit side by side), or
  // sequences by length (their partitions side by side).
  int part, kvh, b;
  if (a.units) {
    kvh = blockIdx.x;
    dev::pdl_wait();
    const int u = a.units[blockIdx.y];
    b = u / a.max_parts;
    part = u - b * a.max_parts;
  } else {
    part = blockIdx.x * nsub;
    kvh = blockIdx.y;
    b = blockIdx.z;
    if (a.order) {
      dev::pdl_wait();
      b = a.order[blockIdx.z];
    }
  }
  const int PS = a.partition_size;
  const int pages_per_part = PS / BS;
  const int page0 = part * pages_per_part;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Geo::kRingBytes);
  int32_t* bt_s = reinterpret_cast<int32_t*>(bars + 2 * S);
  const uint32_t ring = dev::smem_u32(smem);
  const uint32_t full0 = dev::smem_u32(bars);
  const uint32_t empty0 = full0 + S * 8;

  // The context length and this partition's slice of the block table are
  // fetched together: the slice is read as if the partition were full (clipped
  // to the table row) so the two loads do not wait on each other; entries past
  // the sequence's end are never used.
  const int32_t* bt_row =
      a.block_tables + static_cast<int64_t>(b) * a.max_blocks_per_seq + page0;
  const int row_left = a.max_blocks_per_seq - page0;
  const int ctx = a.context_lens[b];
  for (int i = tid; i < nsub * pages_per_part && i < row_left; i += kThreads)
    bt_s[i] = bt_row[i];
  if (ctx < 0 || ctx > a.max_blocks_per_seq * BS || ctx > a.max_context_len) {
    if (part == 0 && kvh == 0 && tid == 0)
      dev::set_error(a.dev_err, PA_ERR_DEVICE_OOB);
    return;
  }
  const int n_parts = ctx > 0 ? (ctx + PS - 1) / PS : 1;
  if (part >= n_parts) return;
  const int tok0 = part * PS;
  // Tokens (and staged pages) of this CTA's partitions; 0 only when ctx == 0.
  const int n_tok = min(ctx - tok0, nsub * PS);
  const int n_pages = (n_tok + BS - 1) / BS;
  const int G = a.group;

  // Check every block id the partition uses (each thread the entries it
  // staged itself).
  int bad = 0;
  for (int i = tid; i < n_pages; i += kThreads)
    bad |= (bt_s[i] < 0 || bt_s[i] >= a.num_blocks);
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      dev::mbar_init(full0 + s * 8, 1);
      dev::mbar_init(empty0 + s * 8, 1);
    }
    dev::fence_mbar_init();
  }
  bad = __syncthreads_or(bad);
  // Everything above reads only host-written inputs; the K/V pages and the
  // outputs may belong to the previous kernel in the stream.
  dev::pdl_wait();
  __shared__ int s_last;
  if (bad) {
    if (tid == 0) dev::set_error(a.dev_err, PA_ERR_DEVICE_OOB);
    if (n_parts > 1) {
      // mark the CTA's partitions empty for the combine
      for (int k = 0; k < nsub && part + k < n_parts; ++k)
        if (tid < G) {
          const int64_t row =
              (static_cast<int64_t>(b) * a.num_q_heads + kvh * G + tid) *
                  a.max_parts + part + k;
          a.ws_ml[2 * row] = -INFINITY;
          a.ws_ml[2 * row + 1] = 0.f;
        }
      if (a.fused) {  // still counts as finished: the others may be fine
        __threadfence();
        __syncthreads();
        if (tid == 0)
          s_last = atomicAdd(a.counters + b * a.num_kv_heads + kvh, 1) ==
                   n_parts - 1;
        __syncthreads();
        if (s_last) {
          __threadfence();
          combine_partials<T, D>(a, b, kvh, n_parts, tid, kThreads);
        }
      }
    }
    return;
  }

  // ---------------- producer ----------------
  if (warp == 0) {
    if (lane == 0 && n_pages > 0) {
      dev::prefetch_tmap(&kmap);
      dev::prefetch_tmap(&vmap);
      // warp_parts: pages are interleaved across the partitions (index i is
      // page i / kConsumers of partition i % kConsumers), so consumer warp w
      // still gets every page i = w (mod kConsumers) and owns its stages;
      // pages past a shorter partition's end are skipped, which only ever
      // stops the reuse of that warp's stages.
      const int n_iter =
          a.warp_parts ? kConsumers * min(n_pages, pages_per_part) : n_pages;
      for (int i = 0; i < n_iter; ++i) {
        int slot = i;
        if (a.warp_parts) {
          slot = (i % kConsumers) * pages_per_part + i / kConsumers;
          if (slot >= n_pages) continue;
        }
        const int s = i % S;
        if (i >= S && !dev::mbar_wait(empty0 + s * 8, ((i / S) - 1) & 1)) {
          dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
          break;
        }
        const uint32_t full = full0 + s * 8;
        dev::mbar_arrive_expect_tx(full, Geo::kStageBytes);
        const int y = (bt_s[slot] * a.num_kv_heads + kvh) * BS;
        const uint32_t kdst = ring + s * Geo::kStageBytes;
#pragma unroll
        for (int bx = 0; bx < Geo::kBoxes; ++bx) {
          dev::tma_load_2d(kdst + bx * Geo::kBoxBytes, &kmap, bx * 64, y, full);
          dev::tma_load_2d(kdst + Geo::kPageBytes + bx * Geo::kBoxBytes, &vmap,
                           bx * 64, y, full);
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp - 1;
  const int ctid = tid - 32;  // 0 .. kConsumers*32-1
  const T* qrow = static_cast<const T*>(a.q) +
                  (static_cast<int64_t>(b) * a.num_q_heads + kvh * G) * D;
  float m_fin[2], l_fin[2];  // per-lane head state handed to the epilogue

  if constexpr (kMma) {
    using M = dev::Mma<T>;
    const int g4 = lane >> 2;  // fragment row group
    const int t4 = lane & 3;   // thread in group
    // B fragments of Q^T (K = head_dim, N = 8 heads): head g4, dims
    // kk*16 + 2*t4 (+1) and +8.  Heads past G are zero.
    uint32_t qf[D / 16][2];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        qf[kk][r] = 0u;
        if (g4 < G)
          qf[kk][r] = *reinterpret_cast<const uint32_t*>(
              qrow + g4 * D + kk * 16 + r * 8 + 2 * t4);
      }
    }
    float o[D / 16][4];
#pragma unroll
    for (int i = 0; i < D / 16; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};

    // ldmatrix lane roles: matrix mi = lane/8, row j = lane%8.
    const int mi = lane >> 3;
    const int j = lane & 7;

    // Tokens this warp's pages cover: the CTA's partition (the warps share
    // it), or with warp_parts this warp's own partition part + cw.
    const int w_tok = a.warp_parts ? max(0, min(n_tok - cw * PS, PS)) : n_tok;
    const int w_iter =
        a.warp_parts ? kConsumers * ((w_tok + BS - 1) / BS) : n_pages;
    for (int i = cw; i < w_iter; i += kConsumers) {
      const int s = i % S;
      if (!dev::mbar_wait(full0 + s * 8, (i / S) & 1)) {
        dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
        break;
      }
      const uint32_t kb = ring + s * Geo::kStageBytes;
      const uint32_t vb = kb + Geo::kPageBytes;
      const int pg = a.warp_parts ? i / kConsumers : i;  // page of w_tok
      const int nv = min(BS, w_tok - pg * BS);
      if (nv < BS) {
        // Slots past the context get P = 0, but 0 * NaN is NaN in the MMA:
        // clear the V rows the sequence never wrote (last page only).
        for (int idx = lane; idx < (BS - nv) * Geo::kBoxes * 8; idx += 32) {
          const int row = nv + idx / (Geo::kBoxes * 8);
          const int c = idx % (Geo::kBoxes * 8);
          dev::st_shared_zero16(vb + (c >> 3) * Geo::kBoxBytes + row * 128 +
                                (c & 7) * 16);
        }
        dev::fence_proxy_async_smem();  // before TMA reuses the stage
        __syncwarp();
      }

      // S^T (tokens x heads) for each 16-token slice of the page.
      float sc[BS / 16][4];
#pragma unroll
      for (int mt = 0; mt < BS / 16; ++mt) {
        float acc0[4] = {0.f, 0.f, 0.f, 0.f};
        float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t af[4];
          dev::ldsm_x4(kb + Geo::offset(mt * 16 + j + (mi & 1) * 8,
                                        kk * 16 + (mi >> 1) * 8),
                       af);
          if (kk & 1)
            M::run(acc1, af, qf[kk][0], qf[kk][1]);
          else
            M::run(acc0, af, qf[kk][0], qf[kk][1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = mt * 16 + g4 + (e >> 1) * 8;
          const float x = (acc0[e] + acc1[e]) * a.scale_log2;
          sc[mt][e] = tok < nv ? x : -INFINITY;
        }
      }
      // Online softmax; this lane holds heads 2*t4 and 2*t4+1.
      float alpha[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mx = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < BS / 16; ++mt)
          mx = fmaxf(mx, fmaxf(sc[mt][h], sc[mt][h + 2]));
        mx = warp_max_xor(mx, 4, 16);
        const float m_new = fmaxf(m_run[h], mx);
        alpha[h] = dev::fast_exp2(m_run[h] - m_new);
        float sum = 0.f;
#pragma unroll
        for (int mt = 0; mt < BS / 16; ++mt) {
          sc[mt][h] = dev::fast_exp2(sc[mt][h] - m_new);
          sc[mt][h + 2] = dev::fast_exp2(sc[mt][h + 2] - m_new);
          sum += sc[mt][h] + sc[mt][h + 2];
        }
        l_run[h] = l_run[h] * alpha[h] + sum;
        m_run[h] = m_new;
      }
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[dt][e] *= alpha[e & 1];

      // P^T as B fragments (K = tokens, N = heads): rounded part and residual.
      uint32_t bh[BS / 16][2], bl[BS / 16][2];
#pragma unroll
      for (int ks = 0; ks < BS / 16; ++ks) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float p0 = sc[ks][2 * r], p1 = sc[ks][2 * r + 1];
          const uint32_t hi = M::pack(p0, p1);
          const float2 hf = M::unpack(hi);
          const uint32_t lo = M::pack(p0 - hf.x, p1 - hf.y);
          bh[ks][r] = dev::movmatrix_trans(hi);
          bl[ks][r] = dev::movmatrix_trans(lo);
        }
      }
      // O^T (head_dim x heads) += V^T . P^T
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
#pragma unroll
        for (int ks = 0; ks < BS / 16; ++ks) {
          uint32_t af[4];
          dev::ldsm_x4_trans(vb + Geo::offset(ks * 16 + j + (mi >> 1) * 8,
                                              dt * 16 + (mi & 1) * 8),
                             af);
          M::run(o[dt], af, bh[ks][0], bh[ks][1]);
          M::run(o[dt], af, bl[ks][0], bl[ks][1]);
        }
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(empty0 + s * 8);
    }

    if (a.warp_parts) {
      // This warp's partition is complete: write its partial directly
      // (no merge with the other warps, which hold other partitions).
      const int mypart = part + cw;
      if (mypart < n_parts) {
        float lt[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float l = l_run[h];
          l += __shfl_xor_sync(0xffffffffu, l, 4);
          l += __shfl_xor_sync(0xffffffffu, l, 8);
          l += __shfl_xor_sync(0xffffffffu, l, 16);
          lt[h] = l;
        }
        const int64_t row0 =
            static_cast<int64_t>(b) * a.num_q_heads + kvh * G;
        if (n_parts == 1) {
          // The reduce kernel skips single-partition rows: write the output.
#pragma unroll
          for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int g = 2 * t4 + (e & 1);
              if (g < G) {
                const float l = lt[e & 1];
                store_out<T>(a, (row0 + g) * D + dt * 16 + g4 + (e >> 1) * 8,
                             l > 0.f ? o[dt][e] / l : 0.f);
              }
            }
          return;
        }
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int g = 2 * t4 + (e & 1);
            if (g < G) {
              const int64_t row = (row0 + g) * a.max_parts + mypart;
              const float l = lt[e & 1];
              a.ws_o[row * D + dt * 16 + g4 + (e >> 1) * 8] =
                  l > 0.f ? o[dt][e] / l : 0.f;
            }
          }
        if (g4 == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int g = 2 * t4 + h;
            if (g < G) {
              const int64_t row = (row0 + g) * a.max_parts + mypart;
              a.ws_ml[2 * row] = m_run[h];
              a.ws_ml[2 * row + 1] = lt[h];
            }
          }
        }
      }
      return;
    }
    // Hand this warp's state to the epilogue area (aliases the ring).
    dev::named_barrier(1, kConsumers * 32);
    float* ep = reinterpret_cast<float*>(smem) + cw * Geo::kEpiWarpFloats;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float l = l_run[h];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      m_fin[h] = m_run[h];
      l_fin[h] = l;
    }
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        ep[(2 * t4 + (e & 1)) * Geo::kORow + dt * 16 + g4 + (e >> 1) * 8] =
            o[dt][e];
    if (g4 == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        ep[kMaxGroup * Geo::kORow + 2 * t4 + h] = m_fin[h];
        ep[kMaxGroup * Geo::kORow + kMaxGroup + 2 * t4 + h] = l_fin[h];
      }
    }
  } else {
    // ---------------- SIMT variant ----------------
    float* q_s = reinterpret_cast<float*>(
        reinterpret_cast<uint8_t*>(bt_s) + bt_bytes(PS / BS));
    float* wsp = q_s + Geo::kSimtQFloats + cw * Geo::kSimtWarpFloats;
    float* sp = wsp;                      // scores / probabilities [BS][8]
    float* alpha_s = wsp + BS * kMaxGroup;
    float* mnew_s = alpha_s + kMaxGroup;

    // q -> fp32 shared copy; half h of a row is skewed by 4h floats.
    for (int idx = ctid; idx < kMaxGroup * D; idx += kConsumers * 32) {
      const int g = idx / D, d = idx % D;
      const float v = g < G ? to_float<T>(qrow[g * D + d]) : 0.f;
      q_s[g * Geo::kQRow + d + (d >= D / 2 ? 4 : 0)] = v;
    }
    dev::named_barrier(1, kConsumers * 32);

    // QK roles: BS=16 -> token lane%16, half lane/16; BS=32 -> token lane.
    constexpr int kHalves = 32 / BS;       // 2 or 1
    constexpr int kDPer = D / kHalves;     // dims per lane in QK
    const int qtok = lane % BS;
    const int qhalf = lane / BS;
    // PV roles: lane owns dims [lane*D/32, +D/32).
    constexpr int kDPV = D / 32;           // 4 or 2
    const int d0 = lane * kDPV;

    float acc_o[kMaxGroup][kDPV];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
#pragma unroll
      for (int e = 0; e < kDPV; ++e) acc_o[g][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // lanes 0..7: head `lane`

    for (int i = cw; i < n_pages; i += kConsumers) {
      const int s = i % S;
      if (!dev::mbar_wait(full0 + s * 8, (i / S) & 1)) {
        dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
        break;
      }
      const uint8_t* kpg = smem + s * Geo::kStageBytes;
      const uint8_t* vpg = kpg + Geo::kPageBytes;
      const int nv = min(BS, n_tok - i * BS);

      float acc[kMaxGroup];
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) acc[g] = 0.f;
#pragma unroll 2
      for (int c = 0; c < kDPer / 8; ++c) {
        const int d = qhalf * kDPer + c * 8;
        const uint4 raw = *reinterpret_cast<const uint4*>(
            kpg + Geo::offset(qtok, d));
        const T* kv = reinterpret_cast<const T*>(&raw);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) kf[e] = to_float<T>(kv[e]);
        const float* qd = q_s + d + (d >= D / 2 ? 4 : 0);
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
          const float4 qa = *reinterpret_cast<const float4*>(qd + g * Geo::kQRow);
          const float4 qb =
              *reinterpret_cast<const float4*>(qd + g * Geo::kQRow + 4);
          acc[g] += qa.x * kf[0] + qa.y * kf[1] + qa.z * kf[2] + qa.w * kf[3] +
                    qb.x * kf[4] + qb.y * kf[5] + qb.z * kf[6] + qb.w * kf[7];
        }
      }
      if (kHalves == 2) {
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
          acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 16);
      }
      if (qhalf == 0) {
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
          sp[qtok * kMaxGroup + g] =
              qtok < nv ? acc[g] * a.scale_log2 : -INFINITY;
      }
      __syncwarp();
      if (lane < kMaxGroup) {
        float mx = -INFINITY;
        for (int t = 0; t < BS; ++t) mx = fmaxf(mx, sp[t * kMaxGroup + lane]);
        const float m_new = fmaxf(m_run, mx);
        alpha_s[lane] = dev::fast_exp2(m_run - m_new);
        mnew_s[lane] = m_new;
        m_run = m_new;
      }
      __syncwarp();
      for (int idx = lane; idx < BS * kMaxGroup; idx += 32)
        sp[idx] = dev::fast_exp2(sp[idx] - mnew_s[idx % kMaxGroup]);
      __syncwarp();
      if (lane < kMaxGroup) {
        float sum = 0.f;
        for (int t = 0; t < BS; ++t) sum += sp[t * kMaxGroup + lane];
        l_run = l_run * alpha_s[lane] + sum;
      }
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) {
        const float al = alpha_s[g];
#pragma unroll
        for (int e = 0; e < kDPV; ++e) acc_o[g][e] *= al;
      }
      for (int t = 0; t < nv; ++t) {
        float vf[kDPV];
        if constexpr (kDPV == 4) {
          const uint2 raw = *reinterpret_cast<const uint2*>(
              vpg + Geo::offset(t, d0));
          const T* vv = reinterpret_cast<const T*>(&raw);
#pragma unroll
          for (int e = 0; e < 4; ++e) vf[e] = to_float<T>(vv[e]);
        } else {
          const uint32_t raw = *reinterpret_cast<const uint32_t*>(
              vpg + Geo::offset(t, d0));
          const T* vv = reinterpret_cast<const T*>(&raw);
#pragma unroll
          for (int e = 0; e < 2; ++e) vf[e] = to_float<T>(vv[e]);
        }
        const float4 pa =
            *reinterpret_cast<const float4*>(sp + t * kMaxGroup);
        const float4 pb =
            *reinterpret_cast<const float4*>(sp + t * kMaxGroup + 4);
        const float p[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
#pragma unroll
          for (int e = 0; e < kDPV; ++e) acc_o[g][e] += p[g] * vf[e];
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(empty0 + s * 8);
    }

    dev::named_barrier(1, kConsumers * 32);
    float* ep = reinterpret_cast<float*>(smem) + cw * Geo::kEpiWarpFloats;
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
#pragma unroll
      for (int e = 0; e < kDPV; ++e)
        ep[g * Geo::kORow + d0 + e] = acc_o[g][e];
    if (lane < kMaxGroup) {
      ep[kMaxGroup * Geo::kORow + lane] = m_run;
      ep[kMaxGroup * Geo::kORow + kMaxGroup + lane] = l_run;
    }
    (void)m_fin;
    (void)l_fin;
  }

  // ---------------- merge the consumer warps, write the result -------------
  dev::named_barrier(1, kConsumers * 32);
  const float* ep0 = reinterpret_cast<const float*>(smem);
  const bool split = n_parts > 1;
  for (int idx = ctid; idx < G * D; idx += kConsumers * 32) {
    const int g = idx / D, d = idx % D;
    float mmax = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w)
      mmax = fmaxf(mmax,
                   ep0[w * Geo::kEpiWarpFloats + kMaxGroup * Geo::kORow + g]);
    float val = 0.f, wsum = 0.f;
    if (mmax != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
        const float* e = ep0 + w * Geo::kEpiWarpFloats;
        const float mw = e[kMaxGroup * Geo::kORow + g];
        const float sc = mw == -INFINITY ? 0.f : dev::fast_exp2(mw - mmax);
        wsum += e[kMaxGroup * Geo::kORow + kMaxGroup + g] * sc;
        val += e[g * Geo::kORow + d] * sc;
      }
      val = wsum > 0.f ? val / wsum : 0.f;
    }
    const int qh = kvh * G + g;
    if (!split) {
      store_out<T>(a, (static_cast<int64_t>(b) * a.num_q_heads + qh) * D + d,
                   val);
    } else {
      const int64_t row =
          (static_cast<int64_t>(b) * a.num_q_heads + qh) * a.max_parts + part;
      a.ws_o[row * D + d] = val;
      if (d == 0) {
        a.ws_ml[2 * row] = mmax;
        a.ws_ml[2 * row + 1] = wsum;
      }
    }
  }
  if (split && a.fused) {
    // Publish this partition; the partition CTA that finishes last combines
    // all of them (fence + ticket: nobody waits for anybody).
    __threadfence();
    dev::named_barrier(1, kConsumers * 32);
    if (ctid == 0)
      s_last = atomicAdd(a.counters + b * a.num_kv_heads + kvh, 1) ==
               n_parts - 1;
    dev::named_barrier(1, kConsumers * 32);
    if (s_last) {
      __threadfence();
      combine_partials<T, D>(a, b, kvh, n_parts, ctid, kConsumers * 32);
    }
  }
}

// ---------------------------------------------------------------------------
// Prep kernel (one CTA), run before every decode: orders the sequences
// longest first (a counting sort on context_len >> shift, 1024 buckets,
// descending) into `order` (with a unit grid: the (sequence, partition)
// units by token count into `units` instead), and zeroes the per-(sequence,
// KV head) partition counters when the decode combines in place.  Launched
// with programmatic stream serialization: it sorts while the previous kernel
// drains (it reads only host-written lengths), then waits for that kernel,
// which may still read `order`, the counters and `units`, before writing
// them.  The decode's own wait covers the prep kernel.  Within one bucket the
// order follows the atomics; results do not depend on it (each unit is
// computed on its own and partials are combined in partition order).
__global__ void __launch_bounds__(kOrderThreads)
    prep_kernel(const int32_t* __restrict__ context_lens, int num_seqs,
                int shift, int32_t* __restrict__ order, int* counters,
                int n_counters, int32_t* __restrict__ units, int max_parts,
                int partition_size, int unit_shift) {
  dev::pdl_trigger();
  if (units) {
    // Partition units by token count, largest first: unit u is partition
    // u % max_parts of sequence u / max_parts (empty past the sequence).
    // The unit grid does not read `order`.
    counting_sort_desc(
        num_seqs * max_parts,
        [&](int u) {
          const int b = u / max_parts;
          const int p = u - b * max_parts;
          const int left = context_lens[b] - p * partition_size;
          const int n = left <= 0 ? 0 : min(left, partition_size);
          return n >> unit_shift;
        },
        units, [] { dev::pdl_wait(); });
  } else {
    sort_longest_first(context_lens, num_seqs, shift, order,
                       [] { dev::pdl_wait(); });
  }
  for (int i = threadIdx.x; i < n_counters; i += kOrderThreads)
    counters[i] = 0;
}

// ---------------------------------------------------------------------------
// Partition reduce: out = sum_j w_j o_j / sum_j w_j, w_j = l_j 2^(m_j - M),
// M = max_j m_j (all in base-2 units).
// One CTA per (query head, sequence); warp w folds partitions w, w+8, ...
// with a running max, sixteen partitions in flight per warp (eight at
// head_dim 64; one 16- or 8-byte load per lane each), and the eight warp
// states are merged through shared memory.  The partials were just written
// by the decode and are read once, so the time is the latency of a few
// rounds of loads: 128 partitions in flight per CTA keep that to one or two
// rounds for the longest sequences, and 256 threads let two CTAs share an SM
// (the grid, one CTA per query head and sequence, is a few waves).  Used
// when a sequence has many partitions (the fused combine handles few).
constexpr int kReduceWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
    reduce_kernel(const DecodeArgs a, int block_size) {
  constexpr int kPer = D / 32;  // dims per lane
  __shared__ float s_m[kReduceWarps], s_w[kReduceWarps];
  __shared__ float s_acc[kReduceWarps][D];
  const int qh = blockIdx.x;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  dev::pdl_trigger();
  const int ctx = a.context_lens[b];
  if (ctx < 0 || ctx > a.max_blocks_per_seq * block_size ||
      ctx > a.max_context_len)
    return;  // flagged by the decode kernel
  const int n_parts = ctx > 0 ? (ctx + a.partition_size - 1) / a.partition_size
                              : 1;
  if (n_parts <= 1) return;  // the decode kernel wrote this row itself
  dev::pdl_wait();           // partials of the decode kernel are visible

  const int64_t row0 =
      (static_cast<int64_t>(b) * a.num_q_heads + qh) * a.max_parts;
  const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + row0;
  const float* o = a.ws_o + row0 * D + lane * kPer;
  float M = -INFINITY, W = 0.f;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  // partitions in flight per warp (head_dim 64: 8, which needs no spill)
  constexpr int kBatch = kPer == 4 ? 16 : 8;
  static_assert(kPer == 4 || kPer == 2, "head_dim 128 or 64");
  for (int j0 = warp; j0 < n_parts; j0 += kBatch * kReduceWarps) {
    float2 mlj[kBatch];
    float oj[kBatch][kPer];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u * kReduceWarps;
      mlj[u] = j < n_parts ? __ldcg(ml + j) : make_float2(-INFINITY, 0.f);
      // this lane's kPer consecutive dims: one 16- (or 8-) byte load; a
      // partial row is D floats, 16-byte aligned
      const float* src = o + static_cast<int64_t>(j) * D;
      if constexpr (kPer == 4) {
        const float4 v = j < n_parts
                             ? __ldcg(reinterpret_cast<const float4*>(src))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        oj[u][0] = v.x;
        oj[u][1] = v.y;
        oj[u][2] = v.z;
        oj[u][3] = v.w;
      } else {
        const float2 v = j < n_parts
                             ? __ldcg(reinterpret_cast<const float2*>(src))
                             : make_float2(0.f, 0.f);
        oj[u][0] = v.x;
        oj[u][1] = v.y;
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (mlj[u].x == -INFINITY) continue;  // empty or skipped partition
      if (mlj[u].x > M) {
        const float sc = dev::fast_exp2(M - mlj[u].x);  // 0 when M = -inf
        W *= sc;
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] *= sc;
        M = mlj[u].x;
      }
      const float w = mlj[u].y * dev::fast_exp2(mlj[u].x - M);
      W += w;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += w * oj[u][e];
    }
  }
  if (lane == 0) {
    s_m[warp] = M;
    s_w[warp] = W;
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) s_acc[warp][lane * kPer + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += kReduceWarps * 32) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) mx = fmaxf(mx, s_m[w]);
    float tw = 0.f, tv = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kReduceWarps; ++w) {
        const float sc =
            s_m[w] == -INFINITY ? 0.f : dev::fast_exp2(s_m[w] - mx);
        tw += s_w[w] * sc;
        tv += s_acc[w][d] * sc;
      }
    }
    store_out<T>(a, (static_cast<int64_t>(b) * a.num_q_heads + qh) * D + d,
                 tw > 0.f ? tv / tw : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Host side.

// The cache viewed as a 2-D tensor of rows (block, kv head, slot) x head_dim;
// one TMA box is block_size rows x 64 elements (128 bytes), swizzled.
bool encode_cache_map(CUtensorMap* map, const void* base, uint64_t rows,
                      int head_dim, int block_size, pa_dtype dtype) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(block_size)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map,
                   dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

#ifndef PAGEDKV_RING_BYTES
#define PAGEDKV_RING_BYTES 65536
#endif
#ifndef PAGEDKV_PDL
#define PAGEDKV_PDL 1  // programmatic dependent launch between the kernels
#endif
constexpr int kUsePdl = PAGEDKV_PDL;
constexpr int stages_for(int bs, int d) {
  // 64 KB ring per CTA: three CTAs fit one SM's shared memory.  Whole
  // multiples of the consumer count (see Geometry).
  return (PAGEDKV_RING_BYTES / (2 * 2 * bs * d)) / kConsumers * kConsumers;
}

int resolve_partition(const pa_decode_desc* d, int max_ctx) {
  if (d->partition_size > 0) return d->partition_size;
  const int64_t pairs = static_cast<int64_t>(d->num_seqs) * d->num_kv_heads;
  const int64_t target = 3LL * device_sm_count();
  // Long partitions (fewer CTAs, less ramp-up and fewer partials) as long as
  // the grid keeps at least 6 units per SM were every sequence max_ctx long;
  // the prep kernel's longest-first order keeps the tail short.  Measured:
  // 4096 is best on the batch-256 and 8-sequence long-context mixes, 2048 on
  // the batch-64 mix (8192 loses everywhere).
  for (int big = 4096; big >= 2048; big /= 2)
    if (pairs * ((max_ctx + big - 1) / big) >= 6LL * device_sm_count() &&
        big % d->block_size == 0)
      return big;
  int ps = 1024;
  while (ps > 2 * d->block_size && ps > 64 &&
         pairs * ((max_ctx + ps - 1) / ps) < target)
    ps /= 2;
  if (ps < d->block_size) ps = d->block_size;
  return ps;
}

int resolve_max_ctx(const pa_decode_desc* d) {
  return d->max_context_len > 0 ? d->max_context_len
                                : d->max_blocks_per_seq * d->block_size;
}

pa_status check_desc(const pa_decode_desc* d) {
  if (!d) return fail(PA_ERR_INVALID_ARG, "pa_decode: desc is NULL");
  if (d->num_seqs < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
      d->max_blocks_per_seq <= 0 || d->num_blocks < 0 ||
      d->max_context_len < 0 || d->partition_size < 0)
    return fail(PA_ERR_INVALID_ARG,
                "pa_decode: num_seqs=%d num_q_heads=%d num_kv_heads=%d "
                "max_blocks_per_seq=%d num_blocks=%d max_context_len=%d "
                "partition_size=%d", d->num_seqs, d->num_q_heads,
                d->num_kv_heads, d->max_blocks_per_seq, d->num_blocks,
                d->max_context_len, d->partition_size);
  if (d->num_q_heads % d->num_kv_heads)
    return fail(PA_ERR_INVALID_ARG,
                "pa_decode: num_q_heads %d is not a multiple of num_kv_heads %d",
                d->num_q_heads, d->num_kv_heads);
  if (d->num_q_heads / d->num_kv_heads > kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: group size %d > %d",
                d->num_q_heads / d->num_kv_heads, kMaxGroup);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: head_dim %d not in {64, 128}",
                d->head_dim);
  if (d->block_size != 16 && d->block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: block_size %d not in {16, 32}",
                d->block_size);
  if (d->dtype != PA_F16 && d->dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: dtype %d",
                static_cast<int>(d->dtype));
  if (d->reduce != PA_REDUCE_AUTO && d->reduce != PA_REDUCE_KERNEL)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: reduce %d",
                static_cast<int>(d->reduce));
  if (d->out_fp32 != 0 && d->out_fp32 != 1)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: out_fp32 %d", d->out_fp32);
  if (d->kernel != PA_KERNEL_AUTO && d->kernel != PA_KERNEL_SIMT &&
      d->kernel != PA_KERNEL_MMA)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: kernel %d",
                static_cast<int>(d->kernel));
  if (d->partition_size > 0 &&
      (d->partition_size % d->block_size || d->partition_size > kMaxPartition))
    return fail(PA_ERR_INVALID_ARG,
                "pa_decode: partition_size %d must be a multiple of block_size "
                "%d and <= %d", d->partition_size, d->block_size,
                kMaxPartition);
  if (static_cast<int64_t>(d->max_blocks_per_seq) * d->block_size >
      0x7fffffffLL)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: max_blocks_per_seq too large");
  if (static_cast<int64_t>(d->num_blocks) * d->num_kv_heads * d->block_size >
      0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED,
                "pa_decode: num_blocks * num_kv_heads * block_size exceeds "
                "2^31 rows");
  if (d->num_seqs > 65535 || d->num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED,
                "pa_decode: num_seqs and num_kv_heads must be <= 65535");
  return PA_OK;
}

// Workspace layout, in bytes from the start: partials o and (m, l) and the
// partition counters (only with more than one partition), then the sequence
// order; each piece 16-byte aligned.
struct WsLayout {
  size_t o = 0, ml = 0, counters = 0, units = 0, order = 0, total = 0;
};

WsLayout ws_layout(const pa_decode_desc* d) {
  auto up16 = [](size_t x) { return (x + 15) & ~size_t(15); };
  const int max_ctx = resolve_max_ctx(d);
  const int ps = resolve_partition(d, max_ctx);
  const int64_t parts = max_ctx > 0 ? (max_ctx + ps - 1) / ps : 1;
  WsLayout w;
  size_t at = 0;
  if (parts > 1) {
    const size_t rows = static_cast<size_t>(d->num_seqs) * d->num_q_heads *
                        static_cast<size_t>(parts);
    w.o = at;
    at += up16(rows * d->head_dim * sizeof(float));
    w.ml = at;
    at += up16(rows * 2 * sizeof(float));
    w.counters = at;
    at += up16(static_cast<size_t>(d->num_seqs) * d->num_kv_heads *
               sizeof(int));
    w.units = at;
    at += up16(static_cast<size_t>(d->num_seqs) * static_cast<size_t>(parts) *
               sizeof(int32_t));
  }
  w.order = at;
  at += up16(static_cast<size_t>(d->num_seqs) * sizeof(int32_t));
  w.total = at;
  return w;
}

size_t workspace_bytes(const pa_decode_desc* d) { return ws_layout(d).total; }


// Combine partitions inside the decode kernel (few partitions) or with the
// separate reduce kernel.
bool use_fused(const pa_decode_desc* d, int parts) {
  return d->reduce == PA_REDUCE_AUTO && parts <= kFusedMaxParts;
}

template <typename T, int BS, int D, bool kMma>
pa_status launch(const pa_decode_desc* d, DecodeArgs& a, const CUtensorMap& km,
                 const CUtensorMap& vm, cudaStream_t stream) {
  constexpr int S = stages_for(BS, D);
  auto kern = decode_kernel<T, BS, D, S, kMma>;
  const size_t smem = smem_bytes_for<BS, D, S, kMma>(
      (a.warp_parts ? kConsumers : 1) * a.partition_size / BS);
  int dev = 0;
  cudaGetDevice(&dev);
  static bool configured[64] = {false};
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
        static_cast<int>(smem_bytes_for<BS, D, S, kMma>(kMaxPartition / BS)));
    if (e != cudaSuccess)
      return fail(PA_ERR_CUDA, "pa_decode: cudaFuncSetAttribute: %s",
                  cudaGetErrorString(e));
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  // Every kernel here (the prep, the decode, the reduce) is
  // launched with programmatic stream serialization: each may start while
  // its predecessor drains and waits (griddepcontrol.wait) before touching
  // memory the predecessor writes.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = kUsePdl;
  {
    const int n = (a.max_parts > 1 && a.fused)
                      ? d->num_seqs * d->num_kv_heads
                      : 0;
    cudaLaunchConfig_t pcfg = {};
    pcfg.gridDim = dim3(1);
    pcfg.blockDim = dim3(kOrderThreads);
    pcfg.stream = stream;
    pcfg.attrs = attr;
    pcfg.numAttrs = 1;
    const cudaError_t pe = cudaLaunchKernelEx(
        &pcfg, prep_kernel, a.context_lens, d->num_seqs,
        order_shift(a.max_context_len), const_cast<int32_t*>(a.order),
        a.counters, n, const_cast<int32_t*>(a.units), a.max_parts,
        a.partition_size, order_shift(a.partition_size));
    count_launch();
    if (pe != cudaSuccess)
      return fail(PA_ERR_CUDA, "pa_decode: prep launch failed: %s",
                  cudaGetErrorString(pe));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim =
      a.units ? dim3(d->num_kv_heads, d->num_seqs * a.max_parts, 1)
              : dim3(a.warp_parts ? (a.max_parts + kConsumers - 1) / kConsumers
                                  : a.max_parts,
                     d->num_kv_heads, d->num_seqs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, a);
  count_launch();
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_decode: decode launch failed: %s",
                cudaGetErrorString(e));
  if (a.max_parts > 1 && !a.fused) {
    cudaLaunchConfig_t rcfg = {};
    rcfg.gridDim = dim3(d->num_q_heads, d->num_seqs);
    rcfg.blockDim = dim3(kReduceWarps * 32);
    rcfg.dynamicSmemBytes = 0;
    rcfg.stream = stream;
    rcfg.attrs = attr;
    rcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&rcfg, reduce_kernel<T, D>, a, BS);
    count_launch();
    if (e != cudaSuccess)
      return fail(PA_ERR_CUDA, "pa_decode: reduce launch failed: %s",
                  cudaGetErrorString(e));
  }
  return PA_OK;
}

template <typename T, bool kMma>
pa_status dispatch_shape(const pa_decode_desc* d, DecodeArgs& a,
                         const CUtensorMap& km, const CUtensorMap& vm,
                         cudaStream_t st) {
  if (d->block_size == 16)
    return d->head_dim == 128 ? launch<T, 16, 128, kMma>(d, a, km, vm, st)
                              : launch<T, 16, 64, kMma>(d, a, km, vm, st);
  return d->head_dim == 128 ? launch<T, 32, 128, kMma>(d, a, km, vm, st)
                            : launch<T, 32, 64, kMma>(d, a, km, vm, st);
}

// The built-in scratch's device address belongs to a CUDA context, not to a
// device ordinal: after cudaDeviceReset, or under a context the caller made
// current through the driver API, the module is loaded again and the array
// may sit elsewhere.  So the cache is keyed on the current context's unique
// id (cuCtxGetId, never reused within a process), filled under a mutex.
using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault,
                                       &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(p);
  return nullptr;
}

// Unique id of the calling thread's current context; false if there is none.
bool current_context_id(unsigned long long* id) {
  static const PFN_ctxGetCurrent get_current =
      driver_fn<PFN_ctxGetCurrent>("cuCtxGetCurrent");
  static const PFN_ctxGetId get_id = driver_fn<PFN_ctxGetId>("cuCtxGetId");
  CUcontext ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

void* scratch_address(pa_status* st) {
  struct Entry {
    unsigned long long ctx_id;
    void* addr;
  };
  constexpr int kMaxEntries = 64;
  static std::mutex mu;
  static Entry cache[kMaxEntries];
  static int used = 0;
  unsigned long long id = 0;
  if (current_context_id(&id)) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (cache[i].ctx_id == id) {
        *st = PA_OK;
        return cache[i].addr;
      }
  }
  // First call in this context (or no context yet: the runtime creates the
  // device's primary context here).
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, ::g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    *st = fail(PA_ERR_CUDA,
               "pa_decode_noalloc: cudaGetSymbolAddress of the built-in "
               "scratch failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if (current_context_id(&id)) {
    std::lock_guard<std::mutex> lock(mu);
    bool known = false;
    for (int i = 0; i < used; ++i) known |= cache[i].ctx_id == id;
    if (!known && used < kMaxEntries) cache[used++] = Entry{id, p};
  }
  *st = PA_OK;
  return p;
}

}  // namespace
}  // namespace pagedkv

using pagedkv::fail;

extern "C" {

pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, float scale,
                            const pa_decode_desc* desc, int32_t* dev_err,
                            void* stream) {
  pagedkv::clear_error();
  pa_status st = pagedkv::check_desc(desc);
  if (st != PA_OK) return st;
  const size_t need = pagedkv::workspace_bytes(desc);
  if (need > PA_NOALLOC_SCRATCH_BYTES)
    return fail(PA_ERR_WORKSPACE,
                "pa_decode_noalloc: this shape needs %zu bytes of scratch but "
                "the built-in area holds %llu; use a larger partition_size, "
                "fewer sequences, or pa_decode with a caller workspace", need,
                static_cast<unsigned long long>(PA_NOALLOC_SCRATCH_BYTES));
  void* scratch = pagedkv::scratch_address(&st);
  if (st != PA_OK) return st;
  return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens,
                   scale, desc, scratch, PA_NOALLOC_SCRATCH_BYTES, dev_err,
                   stream);
}

size_t pa_decode_workspace_bytes(const pa_decode_desc* desc) {
  pagedkv::clear_error();
  if (pagedkv::check_desc(desc) != PA_OK) return 0;
  return pagedkv::workspace_bytes(desc);
}

int pa_decode_partition_size(const pa_decode_desc* desc) {
  pagedkv::clear_error();
  if (pagedkv::check_desc(desc) != PA_OK) return -1;
  return pagedkv::resolve_partition(desc, pagedkv::resolve_max_ctx(desc));
}

pa_status pa_decode(void* out, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables,
                    const int32_t* context_lens, float scale,
                    const pa_decode_desc* desc, void* workspace,
                    size_t workspace_bytes, int32_t* dev_err, void* stream) {
  pagedkv::clear_error();
  pa_status st = pagedkv::check_desc(desc);
  if (st != PA_OK) return st;
  if (!std::isfinite(scale))
    return fail(PA_ERR_INVALID_ARG, "pa_decode: scale is not finite");
  if (desc->num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: NULL tensor pointer");
  if (!pagedkv::aligned16(out) || !pagedkv::aligned16(q) ||
      !pagedkv::aligned16(k_cache) || !pagedkv::aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG,
                "pa_decode: out, q and the caches must be 16-byte aligned");
  if (desc->num_blocks == 0)
    return fail(PA_ERR_INVALID_ARG, "pa_decode: empty block pool");

  const int max_ctx = pagedkv::resolve_max_ctx(desc);
  const int ps = pagedkv::resolve_partition(desc, max_ctx);
  const int parts = max_ctx > 0 ? (max_ctx + ps - 1) / ps : 1;
  if (parts > pagedkv::kMaxParts)
    return fail(PA_ERR_UNSUPPORTED,
                "pa_decode: %d partitions of %d tokens exceed %d; use a "
                "larger partition_size", parts, ps, pagedkv::kMaxParts);
  const size_t need = pagedkv::workspace_bytes(desc);
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   !pagedkv::aligned16(workspace)))
    return fail(PA_ERR_WORKSPACE,
                "pa_decode: workspace of %zu bytes (16-byte aligned) needed, "
                "got %zu at %p", need, workspace_bytes, workspace);

  CUtensorMap kmap, vmap;
  const uint64_t rows = static_cast<uint64_t>(desc->num_blocks) *
                        desc->num_kv_heads * desc->block_size;
  if (!pagedkv::encode_cache_map(&kmap, k_cache, rows, desc->head_dim,
                                 desc->block_size, desc->dtype) ||
      !pagedkv::encode_cache_map(&vmap, v_cache, rows, desc->head_dim,
                                 desc->block_size, desc->dtype))
    return fail(PA_ERR_CUDA, "pa_decode: cuTensorMapEncodeTiled failed");

  pagedkv::DecodeArgs a;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  const pagedkv::WsLayout wl = pagedkv::ws_layout(desc);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.ws_o = parts > 1 ? reinterpret_cast<float*>(ws + wl.o) : nullptr;
  a.ws_ml = parts > 1 ? reinterpret_cast<float*>(ws + wl.ml) : nullptr;
  a.counters = parts > 1 ? reinterpret_cast<int*>(ws + wl.counters) : nullptr;
  a.order = reinterpret_cast<const int32_t*>(ws + wl.order);
  a.fused = pagedkv::use_fused(desc, parts) ? 1 : 0;
  // Short partitions combined by the reduce kernel: one partition per
  // consumer warp, kConsumers per CTA (fewer, longer CTAs; no merge).
  a.warp_parts = (desc->kernel != PA_KERNEL_SIMT && !a.fused && parts > 1 &&
                  ps <= pagedkv::kWarpPartsMaxPartition)
                     ? 1
                     : 0;
  a.dev_err = dev_err;
  a.scale_log2 = scale * pagedkv::kLog2e;
  a.num_q_heads = desc->num_q_heads;
  a.num_kv_heads = desc->num_kv_heads;
  a.group = desc->num_q_heads / desc->num_kv_heads;
  a.max_blocks_per_seq = desc->max_blocks_per_seq;
  a.num_blocks = desc->num_blocks;
  a.partition_size = ps;
  a.max_parts = parts;
  a.max_context_len = max_ctx;
  a.out_f32 = desc->out_fp32;
  // Long partitions, one per CTA, in a grid of a few waves: the grid runs
  // (KV head, unit) with the units longest first, so the last CTAs hold the
  // shortest partitions.  Ordered by sequence instead, the second wave can
  // start full-length partitions of mid-length sequences and end on a long
  // tail (batch 64 at 2048-token partitions: 6.12 -> 6.24 TB/s).  With many
  // waves the sequence order already ends on short work, and with short
  // partitions the extra sort in the prep kernel costs more than the tail
  // (gridDim.y caps the unit count).
  const int64_t n_units = static_cast<int64_t>(desc->num_seqs) * parts;
  a.units = (parts > 1 && !a.warp_parts && ps >= 1024 && n_units <= 65535 &&
             // at most four waves of three CTAs per SM
             n_units * desc->num_kv_heads <= 12LL * pagedkv::device_sm_count())
                ? reinterpret_cast<const int32_t*>(ws + wl.units)
                : nullptr;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool mma = desc->kernel != PA_KERNEL_SIMT;
  if (desc->dtype == PA_BF16)
    return mma ? pagedkv::dispatch_shape<__nv_bfloat16, true>(desc, a, kmap,
                                                              vmap, s)
               : pagedkv::dispatch_shape<__nv_bfloat16, false>(desc, a, kmap,
                                                               vmap, s);
  return mma ? pagedkv::dispatch_shape<__half, true>(desc, a, kmap, vmap, s)
             : pagedkv::dispatch_shape<__half, false>(desc, a, kmap, vmap, s);
}

}  // extern "C"
