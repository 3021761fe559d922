// pa_prefill: causal attention of each sequence's new tokens over its paged
// K/V cache, on the 5th-generation tensor cores (tcgen05, tensor memory).
//
// What is computed: for sequence b with L = context_lens[b] tokens cached, of
// which the last q_len are new (query rows query_start[b] .. +q_len), new
// token i at position p = L - q_len + i attends to positions 0 .. p with the
// scores and softmax of contiguous attention ([vLLM PagedAttention FAQ] "Does
// PagedAttention change the mathematical attention output?").  q_len = L is a
// whole prompt, q_len < L a chunk of one; a few new tokens at once is how a
// target model checks speculative draft tokens ([Taming the Tail] "The
// Future: Speculative Decoding and Beyond"); the attention is tiled as
// [KV-cache chapter] "Common misconception..." describes serving kernels
// doing: FlashAttention-style tiles over paged memory.
//
// B200 design.  Work item = (tile of 128 query rows, KV head, sequence); a
// row is a (new token, query head of this KV head) pair, so with G query heads
// per KV head a tile holds 128/G tokens and each K/V byte serves all G heads.
//   * A one-CTA plan kernel sorts the sequences longest context first and
//     lists their query tiles in that order (each sequence's last tile, the
//     one that sees the most keys, first).  The prefill grid is persistent,
//     two CTAs per SM: each takes (listed tile, KV head) items from a
//     counter, heaviest first, so the CTAs end together.
//   * Warp 0, lane 0 takes the items and publishes each to the other warps
//     through a two-slot ring in shared memory.  It loads an item's Q tile
//     with one 3-D TMA box per half of head_dim (once the previous item's S
//     MMAs are done with the buffer), then streams 64-key K and V tiles page
//     by page (2-D TMA boxes
//     of block_size rows x 128 B, 128-byte swizzle, no multicast) into
//     separate 2-stage K and V rings: a K stage is free again once S(j) has
//     read it, a V stage once P(j).V has, and V tile j is loaded after K
//     tile j+1 since it is needed a tile later.  Pages are placed so that a
//     tile is the canonical 128-byte-swizzled layout the tensor core reads.
//   * Warp 1 allocates 256 tensor-memory columns (S 64, P 64, O 128); its
//     lane 0 issues S = Q K^T (M=128, N=64, both operands in shared memory)
//     and O += P V (M=128, N=128; P read from tensor memory, V from shared
//     memory, MN-major) as tcgen05.mma with fp32 accumulators, and signals
//     completion with tcgen05.commit.  S and P have buffers of their own:
//     S(j+1) is issued as soon as the softmax warps hold S(j) in registers,
//     so it is ready when they finish tile j, and the softmax stores P(j+1)
//     once P(j).V has read the P buffer.  (With P written over the S it came
//     from, S(j+2) had to wait for P(j).V, and that round trip set half of
//     every tile's period.)
//   * Warps 2..5 own one tensor-memory row each (thread = query row): they
//     read S with tcgen05.ld, apply the causal mask (diagonal tiles only),
//     keep the online softmax in registers (no shuffles: a row is one
//     thread), rescale O in tensor memory only when the running maximum
//     grows by more than 2^8 (the final division uses the same reference,
//     so the result is unchanged), and store P with tcgen05.st as 16-bit
//     values.  In the tiles where some row may end with a key of weight
//     above 1/16 they also store P's residual (P minus its rounding), and a
//     second MMA adds residual . V, so those weights keep ~16 bits.
//   * With at most 64 query rows per KV head (a few new tokens), a
//     compile-time variant spreads the rows over all four softmax warps,
//     8 or 16 per lane quarter, and reads S / writes P / reads O with the
//     16-lane tensor-memory shapes: four threads per row, 16 keys each.  A
//     warp whose rows are all padding computes nothing.  Its MMAs use
//     M = 64 (half the tensor work), whose accumulator rows 16q + i sit in
//     lanes 32q + i, and the 16 KB of Q this frees holds a third V stage.
//   * Shared memory is ~99 KB (Q, the rings, barriers; block ids are read
//     from global memory a tile ahead) and tensor memory 256 columns, so two
//     CTAs share an SM at any context length: one CTA's softmax runs while
//     the other's tiles are on the tensor cores.
//   * Barrier phases count a CTA's tiles over all its items, so the next
//     item's Q, first K tiles and first S are in flight while the current
//     item's last tiles and output are computed: the CTA start and the gap
//     between CTAs are paid once per SM slot, not once per query tile.
//   * Every wait is bounded (1 s) and reports PA_ERR_DEVICE_TIMEOUT; tensor
//     memory is always released.  A barrier that is waited on by parity is
//     never allowed to run two phases ahead of its waiter: each double
//     buffer has its own barriers, and a buffer is refilled only after its
//     consumer has observed the previous fill.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "device_utils.cuh"
#include "order.cuh"
#include "pagedkv.h"
#include "status.h"
#include "tcgen05_ts.cuh"

namespace pagedkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRows = 128;      // query rows per tile (tensor memory lanes)
constexpr int kKeys = 64;       // keys per K/V tile
// Ring depths and Q rows per layout.  Tiles of 128 query rows: two K and
// two V stages.  The few-row layouts (M = 64 MMAs, a 64-row Q operand)
// stream K/V at HBM speed; the 16 KB their Q operand does not need holds a
// third V stage (a V stage is held longest: until P.V, after the softmax).
template <int RQ> __host__ __device__ constexpr int k_stages() { return 2; }
template <int RQ> __host__ __device__ constexpr int v_stages() {
  return RQ > 0 ? 3 : 2;
}
template <int RQ> __host__ __device__ constexpr int q_rows() {
  return RQ > 0 ? 64 : 128;
}
constexpr int kThreads = 192;   // producer, MMA, 4 softmax warps
constexpr int kTmemCols = 256;  // S [0, 64), P [64, 128), O [128, 128 + D)
constexpr float kRescaleLog2 = 8.f;
// P . V runs on 16-bit P.  A single rounding of P moves each weight by up to
// 2^-8 of itself (bf16), which on a row whose weight sits on a few keys can
// move the output by more than the 2e-3 tolerance.  So P is also split into a
// rounded part and its residual, and a second MMA adds residual . V, for every
// tile in which some row has a key with p > l / kSplitInv, where l is the
// row's running sum including this tile: such a key's final weight may exceed
// 1/kSplitInv.  Keys of the other tiles each end with a weight below
// 1/kSplitInv, and their rounding errors, of either sign, average out.
constexpr float kSplitInv = 16.f;

// Tensor-memory access shapes with four threads per lane, used when at most
// 32 query rows are real.  16x256b: thread t gets lanes t/4 and t/4 + 8 of
// the 16 addressed, columns 2 (t % 4) and 2 (t % 4) + 1 of every 8 (the
// layout of an m16n8 accumulator).  16x128b: the same lanes, column t % 4 of
// every 4.
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr,
                                                 float (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
      "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]),
        "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]), "=f"(v[9]),
        "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]),
        "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]),
        "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]),
        "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]),
        "=f"(v[30]), "=f"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16x256_x4(uint32_t taddr,
                                                 float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]),
        "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]), "=f"(v[9]),
        "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]),
        "=f"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16x256_x4(uint32_t taddr,
                                                 const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%16], {%0, %1, %2, %3, %4, "
      "%5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15};" ::"f"(v[0]),
      "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
      "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]),
      "f"(v[13]), "f"(v[14]), "f"(v[15]), "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16x128_x8(uint32_t taddr,
                                                 const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%16], {%0, %1, %2, %3, %4, "
      "%5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15};" ::"r"(v[0]),
      "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
      "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
      "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(taddr)
      : "memory");
}

struct PrefillArgs {
  void* out;
  const int2* tiles;  // tile map: (sequence, query tile) per grid row
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;
  int32_t* dev_err;
  float scale_log2;
  int num_q_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int num_blocks;
  int max_context_len;
  int total_q;
  int out_f32;  // 1: out is float32 (the value before the cast to T)
  int pv_split;  // pa_prefill_pv: 0 per tile as needed, 1 always, 2 never
  int* counter;   // next work item (zeroed by the plan kernel)
  int num_items;  // tile-map entries x KV heads
};

// barriers: q_full, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV],
// s_full, s_free, p_full, o_ready, done, q_empty, item_full[2],
// item_empty[2]; then the tensor-memory base address word, the residual vote
// and (16 bytes on) two work-item slots.
template <int KS, int VS> __host__ __device__ constexpr int num_bars() {
  return 1 + 2 * KS + 2 * VS + 4 + 1 + 1 + 4;
}
constexpr int kItemWords = 8;  // one published work item
constexpr int kTileHalf = kKeys * 128;  // 8 KB: 64 keys x 64 dims (128 B)

// Shared memory for head_dim D (offsets from a 1024-byte aligned base): the
// head dimension is held in 64-element halves of 128 bytes, each its own
// 128-byte-swizzled region.
template <int D, int QR, int KS, int VS>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfQ = QR * 128;                 // 16 or 8 KB
  static constexpr int kQBytes = kHalves * kHalfQ;
  static constexpr int kKVTile = kHalves * kTileHalf;     // per K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + KS * kKVTile;
  static constexpr int kOffBars = kOffV + VS * kKVTile;
  // 1024 bytes of slack for aligning the base, then the layout above; after
  // the barriers, the tensor-memory address word and the residual vote (16
  // bytes with padding) and two work-item slots.
  static constexpr size_t kSmemBytes =
      1024 + kOffBars + num_bars<KS, VS>() * 8 + 16 + 2 * kItemWords * 4;
};
template <int D, int RQ>
using LayoutFor = Layout<D, q_rows<RQ>(), k_stages<RQ>(), v_stages<RQ>()>;

template <typename T, int BS, int G, int D, int RQ>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap,
                   const PrefillArgs a) {
  using Lay = LayoutFor<D, RQ>;
  constexpr int kKStages = k_stages<RQ>();
  constexpr int kVStages = v_stages<RQ>();
  constexpr int kNumBars = num_bars<kKStages, kVStages>();
  constexpr int kHalves = Lay::kHalves;
  constexpr int kHalfQ = Lay::kHalfQ;
  constexpr int kQBytes = Lay::kQBytes;
  constexpr int kKVTile = Lay::kKVTile;
  constexpr int kOffBars = Lay::kOffBars;
  constexpr int kTok = kRows / G;         // new tokens per tile
  constexpr int kPagesPerTile = kKeys / BS;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using M = dev::Mma<T>;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem =
      smem_dyn + ((1024u - (dev::smem_u32(smem_dyn) & 1023u)) & 1023u);
  const uint32_t base = dev::smem_u32(smem);
  const uint32_t q_s = base + Lay::kOffQ;
  const uint32_t kring = base + Lay::kOffK;
  const uint32_t vring = base + Lay::kOffV;
  const uint32_t bars = base + kOffBars;
  const uint32_t q_full = bars;
  const uint32_t k_full0 = bars + 8;
  const uint32_t k_empty0 = k_full0 + kKStages * 8;
  const uint32_t v_full0 = k_empty0 + kKStages * 8;
  const uint32_t v_empty0 = v_full0 + kVStages * 8;
  // S, P and P.V barriers, one each: the CTA's tile t (counted over all its
  // work items) completes phase t (waited on with parity t & 1).  s_full:
  // S(t) is in tensor memory; s_free: the softmax warps have S(t) in
  // registers; p_full: P(t) is in tensor memory; o_ready: P(t).V has
  // completed (O is current, the P buffer is free).
  const uint32_t s_full = v_empty0 + kVStages * 8;
  const uint32_t s_free = s_full + 8;
  const uint32_t p_full = s_free + 8;
  const uint32_t o_ready = p_full + 8;
  const uint32_t done = o_ready + 8;
  // q_empty: an item's S MMAs are done with the Q buffer (one phase per
  // computed item).  item_full[s] / item_empty[s]: work-item slot s was
  // published / read by all five consumers (the MMA thread and the four
  // softmax warps).
  const uint32_t q_empty = done + 8;
  const uint32_t item_full0 = q_empty + 8;
  const uint32_t item_empty0 = item_full0 + 16;
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(smem + kOffBars + kNumBars * 8);
  // Residual vote: a softmax warp whose rows need P's residual in tile t
  // stores t + 1 into the word before it arrives on p_full, and the MMA
  // issuer reads it after that barrier; a stale word holds t or less, so it
  // never needs clearing.
  volatile uint32_t* pv_vote = tmem_slot + 1;
  volatile int* item_s = reinterpret_cast<volatile int*>(tmem_slot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  dev::pdl_trigger();  // the next call's plan kernel may start its reads
  if (tid == 0) {
    dev::mbar_init(q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      dev::mbar_init(k_full0 + 8 * s, 1);
      dev::mbar_init(k_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      dev::mbar_init(v_full0 + 8 * s, 1);
      dev::mbar_init(v_empty0 + 8 * s, 1);
    }
    dev::mbar_init(s_full, 1);
    dev::mbar_init(s_free, 4);
    dev::mbar_init(p_full, 4);
    dev::mbar_init(o_ready, 1);
    dev::mbar_init(done, 4);
    dev::mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      dev::mbar_init(item_full0 + 8 * s, 1);
      dev::mbar_init(item_empty0 + 8 * s, 5);
    }
    dev::fence_mbar_init();
    pv_vote[0] = 0u;
  }
  if (warp == 1) {  // the whole warp allocates tensor memory
    dev::tmem_alloc(dev::smem_u32(tmem_slot), kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // S: columns [0, 64); P: columns [64, 128) (rounded part in the first 32,
  // residual in the next 32, two 16-bit values per column); O: columns
  // [128, 256).  S and P have buffers of their own, so S(t+1) can be
  // computed as soon as the softmax warps hold S(t) in registers, without
  // waiting for P(t).V (which only P's buffer holds up).
  const uint32_t s_tmem = tbase;
  const uint32_t p_tmem = tbase + kKeys;
  const uint32_t o_tmem = tbase + 128;
  // The tile map and the item counter come from the plan kernel, which this
  // grid follows by programmatic launch.
  dev::pdl_wait();

  // The grid is persistent: two CTAs per SM, each taking work items from a
  // counter in the workspace.  Item i is KV head i % num_kv_heads of tile-
  // map entry i / num_kv_heads; the map lists the sequences longest context
  // first and each sequence's query tiles from its last one, which sees the
  // most keys (the causal triangle), so items are taken heaviest first and
  // the CTAs end together whatever the mix of tile lengths.  The producer
  // takes each item and publishes it to the other warps through a two-slot
  // ring; the next item's Q tile, first K tiles and first S are in flight
  // while the current item's last tiles and output are computed.
  struct Item {
    int state;  // kWork, kSkip (invalid input, flagged) or kEnd
    int b, kvh, qt, L, q0, q_len;
  };
  constexpr int kWork = 0, kSkip = 1, kEnd = 2;
  // What an item computes: new tokens tok0 .. tok0 + n_q - 1 of its
  // sequence, over keys [0, kv_end) in n_tiles tiles of 64.
  struct Span {
    int tok0, n_q, kv_end, n_tiles;
  };
  auto span_of = [](const Item& it) {
    Span sp;
    sp.tok0 = it.qt * kTok;
    sp.n_q = min(kTok, it.q_len - sp.tok0);
    sp.kv_end = it.L - it.q_len + sp.tok0 + sp.n_q;
    sp.n_tiles = (sp.kv_end + kKeys - 1) / kKeys;
    return sp;
  };
  // Consumers read item n from slot n & 1 once it is published (the
  // barrier's acquire orders the reads after the producer's writes).
  auto read_item = [&](int n, Item& it) -> bool {
    const int slot = n & 1;
    if (!dev::mbar_wait(item_full0 + 8 * slot, (n >> 1) & 1)) return false;
    const volatile int* d = item_s + kItemWords * slot;
    it.state = d[0];
    it.b = d[1];
    it.kvh = d[2];
    it.qt = d[3];
    it.L = d[4];
    it.q0 = d[5];
    it.q_len = d[6];
    return true;
  };

  if (warp == 0) {
    // ---------------- work items and TMA producer ----------------
    if (lane == 0) {
      dev::prefetch_tmap(&qmap);
      dev::prefetch_tmap(&kmap);
      dev::prefetch_tmap(&vmap);
      // Take item n: past the map's last tile (or its end) there is no more
      // work.  A sequence outside the table or the rows, or with more new
      // tokens than the few-row layout holds, is flagged and skipped.
      auto draw = [&](Item& it) {
        it = Item{kEnd, 0, 0, 0, 0, 0, 0};
        // Unsigned: each CTA draws once past the last item, which must not
        // wrap to a negative index however close num_items is to 2^31.
        const unsigned u =
            atomicAdd(reinterpret_cast<unsigned*>(a.counter), 1u);
        if (u >= static_cast<unsigned>(a.num_items)) return;
        const int i = static_cast<int>(u);
        const int2 e = a.tiles[i / a.num_kv_heads];
        if (e.x < 0) return;
        it.b = e.x;
        it.qt = e.y;
        it.kvh = i % a.num_kv_heads;
        it.L = a.context_lens[it.b];
        it.q0 = a.query_start[it.b];
        it.q_len = a.query_start[it.b + 1] - it.q0;
        const bool bad =
            it.L < 0 || it.L > a.max_blocks_per_seq * BS ||
            it.L > a.max_context_len || it.q_len < 0 || it.q_len > it.L ||
            it.q0 < 0 || it.q0 + it.q_len > a.total_q ||
            it.qt * kTok >= it.q_len || (RQ > 0 && it.q_len * G > 4 * RQ);
        if (bad) dev::set_error(a.dev_err, PA_ERR_DEVICE_OOB);
        it.state = bad ? kSkip : kWork;
      };
      // K tile t and V tile t-1 per step (t counted over the CTA's items): a
      // K stage is free once S(t) has read it, a V stage once P(t).V has,
      // and V is needed a tile later.
      auto load = [&](uint32_t t, bool is_v, int kvh,
                      const int32_t (&ids)[kPagesPerTile]) -> bool {
        const int ns = is_v ? kVStages : kKStages;
        const int s = t % ns;
        const uint32_t empty = (is_v ? v_empty0 : k_empty0) + 8 * s;
        if (t >= static_cast<uint32_t>(ns) &&
            !dev::mbar_wait(empty, ((t / ns) - 1) & 1))
          return false;
        const uint32_t full = (is_v ? v_full0 : k_full0) + 8 * s;
        dev::mbar_arrive_expect_tx(full, kKVTile);
        const uint32_t dst = (is_v ? vring : kring) + s * kKVTile;
        const CUtensorMap* map = is_v ? &vmap : &kmap;
#pragma unroll
        for (int p = 0; p < kPagesPerTile; ++p) {
          const int y = (ids[p] * a.num_kv_heads + kvh) * BS;
          const uint32_t off = p * BS * 128;
#pragma unroll
          for (int h = 0; h < kHalves; ++h)
            dev::tma_load_2d(dst + h * kTileHalf + off, map, 64 * h, y, full);
        }
        return true;
      };
      uint32_t g = 0;  // tiles of this CTA's earlier items
      int v = 0;       // items computed so far
      bool ok = true;
      for (int n = 0; ok; ++n) {
        Item it;
        draw(it);
        const int slot = n & 1;
        if (n >= 2 &&
            !dev::mbar_wait(item_empty0 + 8 * slot, ((n >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        volatile int* d = item_s + kItemWords * slot;
        d[0] = it.state;
        d[1] = it.b;
        d[2] = it.kvh;
        d[3] = it.qt;
        d[4] = it.L;
        d[5] = it.q0;
        d[6] = it.q_len;
        dev::mbar_arrive(item_full0 + 8 * slot);
        if (it.state == kEnd) break;
        if (it.state == kSkip) continue;
        const Span sp = span_of(it);
        const int kvh = it.kvh;
        // The Q buffer is free once the previous item's S MMAs are done.
        if (v >= 1 && !dev::mbar_wait(q_empty, (v - 1) & 1)) {
          ok = false;
          break;
        }
        if constexpr (RQ > 0) {
          // Few query rows: RQ/G tokens of G heads (RQ rows) into the first
          // RQ of each 16-row quarter of the 64-row A operand (the rest is
          // padding).  With M = 64 the tensor cores put row 16q + i of S and
          // O in tensor-memory lane 32q + i, and read P's row 16q + i from
          // that lane: the same lanes the softmax warps use.
          constexpr int kQTok = RQ / G;
          dev::mbar_arrive_expect_tx(q_full, 4 * kHalves * RQ * 128);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
#pragma unroll
            for (int h = 0; h < kHalves; ++h)
              dev::tma_load_3d(q_s + h * kHalfQ + qq * 16 * 128, &qmap,
                               64 * h, kvh * G, it.q0 + sp.tok0 + qq * kQTok,
                               q_full);
        } else {
          dev::mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
          for (int h = 0; h < kHalves; ++h)
            dev::tma_load_3d(q_s + h * kHalfQ, &qmap, 64 * h, kvh * G,
                             it.q0 + sp.tok0, q_full);
        }
        // Block ids of a tile's pages, read a tile ahead of its loads and
        // checked there: an id outside the pool sets PA_ERR_DEVICE_OOB and
        // reads page 0 instead (the item's rows are then unspecified).
        // Pages past the sequence are masked, so they read its first page.
        const int32_t* row = a.block_tables +
                             static_cast<int64_t>(it.b) * a.max_blocks_per_seq;
        const int n_pages = (sp.kv_end + BS - 1) / BS;
        bool bad_id = false;
        auto valid_id = [&](int32_t id) {
          const bool bad = id < 0 || id >= a.num_blocks;
          bad_id |= bad;
          return bad ? 0 : id;
        };
        const int32_t first = valid_id(__ldg(row));
        auto fetch = [&](int j, int32_t (&ids)[kPagesPerTile]) {
#pragma unroll
          for (int p = 0; p < kPagesPerTile; ++p) {
            const int page = j * kPagesPerTile + p;
            ids[p] = page < n_pages ? valid_id(__ldg(row + page)) : first;
          }
        };
        int32_t cur[kPagesPerTile], nxt[kPagesPerTile], prv[kPagesPerTile];
        fetch(0, nxt);
        for (int t = 0; t <= sp.n_tiles; ++t) {
          if (t < sp.n_tiles) {
#pragma unroll
            for (int p = 0; p < kPagesPerTile; ++p) cur[p] = nxt[p];
            if (t + 1 < sp.n_tiles) fetch(t + 1, nxt);  // in flight meanwhile
          }
          if ((t < sp.n_tiles && !load(g + t, false, kvh, cur)) ||
              (t >= 1 && !load(g + t - 1, true, kvh, prv))) {
            ok = false;
            break;
          }
#pragma unroll
          for (int p = 0; p < kPagesPerTile; ++p) prv[p] = cur[p];
        }
        if (bad_id) dev::set_error(a.dev_err, PA_ERR_DEVICE_OOB);
        g += sp.n_tiles;
        ++v;
      }
      if (!ok) dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
    }
    return;
  }

  if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool ok = true;
      // M = 128 query rows per MMA, or 64 in the few-row layouts (at most 16
      // real rows per lane quarter): half the tensor work per tile.
      constexpr int kMmaM = RQ > 0 ? 64 : kRows;
      constexpr uint32_t idesc_qk = dev::umma_idesc_f16(kBf16, kMmaM, kKeys,
                                                        false, false);
      constexpr uint32_t idesc_pv = dev::umma_idesc_f16(kBf16, kMmaM, D,
                                                        false, true);
      // O += P(t).V for the CTA's tile t; an item's first tile overwrites O.
      auto issue_pv = [&](uint32_t t, bool first) -> bool {
        if (!dev::mbar_wait(p_full, t & 1) ||
            !dev::mbar_wait(v_full0 + 8 * (t % kVStages), (t / kVStages) & 1))
          return false;
        dev::tc_fence_after();
        const uint32_t vt = vring + (t % kVStages) * kKVTile;
        const int parts =
            a.pv_split == 1 || (a.pv_split == 0 && pv_vote[0] == t + 1u) ? 2
                                                                         : 1;
        for (int part = 0; part < parts; ++part) {  // P rounded, residual
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            // V as the MN-major B operand: 64-wide d halves kTileHalf apart,
            // 8-key groups 1024 bytes apart.
            const uint64_t bd =
                dev::sw128_desc(vt + kk * 2048, kTileHalf, 1024);
            dev::umma_f16_ts(o_tmem, p_tmem + part * (kKeys / 2) + kk * 8,
                             bd, idesc_pv,
                             (!first || part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        dev::umma_commit(o_ready);
        dev::umma_commit(v_empty0 + 8 * (t % kVStages));
        return true;
      };
      // S(t) = Q K(t)^T, once K(t) has landed and the softmax warps hold
      // S(t-1) in registers; after an item's last S the Q buffer is free.
      auto issue_s = [&](uint32_t t, bool last) -> bool {
        const int s = t % kKStages;
        if (!dev::mbar_wait(k_full0 + 8 * s, (t / kKStages) & 1) ||
            (t >= 1 && !dev::mbar_wait(s_free, (t - 1) & 1)))
          return false;
        dev::tc_fence_after();
        const uint32_t kt = kring + s * kKVTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int h = kk >> 2, k4 = kk & 3;
          const uint64_t ad = dev::sw128_desc(q_s + h * kHalfQ + k4 * 32, 16,
                                              1024);
          const uint64_t bd = dev::sw128_desc(kt + h * kTileHalf + k4 * 32,
                                              16, 1024);
          dev::umma_f16(s_tmem, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        dev::umma_commit(s_full);
        dev::umma_commit(k_empty0 + 8 * s);
        if (last) dev::umma_commit(q_empty);
        return true;
      };
      uint32_t g = 0;  // tiles of this CTA's earlier items
      int v = 0;       // items computed so far
      for (int n = 0; ok; ++n) {
        Item it;
        if (!read_item(n, it)) {
          ok = false;
          break;
        }
        dev::mbar_arrive(item_empty0 + 8 * (n & 1));
        if (it.state == kEnd) break;
        if (it.state == kSkip) continue;
        const int nt = span_of(it).n_tiles;
        // S(j+1) is issued while the softmax works on tile j, before
        // P(j).V, which waits for the softmax.
        ok = dev::mbar_wait(q_full, v & 1) && issue_s(g, nt == 1);
        for (int j = 0; ok && j < nt; ++j) {
          if (j + 1 < nt) ok = issue_s(g + j + 1, j + 2 == nt);
          if (ok) ok = issue_pv(g + j, j == 0);
        }
        g += nt;
        ++v;
      }
      if (ok && g > 0) ok = dev::mbar_wait(o_ready, (g - 1) & 1);
      if (!ok) dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
      // Release tensor memory only after the softmax warps are done with it
      // (they arrive after their last item's output).
      if (!dev::mbar_wait(done, 0))
        dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tbase, kTmemCols);
    return;
  }

  // Softmax warps: each reads every item in turn, like the MMA thread, and
  // writes back its share of the item's output.  Wait results are made
  // warp-uniform: the tcgen05 loads and stores are warp-collective.
  const int quarter = warp & 3;  // tensor-memory lane quarter of this warp
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const float c = a.scale_log2;
  auto wait_pv = [&](uint32_t t) {  // P(t).V has completed
    return __all_sync(0xffffffffu, dev::mbar_wait(o_ready, t & 1));
  };
  auto next_item = [&](int n, Item& it) -> bool {
    if (!__all_sync(0xffffffffu, read_item(n, it))) return false;
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(item_empty0 + 8 * (n & 1));
    return true;
  };
  // Keys past the context get P = 0, but 0 * NaN is NaN in the MMA: in the
  // last tile (k0 + 64 > L), clear the V rows of slots the sequence never
  // wrote (and of pages past it).  Warp q clears rows 16q .. 16q+15, once
  // the tile has landed (P(t).V, the stage's next reader, waits for p_full).
  auto clear_v_tail = [&](uint32_t t, int k0, int L) -> bool {
    if (!__all_sync(0xffffffffu,
                    dev::mbar_wait(v_full0 + 8 * (t % kVStages),
                                   (t / kVStages) & 1)))
      return false;
    const uint32_t vt = vring + (t % kVStages) * kKVTile;
    for (int idx = lane; idx < 16 * 8 * kHalves; idx += 32) {
      const int krow = quarter * 16 + idx / (8 * kHalves);
      const int ch = idx % (8 * kHalves);
      if (k0 + krow >= L)
        dev::st_shared_zero16(vt + (ch >> 3) * kTileHalf + krow * 128 +
                              (ch & 7) * 16);
    }
    dev::fence_proxy_async_smem();  // visible to the tensor cores' P.V
    return true;
  };
  bool ok = true;
  uint32_t g = 0;  // tiles of this CTA's earlier items

  if constexpr (RQ > 0) {
    // ------ softmax warps, few query rows (<= 4 * RQ real, RQ per quarter) --
    // Query row r = i * G + h (token i, head h) sits in lane
    // 32 * (r / RQ) + r % RQ: each warp owns RQ rows, and four threads share
    // a row, each taking 16 of a tile's 64 keys (the 16x256b shape gives a
    // thread lanes t/4 and t/4 + 8: one row when RQ = 8, the other lane
    // being padding, two rows when RQ = 16).  Lanes RQ .. 31 of every
    // quarter are padding: never read back.
    constexpr int kR = RQ / 8;  // rows per thread
    const int c4 = lane & 3;  // this thread's key pairs
    int t_loc[kR], hq[kR];
#pragma unroll
    for (int x = 0; x < kR; ++x) {
      const int rr = quarter * RQ + (lane >> 2) + 8 * x;  // query row
      t_loc[x] = rr / G;
      hq[x] = rr - t_loc[x] * G;
    }
    for (int n = 0; ok; ++n) {
      Item it;
      ok = next_item(n, it);
      if (!ok || it.state == kEnd) break;
      if (it.state == kSkip) continue;
      const Span sp = span_of(it);
      const int L = it.L;
      int qpos[kR];
      bool valid[kR];
#pragma unroll
      for (int x = 0; x < kR; ++x) {
        valid[x] = t_loc[x] < sp.n_q;
        qpos[x] = valid[x] ? L - it.q_len + sp.tok0 + t_loc[x]
                           : sp.kv_end - 1;
      }
      const bool idle = quarter * RQ >= sp.n_q * G;  // no real row here
      float m_ref[kR], l[kR];  // l: this thread's keys only
#pragma unroll
      for (int x = 0; x < kR; ++x) {
        m_ref[x] = -INFINITY;
        l[x] = 0.f;
      }
      for (int j = 0; j < sp.n_tiles && ok; ++j) {
        const uint32_t t = g + j;
        ok = __all_sync(0xffffffffu, dev::mbar_wait(s_full, t & 1));
        if (!ok) break;
        float sa[32];
        if (!idle) {
          dev::tc_fence_after();
          tmem_ld16x256_x8(s_tmem + lane_off, sa);
          dev::tmem_ld_wait();
          dev::tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(s_free);
        const int k0 = j * kKeys;
        if (k0 + kKeys > L && !(ok = clear_v_tail(t, k0, L))) break;
        if (idle) {
          // Like the other warps, arrive for tile t only once P(t-1).V is
          // done: a warp that ran a tile ahead would have its arrival
          // counted toward tile t-1 on the single p_full barrier.
          if (t >= 1 && !wait_pv(t - 1)) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) dev::mbar_arrive(p_full);
          continue;
        }
        // sa[4k + 2x + e]: row x, key 8k + 2 c4 + e.
        float sv[kR][16];
        float factor[kR];
        bool grow = false, want = false;
#pragma unroll
        for (int x = 0; x < kR; ++x) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            sv[x][2 * k] = sa[4 * k + 2 * x];
            sv[x][2 * k + 1] = sa[4 * k + 2 * x + 1];
          }
          const int lim = qpos[x] - k0;
          if (lim < kKeys - 1) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                if (8 * k + 2 * c4 + e > lim) sv[x][2 * k + e] = -INFINITY;
          }
          float m4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) m4[u] = fmaxf(sv[x][u], sv[x][u + 4]);
#pragma unroll
          for (int k = 8; k < 16; ++k) m4[k & 3] = fmaxf(m4[k & 3], sv[x][k]);
          float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          mx *= c;
          factor[x] = 1.f;
          if (j == 0) {
            m_ref[x] = mx;
          } else if (mx > m_ref[x] + kRescaleLog2) {
            factor[x] = dev::fast_exp2(m_ref[x] - mx);
            m_ref[x] = mx;
            l[x] *= factor[x];
            grow = true;
          }
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            sv[x][k] = dev::fast_exp2(fmaf(sv[x][k], c, -m_ref[x]));
            l4[k & 3] += sv[x][k];
          }
          l[x] += (l4[0] + l4[1]) + (l4[2] + l4[3]);
          // Residual vote, as in the one-row-per-thread layout: the row's
          // sum so far is spread over its four threads.
          if (a.pv_split == 0) {
            float lr = l[x] + __shfl_xor_sync(0xffffffffu, l[x], 1);
            lr += __shfl_xor_sync(0xffffffffu, lr, 2);
            want |=
                valid[x] && dev::fast_exp2(mx - m_ref[x]) * kSplitInv > lr;
          }
        }
        const bool split = __any_sync(0xffffffffu, want || a.pv_split == 1);
        if (__any_sync(0xffffffffu, grow)) {
          ok = wait_pv(t - 1);
          if (!ok) break;
          dev::tc_fence_after();
#pragma unroll
          for (int col = 0; col < D; col += 32) {
            float ov[16];
            tmem_ld16x256_x4(o_tmem + lane_off + col, ov);
            dev::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int x = 0; x < kR; ++x) {
                ov[4 * k + 2 * x] *= factor[x];
                ov[4 * k + 2 * x + 1] *= factor[x];
              }
            tmem_st16x256_x4(o_tmem + lane_off + col, ov);
          }
          dev::tmem_st_wait();
        }
        // P(t) into its buffer: column 4k + c4 of each half holds keys
        // 8k + 2 c4 and 8k + 2 c4 + 1 of row x in lane t/4 + 8x; a padding
        // lane gets zeros.
        {
          uint32_t hw[16], lw[16];
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (x < kR) {
                const uint32_t w = M::pack(sv[x][2 * k], sv[x][2 * k + 1]);
                hw[2 * k + x] = w;
                if (split) {
                  const float2 hf = M::unpack(w);
                  lw[2 * k + x] =
                      M::pack(sv[x][2 * k] - hf.x, sv[x][2 * k + 1] - hf.y);
                } else {
                  lw[2 * k + x] = 0u;
                }
              } else {
                hw[2 * k + x] = 0u;
                lw[2 * k + x] = 0u;
              }
            }
          // P(t-1).V must have read the P buffer before it is overwritten.
          if (t >= 1 && !wait_pv(t - 1)) {
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t pa = p_tmem + lane_off;
          tmem_st16x128_x8(pa, hw);
          if (a.pv_split != 2) tmem_st16x128_x8(pa + kKeys / 2, lw);
          dev::tmem_st_wait();
        }
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (split) pv_vote[0] = t + 1u;
          dev::mbar_arrive(p_full);
        }
      }
      // The item's output: the row sums over the four threads, O / l -> out.
      float inv[kR];
#pragma unroll
      for (int x = 0; x < kR; ++x) {
        l[x] += __shfl_xor_sync(0xffffffffu, l[x], 1);
        l[x] += __shfl_xor_sync(0xffffffffu, l[x], 2);
        inv[x] = l[x] > 0.f ? 1.f / l[x] : 0.f;
      }
      if (ok && !idle) ok = wait_pv(g + sp.n_tiles - 1);
      if (ok && !idle) {
        dev::tc_fence_after();
#pragma unroll
        for (int col = 0; col < D; col += 32) {
          float ov[16];
          tmem_ld16x256_x4(o_tmem + lane_off + col, ov);
          dev::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < kR; ++x) {
            if (!valid[x]) continue;
            const int64_t idx =
                (static_cast<int64_t>(it.q0 + sp.tok0 + t_loc[x]) *
                     a.num_q_heads +
                 it.kvh * G + hq[x]) * D + 2 * c4 + col;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int64_t e = idx + 8 * k;  // dims e, e + 1
              const float v0 = ov[4 * k + 2 * x] * inv[x];
              const float v1 = ov[4 * k + 2 * x + 1] * inv[x];
              if (a.out_f32)
                *reinterpret_cast<float2*>(static_cast<float*>(a.out) + e) =
                    make_float2(v0, v1);
              else
                *reinterpret_cast<uint32_t*>(static_cast<T*>(a.out) + e) =
                    M::pack(v0, v1);
            }
          }
        }
      }
      g += sp.n_tiles;
    }
    if (!ok) dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
    dev::tc_fence_before();
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(done);
    return;
  }

  // ---------------- softmax warps (thread = query row) ----------------
  const int r = quarter * 32 + lane;
  const int t_loc = r / G;
  const int hg = r - t_loc * G;  // query head within the group
  // The residual columns of this warp's rows hold something other than
  // zeros (tensor memory starts undefined).
  bool res_dirty = true;
  for (int n = 0; ok; ++n) {
    Item it;
    ok = next_item(n, it);
    if (!ok || it.state == kEnd) break;
    if (it.state == kSkip) continue;
    const Span sp = span_of(it);
    const int L = it.L;
    const int tok = sp.tok0 + t_loc;
    const bool valid = t_loc < sp.n_q;
    // Padding rows (no query) see every key the tile loads; never stored.
    const int qpos = valid ? L - it.q_len + tok : sp.kv_end - 1;
    // A warp whose 32 rows are all padding (few new tokens: 4 drafts x 8
    // heads fill one warp's rows of 128) computes nothing: it keeps the
    // barrier protocol (including the wait for P(t-1).V before it arrives
    // for tile t) and its share of the V clearing only.  Its rows of P hold
    // stale values, which reach only its own (never stored) rows of O.
    const bool idle = quarter * 32 >= sp.n_q * G;
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < sp.n_tiles && ok; ++j) {
      const uint32_t t = g + j;
      ok = __all_sync(0xffffffffu, dev::mbar_wait(s_full, t & 1));
      if (!ok) break;
      float sv[kKeys];
      if (!idle) {
        dev::tc_fence_after();
        const uint32_t sa = s_tmem + lane_off;
        float (&lo)[32] = *reinterpret_cast<float(*)[32]>(sv);
        float (&hi)[32] = *reinterpret_cast<float(*)[32]>(sv + 32);
        dev::tmem_ld32(sa, lo);
        dev::tmem_ld32(sa + 32, hi);
        dev::tmem_ld_wait();
        dev::tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(s_free);
      const int k0 = j * kKeys;
      if (k0 + kKeys > L && !(ok = clear_v_tail(t, k0, L))) break;
      if (idle) {
        // Like the other warps, arrive for tile t only once P(t-1).V is done:
        // a warp that ran a tile ahead would have its arrival counted toward
        // tile t-1 on the single p_full barrier.
        if (t >= 1 && !wait_pv(t - 1)) {
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(p_full);
        continue;
      }
      // Causal mask: only tiles that reach past this row's position.
      const int lim = qpos - k0;
      if (lim < kKeys - 1) {
#pragma unroll
        for (int k = 0; k < kKeys; ++k)
          if (k > lim) sv[k] = -INFINITY;
      }
      // Eight independent partial maxima of eight keys each (and eight partial
      // sums below), three inputs per max instruction: a 64-long serial chain
      // of dependent instructions would stall the warp on each step.
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        m8[u] = dev::fmax3(dev::fmax3(sv[u], sv[u + 8], sv[u + 16]),
                           dev::fmax3(sv[u + 24], sv[u + 32], sv[u + 40]),
                           fmaxf(sv[u + 48], sv[u + 56]));
      float mx = dev::fmax3(dev::fmax3(m8[0], m8[1], m8[2]),
                            dev::fmax3(m8[3], m8[4], m8[5]),
                            fmaxf(m8[6], m8[7]));
      mx *= c;  // the scale is positive: max commutes with it
      float factor = 1.f;
      if (j == 0) {
        m_ref = mx;  // O is still empty: the first P.V overwrites it
      } else if (mx > m_ref + kRescaleLog2) {
        factor = dev::fast_exp2(m_ref - mx);
        m_ref = mx;
        l *= factor;
      }
      if (__any_sync(0xffffffffu, factor != 1.f)) {
        // O must hold P(t-1).V before it is rescaled (P(t).V is not issued
        // until this warp arrives on p_full below).
        ok = wait_pv(t - 1);
        if (!ok) break;
        dev::tc_fence_after();
#pragma unroll
        for (int col = 0; col < D; col += 32) {
          float ov[32];
          dev::tmem_ld32(o_tmem + lane_off + col, ov);
          dev::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= factor;
          dev::tmem_st32(o_tmem + lane_off + col, ov);
        }
        dev::tmem_st_wait();
      }
      // P = 2^(s * c - m_ref) in two halves of 32 keys, two keys per
      // instruction for the exponents and the sums.  Each half's rounded part
      // goes to tensor memory as soon as it is packed (once P(j-1).V has read
      // the buffer), so the store of the first half overlaps the exponentials
      // of the second.
      uint32_t hw[kKeys / 2];
      {
        const float2 c2 = make_float2(c, c);
        const float2 nm2 = make_float2(-m_ref, -m_ref);
        float2 l4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int e = 16 * h; e < 16 * h + 16; ++e) {
            const float2 x =
                dev::ffma2(make_float2(sv[2 * e], sv[2 * e + 1]), c2, nm2);
            sv[2 * e] = dev::fast_exp2(x.x);
            sv[2 * e + 1] = dev::fast_exp2(x.y);
            l4[e & 3] =
                dev::fadd2(l4[e & 3], make_float2(sv[2 * e], sv[2 * e + 1]));
            hw[e] = M::pack(sv[2 * e], sv[2 * e + 1]);
          }
          if (h == 0) {
            // P(t-1).V must have read the P buffer before it is overwritten.
            if (t >= 1 && !wait_pv(t - 1)) ok = false;
            if (!ok) break;
            dev::tc_fence_after();
          }
          dev::tmem_st16u(
              p_tmem + lane_off + 16 * h,
              *reinterpret_cast<const uint32_t(*)[16]>(hw + 16 * h));
        }
        if (!ok) break;
        const float2 la = dev::fadd2(l4[0], l4[1]);
        const float2 lb = dev::fadd2(l4[2], l4[3]);
        l += (la.x + la.y) + (lb.x + lb.y);
      }
      // Does a key of this tile need P's residual?  Its p is at most
      // 2^(mx - m_ref); it needs it if that can exceed l / kSplitInv.
      const bool split = __any_sync(
          0xffffffffu,
          a.pv_split == 1 ||
              (a.pv_split == 0 && valid &&
               dev::fast_exp2(mx - m_ref) * kSplitInv > l));
      // The residual P - hi.  When this warp's rows need none, its residual
      // columns must read as zeros (another warp's rows may make the MMA add
      // them): they are cleared once after a tile that wrote a residual, not
      // every tile.
      if (a.pv_split != 2 && (split || res_dirty)) {
        uint32_t lw[kKeys / 2];
        if (split) {
          const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
          for (int e = 0; e < kKeys / 2; ++e) {
            const float2 r = dev::ffma2(M::unpack(hw[e]), m1,
                                        make_float2(sv[2 * e], sv[2 * e + 1]));
            lw[e] = M::pack(r.x, r.y);
          }
        } else {
#pragma unroll
          for (int e = 0; e < kKeys / 2; ++e) lw[e] = 0u;
        }
        dev::tmem_st32u(p_tmem + lane_off + kKeys / 2, lw);
      }
      res_dirty = split;
      dev::tmem_st_wait();
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (split) pv_vote[0] = t + 1u;
        dev::mbar_arrive(p_full);
      }
    }
    // The item's output: O / l -> out[token, query head].
    if (ok && !idle) ok = wait_pv(g + sp.n_tiles - 1);
    if (ok && !idle) {
      dev::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t idx =
          (static_cast<int64_t>(it.q0 + tok) * a.num_q_heads + it.kvh * G +
           hg) * D;
      T* dst = static_cast<T*>(a.out) + idx;
      float* dst32 = static_cast<float*>(a.out) + idx;  // out_f32 only
#pragma unroll
      for (int col = 0; col < D; col += 32) {
        float ov[32];
        dev::tmem_ld32(o_tmem + lane_off + col, ov);
        dev::tmem_ld_wait();
        if (valid && a.out_f32) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst32 + col + e) =
                make_float4(ov[e] * inv, ov[e + 1] * inv, ov[e + 2] * inv,
                            ov[e + 3] * inv);
        } else if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = M::pack(ov[e] * inv, ov[e + 1] * inv);
            w.y = M::pack(ov[e + 2] * inv, ov[e + 3] * inv);
            w.z = M::pack(ov[e + 4] * inv, ov[e + 5] * inv);
            w.w = M::pack(ov[e + 6] * inv, ov[e + 7] * inv);
            *reinterpret_cast<uint4*>(dst + col + e) = w;
          }
        }
      }
    }
    g += sp.n_tiles;
  }
  if (!ok) dev::set_error(a.dev_err, PA_ERR_DEVICE_TIMEOUT);
  dev::tc_fence_before();
  __syncwarp();
  if (lane == 0) dev::mbar_arrive(done);
}

// ---------------------------------------------------------------------------
// Host side.

CUtensorMapDataType tma_type(pa_dtype t) {
  return t == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// q [total_q, Hq, D] as a 3-D tensor; box = 64 dims x G heads x tokens.
bool encode_q(CUtensorMap* m, const void* q, int total_q, int hq, int hd,
              int g, int tok, pa_dtype dt) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(hd),
                        static_cast<cuuint64_t>(hq),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(hd) * 2,
                           static_cast<cuuint64_t>(hq) * hd * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(g),
                       static_cast<cuuint32_t>(tok)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  return enc(m, tma_type(dt), 3, const_cast<void*>(q), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_cache(CUtensorMap* m, const void* cache, uint64_t rows, int hd,
                  int bs, pa_dtype dt) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(hd), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(hd) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(bs)};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, tma_type(dt), 2, const_cast<void*>(cache), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One CTA: the longest-first order of the sequences (by context length),
// then the prefill's tile map in that order.  Sequence b's new tokens fill
// ceil(q_len / tok) query tiles of tok tokens; the map lists them, the last
// (the one that sees the most keys) first, as (b, tile) pairs, and (-1, 0)
// after the last one up to its capacity `cap`.  A sequence whose rows fall
// outside q, or that has more new tokens than its context or than
// max_q_len, gets no tiles and sets PA_ERR_DEVICE_OOB; so does a map that
// would overflow (rows of several sequences overlapping), which is cut at
// `cap`.  Launched by programmatic stream serialization: it reads the
// lengths and rows and sorts while the kernel before it drains, then waits
// for that kernel (which may still read the workspace: the previous
// prefill) before writing; the prefill launches early behind it.
__global__ void __launch_bounds__(kOrderThreads)
    prefill_plan_kernel(const int32_t* __restrict__ context_lens,
                        const int32_t* __restrict__ query_start, int num_seqs,
                        int total_q, int max_q_len, int shift, int tok,
                        int cap, int32_t* __restrict__ order,
                        int2* __restrict__ tiles, int* counter,
                        int32_t* dev_err) {
  dev::pdl_trigger();
  // Tile counts and their running sum in 64 bits: sequences whose rows
  // overlap (each range valid on its own) may list more than 2^31 tiles.
  __shared__ int s_b[kOrderThreads];
  __shared__ long long s_n[kOrderThreads], s_start[kOrderThreads];
  __shared__ long long s_warp[kOrderThreads / 32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = false;
  auto tiles_of = [&](int b) -> long long {  // 0 (flagged) if invalid
    const int q0 = query_start[b], q1 = query_start[b + 1];
    if (q0 < 0 || q1 < q0 || q1 > total_q || q1 - q0 > context_lens[b] ||
        q1 - q0 > max_q_len) {
      bad = true;
      return 0;
    }
    return (static_cast<long long>(q1 - q0) + tok - 1) / tok;
  };
  // Up to kOrderThreads sequences, one per thread: a sequence's tile count
  // is loaded with its length and the sort places both at its rank in
  // shared memory (the order itself is not stored); the ranks are scanned
  // there too, so after the wait for the previous kernel only the map's
  // stores are left.  More sequences go through `order` in global memory.
  const bool one_pass = num_seqs <= kOrderThreads;
  const long long my_n = one_pass && tid < num_seqs ? tiles_of(tid) : 0;
  auto key = [&](int i) {
    const int L = context_lens[i];
    return L <= 0 ? 0 : (L >> shift);
  };
  if (one_pass) {
    counting_sort_desc_place(
        num_seqs, key,
        [&](int pos, int i) {  // i == tid
          s_b[pos] = i;
          s_n[pos] = my_n;
        },
        [] {});
  } else {
    counting_sort_desc_place(
        num_seqs, key, [&](int pos, int i) { order[pos] = i; },
        [] { dev::pdl_wait(); });
  }
  if (tid == 0) s_carry = 0;
  __syncthreads();  // the placed ranks (and the order, for more sequences)
  for (int base = 0; base < num_seqs; base += kOrderThreads) {
    const int z = base + tid;
    int b = -1;
    long long n = 0;
    if (z < num_seqs) {
      if (one_pass) {
        b = s_b[z];
        n = s_n[z];
      } else {
        b = order[z];
        n = tiles_of(b);
      }
    }
    // Where sequence z's tiles start: a scan of the tile counts over the
    // CTA, after those of the earlier chunks (s_carry).
    long long x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      long long w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const long long incl = x + (warp > 0 ? s_warp[warp - 1] : 0);
    s_b[tid] = b;
    s_n[tid] = n;
    s_start[tid] = s_carry + incl - n;
    __syncthreads();
    // The previous kernel may still read the workspace (a no-op when
    // already waited for).
    dev::pdl_wait();
    // A warp per sequence writes its tiles, a lane per tile.
    const int cnt = min(kOrderThreads, num_seqs - base);
    for (int i = warp; i < cnt; i += kOrderThreads / 32) {
      const long long st = s_start[i];
      const int sb = s_b[i];
      // Only the tiles that fit the map: slots st .. min(st + n, cap) - 1.
      const long long end = min(st + s_n[i], static_cast<long long>(cap));
      for (long long slot = st + lane; slot < end; slot += 32)
        tiles[slot] = make_int2(sb, static_cast<int>(st + s_n[i] - 1 - slot));
    }
    __syncthreads();  // every thread has read s_carry and the chunk's rows
    if (tid == kOrderThreads - 1) s_carry += incl;
    __syncthreads();
  }
  dev::pdl_wait();
  const long long total = s_carry;
  if (total > cap) bad = true;
  for (long long i = total + tid; i < cap; i += kOrderThreads)
    tiles[i] = make_int2(-1, 0);
  if (tid == 0) *counter = 0;  // the prefill's work items start at 0
  if (bad) dev::set_error(dev_err, PA_ERR_DEVICE_OOB);
}

// New tokens per query tile (tile rows / query group) and the tile map's
// capacity: the map holds sum over sequences of ceil(q_len / tok) tiles,
// which is at most total_q / tok + num_seqs when the sequences' rows do not
// overlap, and at most num_seqs * ceil(max_q_len / tok) as the plan kernel
// drops a sequence above max_q_len.
int tile_tokens(const pa_prefill_desc* d) {
  return kRows / (d->num_q_heads / d->num_kv_heads);
}
int64_t tile_cap(const pa_prefill_desc* d) {
  const int tok = tile_tokens(d);
  return std::min(static_cast<int64_t>(d->total_q) / tok + d->num_seqs,
                  static_cast<int64_t>(d->num_seqs) *
                      ((static_cast<int64_t>(d->max_q_len) + tok - 1) / tok));
}

// The sequence order (num_seqs int32, rounded up to 16 bytes), the work
// counter (16 bytes), then the tile map (int2 entries, rounded up to 16).
size_t order_bytes(const pa_prefill_desc* d) {
  return (static_cast<size_t>(d->num_seqs) * sizeof(int32_t) + 15) &
         ~size_t(15);
}
constexpr size_t kCounterBytes = 16;
size_t prefill_workspace_bytes(const pa_prefill_desc* d) {
  const size_t order = order_bytes(d);
  const int G = d->num_kv_heads > 0 ? d->num_q_heads / d->num_kv_heads : 0;
  if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->total_q < 0 ||
      d->max_q_len < 0 || d->num_q_heads % d->num_kv_heads || G <= 0 ||
      G > kRows)
    return order;  // the call rejects this shape
  return order + kCounterBytes +
         ((static_cast<size_t>(tile_cap(d)) * sizeof(int2) + 15) &
          ~size_t(15));
}

template <typename T, int BS, int G, int D, int RQ>
pa_status launch(const pa_prefill_desc* d, const PrefillArgs& a,
                 const CUtensorMap& qm, const CUtensorMap& km,
                 const CUtensorMap& vm, cudaStream_t st) {
  auto kern = prefill_kernel<T, BS, G, D, RQ>;
  const size_t smem = LayoutFor<D, RQ>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
      static_cast<int>(smem));
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_prefill: cudaFuncSetAttribute(%zu): %s",
                smem, cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  // Persistent: two CTAs per SM (shared and tensor memory allow no more),
  // fewer when there are fewer work items.
  const int64_t slots = 2LL * std::max(device_sm_count(), 1);
  cfg.gridDim =
      dim3(static_cast<unsigned>(std::min<int64_t>(a.num_items, slots)));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, qm, km, vm, a);
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s",
                cudaGetErrorString(e));
  return PA_OK;
}

template <typename T, int BS, int D, int RQ>
pa_status dispatch_group(const pa_prefill_desc* d, const PrefillArgs& a,
                         const CUtensorMap& qm, const CUtensorMap& km,
                         const CUtensorMap& vm, cudaStream_t st) {
  switch (d->num_q_heads / d->num_kv_heads) {
    case 1: return launch<T, BS, 1, D, RQ>(d, a, qm, km, vm, st);
    case 2: return launch<T, BS, 2, D, RQ>(d, a, qm, km, vm, st);
    case 4: return launch<T, BS, 4, D, RQ>(d, a, qm, km, vm, st);
    default: return launch<T, BS, 8, D, RQ>(d, a, qm, km, vm, st);
  }
}

template <typename T, int RQ>
pa_status dispatch_shape(const pa_prefill_desc* d, const PrefillArgs& a,
                         const CUtensorMap& qm, const CUtensorMap& km,
                         const CUtensorMap& vm, cudaStream_t st) {
  if (d->head_dim == 128)
    return d->block_size == 16
               ? dispatch_group<T, 16, 128, RQ>(d, a, qm, km, vm, st)
               : dispatch_group<T, 32, 128, RQ>(d, a, qm, km, vm, st);
  return d->block_size == 16
             ? dispatch_group<T, 16, 64, RQ>(d, a, qm, km, vm, st)
             : dispatch_group<T, 32, 64, RQ>(d, a, qm, km, vm, st);
}

}  // namespace
}  // namespace pagedkv

using pagedkv::fail;

extern "C" pa_status pa_prefill(void* out, const void* q, const void* k_cache,
                                const void* v_cache,
                                const int32_t* block_tables,
                                const int32_t* context_lens,
                                const int32_t* query_start, float scale,
                                const pa_prefill_desc* d, void* workspace,
                                size_t workspace_bytes, int32_t* dev_err,
                                void* stream) {
  pagedkv::clear_error();
  if (!d) return fail(PA_ERR_INVALID_ARG, "pa_prefill: desc is NULL");
  if (d->num_seqs < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
      d->max_blocks_per_seq <= 0 || d->num_blocks < 0 || d->total_q < 0 ||
      d->max_q_len < 0 || d->max_context_len < 0 ||
      d->num_q_heads % d->num_kv_heads ||
      (d->dtype != PA_F16 && d->dtype != PA_BF16) || !std::isfinite(scale))
    return fail(PA_ERR_INVALID_ARG,
                "pa_prefill: num_seqs=%d num_q_heads=%d num_kv_heads=%d "
                "max_blocks_per_seq=%d total_q=%d max_q_len=%d dtype=%d",
                d->num_seqs, d->num_q_heads, d->num_kv_heads,
                d->max_blocks_per_seq, d->total_q, d->max_q_len,
                static_cast<int>(d->dtype));
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->kernel != PA_PREFILL_AUTO && d->kernel != PA_PREFILL_TILE)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: kernel %d", d->kernel);
  if (d->out_fp32 != 0 && d->out_fp32 != 1)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: out_fp32 %d", d->out_fp32);
  if (d->pv < PA_PV_AUTO || d->pv > PA_PV_SINGLE)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: pv %d", d->pv);
  if ((d->head_dim != 64 && d->head_dim != 128) ||
      (d->block_size != 16 && d->block_size != 32) ||
      (G != 1 && G != 2 && G != 4 && G != 8))
    return fail(PA_ERR_UNSUPPORTED,
                "pa_prefill: needs head_dim 64 or 128 (got %d), block_size "
                "16 or 32 (got %d) and a query group of 1, 2, 4 or 8 (got %d)",
                d->head_dim, d->block_size, G);
  if (d->num_seqs == 0 || d->total_q == 0 || d->max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens ||
      !query_start)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: NULL tensor pointer");
  if (!pagedkv::aligned16(out) || !pagedkv::aligned16(q) ||
      !pagedkv::aligned16(k_cache) || !pagedkv::aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG,
                "pa_prefill: out, q and the caches must be 16-byte aligned");
  // Work items (tile-map entry, KV head) are counted in an int.
  if (pagedkv::tile_cap(d) * d->num_kv_heads > 0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED,
                "pa_prefill: %lld query tiles x %d KV heads exceed 2^31 - 1 "
                "work items",
                static_cast<long long>(pagedkv::tile_cap(d)),
                d->num_kv_heads);
  const size_t need = pagedkv::prefill_workspace_bytes(d);
  if (!workspace || workspace_bytes < need || !pagedkv::aligned16(workspace))
    return fail(PA_ERR_WORKSPACE,
                "pa_prefill: workspace of %zu bytes (16-byte aligned) needed, "
                "got %zu at %p", need, workspace_bytes, workspace);
  if (d->num_blocks == 0 || d->num_seqs > 65535 || d->num_kv_heads > 65535)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: bad pool or batch size");
  if (static_cast<int64_t>(d->num_blocks) * d->num_kv_heads * d->block_size >
      0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED, "pa_prefill: pool exceeds 2^31 rows");
  const int max_ctx = d->max_context_len > 0
                          ? d->max_context_len
                          : d->max_blocks_per_seq * d->block_size;
  // At most 64 query rows per KV head (a few new tokens): the tile kernel
  // spreads them over the four softmax warps, 8 (up to 32 rows) or 16 (up
  // to 64) per warp.
  const int64_t q_rows = static_cast<int64_t>(d->max_q_len) * G;
  const int rq = q_rows <= 32 ? 8 : q_rows <= 64 ? 16 : 0;
  const int tok = rq > 0 ? rq / G : pagedkv::kRows / G;
  CUtensorMap qm, km, vm;
  const uint64_t rows = static_cast<uint64_t>(d->num_blocks) *
                        d->num_kv_heads * d->block_size;
  if (!pagedkv::encode_q(&qm, q, d->total_q, d->num_q_heads, d->head_dim, G,
                         tok, d->dtype) ||
      !pagedkv::encode_cache(&km, k_cache, rows, d->head_dim, d->block_size,
                             d->dtype) ||
      !pagedkv::encode_cache(&vm, v_cache, rows, d->head_dim, d->block_size,
                             d->dtype))
    return fail(PA_ERR_CUDA, "pa_prefill: cuTensorMapEncodeTiled failed");
  pagedkv::PrefillArgs a;
  a.out = out;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* counter = reinterpret_cast<int*>(ws + pagedkv::order_bytes(d));
  int2* tiles = reinterpret_cast<int2*>(ws + pagedkv::order_bytes(d) +
                                        pagedkv::kCounterBytes);
  a.tiles = tiles;
  a.counter = counter;
  a.num_items = static_cast<int>(pagedkv::tile_cap(d) * d->num_kv_heads);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start;
  a.dev_err = dev_err;
  a.scale_log2 = scale * pagedkv::kLog2e;
  a.num_q_heads = d->num_q_heads;
  a.num_kv_heads = d->num_kv_heads;
  a.max_blocks_per_seq = d->max_blocks_per_seq;
  a.num_blocks = d->num_blocks;
  a.max_context_len = max_ctx;
  a.total_q = d->total_q;
  a.out_f32 = d->out_fp32;
  a.pv_split = d->pv;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaLaunchConfig_t pcfg = {};
  pcfg.gridDim = dim3(1);
  pcfg.blockDim = dim3(pagedkv::kOrderThreads);
  pcfg.stream = s;
  cudaLaunchAttribute pattr[1];
  pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pattr[0].val.programmaticStreamSerializationAllowed = 1;
  pcfg.attrs = pattr;
  pcfg.numAttrs = 1;
  cudaError_t oe = cudaLaunchKernelEx(
      &pcfg, pagedkv::prefill_plan_kernel, context_lens, query_start,
      d->num_seqs, d->total_q, d->max_q_len, pagedkv::order_shift(max_ctx),
      pagedkv::tile_tokens(d), static_cast<int>(pagedkv::tile_cap(d)),
      static_cast<int32_t*>(workspace), tiles, counter, dev_err);
  pagedkv::count_launch();
  if (oe == cudaSuccess) oe = cudaGetLastError();
  if (oe != cudaSuccess)
    return fail(PA_ERR_CUDA, "pa_prefill: plan launch failed: %s",
                cudaGetErrorString(oe));
  if (rq == 8)
    return d->dtype == PA_BF16
               ? pagedkv::dispatch_shape<__nv_bfloat16, 8>(d, a, qm, km, vm, s)
               : pagedkv::dispatch_shape<__half, 8>(d, a, qm, km, vm, s);
  if (rq == 16)
    return d->dtype == PA_BF16
               ? pagedkv::dispatch_shape<__nv_bfloat16, 16>(d, a, qm, km, vm, s)
               : pagedkv::dispatch_shape<__half, 16>(d, a, qm, km, vm, s);
  return d->dtype == PA_BF16
             ? pagedkv::dispatch_shape<__nv_bfloat16, 0>(d, a, qm, km, vm, s)
             : pagedkv::dispatch_shape<__half, 0>(d, a, qm, km, vm, s);
}

extern "C" size_t pa_prefill_workspace_bytes(const pa_prefill_desc* d) {
  pagedkv::clear_error();
  if (!d || d->num_seqs < 0) return 0;
  return pagedkv::prefill_workspace_bytes(d);
}
