/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged KV-cache decode attention for
 * NVIDIA B200 (sm_100a), its cache-write and copy-on-write kernels, and the
 * host-side block manager that produces block tables and slot mappings.
 *
 * Sources (cited by short name in the comments below):
 *   [Taming the Tail]          "Taming the Tail: How PagedAttention Solves the
 *                              KV-Cache Fragmentation Crisis in Multi-Tenant
 *                              LLM Serving" (architects-blueprint.vercel.app)
 *   [vLLM PagedAttention FAQ]  "vLLM PagedAttention: Eliminating KV Cache
 *                              Memory Fragmentation & 4x Throughput"
 *                              (tinycto.tv)
 *   [KV-cache chapter]         the "g12s-kv-cache" chapter on KV-cache
 *                              management (aicomputerinstitute.com)
 *
 * Conventions for every call:
 *   - Tensor arguments are DEVICE pointers borrowed from the caller, who
 *     allocates and frees them; the library never frees or keeps them.
 *     Every tensor pointer must be 16-byte aligned and densely packed in the
 *     layout stated for it.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernel calls are asynchronous on that stream; their return
 *     value reports argument checks and launch errors only.
 *   - `dev_err` (nullable) is a device int32.  A kernel that meets a
 *     violation it can only see on the device (a block id outside the pool, a
 *     slot outside the cache, a context length beyond the table) stores
 *     PA_ERR_DEVICE_OOB there, skips the affected work and never touches an
 *     out-of-range address; a bounded wait that gave up stores
 *     PA_ERR_DEVICE_TIMEOUT.  The library never clears it: the caller zeroes
 *     it and reads it after synchronising.
 *   - Ordering on one stream: pa_copy_blocks, then pa_cache_write, then
 *     pa_decode ([KV-cache chapter] "PagedAttention: borrowing virtual
 *     memory...": a private copy is made before the first write into a shared
 *     block).
 *   - pa_cache_write, pa_copy_blocks, pa_decode and pa_prefill only enqueue
 *     kernels (no allocation, no synchronisation), so a sequence of them
 *     can be captured in a CUDA graph and replayed; the graph keeps the
 *     pointers and shapes it was captured with.  Call each shape once
 *     outside capture first (the first call configures its kernel).
 *   - pa_last_error() returns a thread-local text describing the last
 *     non-OK status produced on the calling thread.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer */
  PA_ERR_UNSUPPORTED = 2,     /* a shape the kernels are not built for      */
  PA_ERR_NO_FREE_BLOCKS = 3,  /* block manager: the pool is exhausted       */
  PA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed       */
  PA_ERR_DEVICE_OOB = 5,      /* device-side index check failed (dev_err)   */
  PA_ERR_WORKSPACE = 6,       /* workspace missing or too small             */
  PA_ERR_DEVICE_TIMEOUT = 7   /* a bounded device-side wait gave up         */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Which decode kernel runs.  Both compute the same result.
 *   PA_KERNEL_AUTO  -- the tensor-core kernel.
 *   PA_KERNEL_SIMT  -- fp32 CUDA-core dot products (kept for comparison).
 *   PA_KERNEL_MMA   -- the grouped query heads of one KV head form the N=8
 *                      side of warp-level bf16/fp16 tensor-core MMAs for
 *                      both QK^T and PV, fp32 accumulation. */
typedef enum { PA_KERNEL_AUTO = 0, PA_KERNEL_SIMT = 1, PA_KERNEL_MMA = 2 } pa_kernel;

/* How the partitions of a split sequence are combined.  Both give the same
 * result (out = sum_j w_j o_j / sum_j w_j with w_j = l_j exp(m_j - max m)).
 *   PA_REDUCE_AUTO    -- up to 16 partitions per sequence: the partition
 *                        CTA that finishes last combines them inside the
 *                        decode kernel; more: the separate reduce kernel.
 *   PA_REDUCE_KERNEL  -- always a second, separate reduce kernel. */
typedef enum { PA_REDUCE_AUTO = 0, PA_REDUCE_KERNEL = 1 } pa_reduce;

/* Shape of one decode call.
 *   num_q_heads must be a multiple of num_kv_heads; G = num_q_heads /
 *   num_kv_heads <= 8.  Query head h reads KV head h / G (consecutive
 *   grouping; the pages name grouped-query attention but no mapping).
 *   head_dim in {64, 128}; block_size in {16, 32} ([vLLM PagedAttention FAQ]
 *   "Prevention & Safeguards": block size 16 or 32).
 *   partition_size: tokens per split-context partition of one sequence; 0 =
 *   choose automatically; otherwise a multiple of block_size in [block_size,
 *   8192].  Sequences longer than one partition are computed as independent
 *   partitions whose partial softmax statistics a second kernel combines.
 *   max_context_len: host-side upper bound on every context_lens[] entry;
 *   sizes the grid and the workspace.  0 means num_blocks_per_seq * block_size. */
typedef struct {
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;
  pa_dtype dtype;
  int partition_size;
  int max_context_len;
  pa_kernel kernel;
  pa_reduce reduce;
  int out_fp32;  /* 0: out has q's dtype (rounded once).  1: out is float32,
                    the value before that rounding (a check of the kernel's
                    own error apart from the output rounding). */
} pa_decode_desc;

/* Library version string, and the text of a status code. */
const char* pa_version(void);
const char* pa_status_string(pa_status s);
/* Description of the last non-OK status returned on this thread ("" if none). */
const char* pa_last_error(void);

/* ------------------------------------------------------------------------
 * Decode attention over a paged KV cache.
 *
 * Defines ([Taming the Tail] "Under the Hood: The CUDA Kernel Engineering";
 * [KV-cache chapter] "PagedAttention: borrowing virtual memory..." and
 * "Common misconception..."; [vLLM PagedAttention FAQ] "Does PagedAttention
 * change the mathematical attention output?"): for sequence b and query head
 * h, with K_b / V_b the sequence's tokens gathered through its block table,
 *     out[b,h,:] = softmax(scale * K_b q[b,h,:]) V_b
 * exactly as contiguous multi-head attention would compute it.  A sequence
 * with context length 0 gets a zero output row.
 *
 * Layouts (all dense, row-major):
 *   out, q        [num_seqs, num_q_heads, head_dim]          dtype
 *                 (out float32 when desc->out_fp32 = 1)
 *   k_cache,
 *   v_cache       [num_blocks, num_kv_heads, block_size, head_dim]  dtype
 *   block_tables  [num_seqs, max_blocks_per_seq] int32 physical block ids;
 *                 entries past a sequence's last block are ignored
 *   context_lens  [num_seqs] int32, tokens per sequence, the newest included
 *   workspace     pa_decode_workspace_bytes(desc) bytes of device memory the
 *                 caller owns, 16-byte aligned (always > 0): partition
 *                 partials, per-(sequence, KV head) counters and the order
 *                 in which partitions are served (more than one partition
 *                 only), and the order in which sequences are served
 *                 (longest first, so the grid ends on short work), all
 *                 written by the call on its stream.  Its contents need
 *                 no initialisation and are scratch after the call; calls
 *                 that share a workspace must not overlap on the device.
 * Launches: a one-CTA prep kernel (the longest-first order; counter reset),
 * the decode, and with more than 16 partitions or PA_REDUCE_KERNEL the
 * reduce kernel, chained by programmatic dependent launch.  The prep kernel
 * reads context_lens before it waits for the kernel launched just before
 * the call, so that kernel, if it lets its dependents start early, must
 * not be the one that writes context_lens.
 * Computation: fp32 scores, fp32 online softmax, fp32 accumulation; the
 * output is rounded once to dtype.
 * Errors: PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED / PA_ERR_WORKSPACE before
 * any launch; PA_ERR_CUDA if a launch fails.  Device-side: a context length
 * outside [0, max_blocks_per_seq * block_size] or above max_context_len, or a
 * block id outside [0, num_blocks), sets *dev_err = PA_ERR_DEVICE_OOB and the
 * affected sequence's output rows are unspecified.
 * ---------------------------------------------------------------------- */
size_t pa_decode_workspace_bytes(const pa_decode_desc* desc);

/* Partition size the call will use for this shape (resolves 0 = auto). */
int pa_decode_partition_size(const pa_decode_desc* desc);

pa_status pa_decode(void* out, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables,
                    const int32_t* context_lens, float scale,
                    const pa_decode_desc* desc, void* workspace,
                    size_t workspace_bytes, int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------
 * pa_decode without a caller workspace.  (No counterpart in the pages: this
 * is a convenience of this library, not part of the method.)
 *
 * For callers that cannot allocate device memory: for example a serving
 * process that has handed nearly all of HBM to the KV-cache pool and allows
 * no further device allocations while it decodes, or a host program that
 * drives this library through the C ABI and has no device allocator of its
 * own.  The call computes exactly what pa_decode computes, with the
 * workspace taken from a fixed area of PA_NOALLOC_SCRATCH_BYTES inside the
 * library (a file-scope device array: every GPU that loads the library keeps
 * it until the process exits).  It allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *   - A shape whose pa_decode_workspace_bytes() exceeds
 *     PA_NOALLOC_SCRATCH_BYTES is rejected with PA_ERR_WORKSPACE and a
 *     message naming both sizes (use a larger partition_size or pa_decode).
 *   - The first call in a CUDA context looks up the area's device address
 *     (cudaGetSymbolAddress, with that context current) and keeps it, keyed
 *     on the context's unique id; make that first call before any stream
 *     capture.  A device reset (cudaDeviceReset) or a context the caller
 *     creates through the driver API gives a new id, so the address is
 *     looked up again there rather than reused.  The lookup is guarded by a
 *     mutex, so first calls from several host threads are safe.
 *   - Every call uses the same area, which keeps the previous call's data;
 *     what must start at zero (the per-sequence partition counters) is reset
 *     on the call's stream.  Calls that overlap on the GPU (other streams,
 *     other threads, the same device) race on the area and must be avoided.
 * Arguments, layouts and errors are those of pa_decode.
 * ---------------------------------------------------------------------- */
#define PA_NOALLOC_SCRATCH_BYTES (32ull << 20) /* 32 MiB per device */

pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, float scale,
                            const pa_decode_desc* desc, int32_t* dev_err,
                            void* stream);

/* ------------------------------------------------------------------------
 * Causal attention of new tokens over the paged cache (chunked prefill,
 * several speculative tokens at once).
 *
 * Defines ([vLLM PagedAttention FAQ] "Does PagedAttention change the
 * mathematical attention output?"; [Taming the Tail] "The Future:
 * Speculative Decoding and Beyond"; [KV-cache chapter] "Common
 * misconception...": serving kernels run FlashAttention-style tiles over the
 * paged layout): sequence b holds L = context_lens[b] tokens in the cache
 * (the new ones already written with pa_cache_write); its last
 * q_len = query_start[b+1] - query_start[b] tokens are new, with query rows
 * q[query_start[b] + i].  New token i sits at position p = L - q_len + i and
 *     out[query_start[b] + i, h, :] = softmax(scale * K_b[0..p] q) V_b[0..p]
 * with query head h reading KV head h / G.  q_len = 1 is decode; q_len = L a
 * whole prompt.
 * Layouts: q, out [total_q, num_q_heads, head_dim] dtype (out float32 with
 * desc->out_fp32); query_start [num_seqs+1]
 * int32 on the device, non-decreasing, query_start[0] = 0 and
 * query_start[num_seqs] <= total_q; the rest as for pa_decode.
 * Supported: head_dim 64 or 128, block_size 16 or 32, G = 1, 2, 4 or 8 (else
 * PA_ERR_UNSUPPORTED); any context length the table holds; max_q_len up to
 * 65535 tiles of 128 / G new tokens (PA_ERR_UNSUPPORTED above).  Runs on the
 * tcgen05 tensor cores with fp32 accumulation in tensor memory; output
 * rounded once to dtype.
 * Device-side: a context or query range outside the table, a sequence with
 * more new tokens than max_q_len, or a block id outside the pool sets
 * *dev_err = PA_ERR_DEVICE_OOB and the affected rows are unspecified.
 * ---------------------------------------------------------------------- */
/* Which prefill kernel runs (PA_PREFILL_AUTO and PA_PREFILL_TILE are the
 * same): tiles of 128 query rows (new token, query head) on the MMA's M side,
 * 64 keys on N; with at most 64 query rows per KV head (a few new tokens) the
 * rows are spread over all four softmax warps.  Any other value is
 * PA_ERR_INVALID_ARG. */
typedef enum {
  PA_PREFILL_AUTO = 0,
  PA_PREFILL_TILE = 1
} pa_prefill_kernel;

/* Precision of P in the tile kernel's P . V (the tensor cores take 16-bit
 * operands, so the softmax weights P are rounded to dtype).  One rounding
 * moves each weight by up to 2^-8 of itself in bf16 (2^-11 in fp16); on a
 * row whose weight sits on a few keys that moves the output by up to
 * 2^-8 |v|, more than the 2e-3 tolerance.  Adding residual . V, with the
 * residual = P - round(P) rounded again, keeps about 16 bits of P at the cost
 * of a second P . V MMA.
 *   PA_PV_AUTO    -- the residual only in tiles where some row has a key
 *                    with p > l / 16, l being the row's running sum of
 *                    weights including that tile (such a key may end with a
 *                    weight above 1/16); in every other tile each key ends
 *                    with a weight below 1/16 and the single rounding's
 *                    errors, of either sign, average out.  Within the
 *                    tolerance on every workload tested; on long rows
 *                    only the first few tiles need the residual.
 *   PA_PV_SPLIT   -- the residual in every tile.
 *   PA_PV_SINGLE  -- never: one rounding of P (as FlashAttention does);
 *                    fastest, but short or peaky rows may exceed 2e-3.
 */
typedef enum {
  PA_PV_AUTO = 0,
  PA_PV_SPLIT = 1,
  PA_PV_SINGLE = 2
} pa_prefill_pv;

typedef struct {
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;
  pa_dtype dtype;
  int total_q;          /* rows of q and out */
  int max_q_len;        /* host bound on any sequence's new-token count */
  int max_context_len;  /* host bound on context_lens[] (0: table capacity) */
  int kernel;           /* pa_prefill_kernel (0: automatic) */
  int out_fp32;         /* as in pa_decode_desc: 1 = out is float32 */
  int pv;               /* pa_prefill_pv (0: per tile, as needed) */
} pa_prefill_desc;

/* Bytes of device workspace pa_prefill needs for this shape: the sequence
 * order (num_seqs int32, rounded up to 16), a 16-byte work counter, and the
 * map of query tiles (8 bytes per tile, room for min(total_q / T + num_seqs,
 * num_seqs * ceil(max_q_len / T)) tiles of T = 128 / G new tokens,
 * G = num_q_heads / num_kv_heads, rounded up to 16). */
size_t pa_prefill_workspace_bytes(const pa_prefill_desc* desc);

/* workspace: pa_prefill_workspace_bytes(desc) bytes of caller-owned device
 * memory, 16-byte aligned (PA_ERR_WORKSPACE otherwise); scratch after the
 * call, and calls sharing it must not overlap on the device.  The call
 * launches a one-CTA kernel that orders the sequences longest context
 * first and lists their query tiles (128 / G new tokens each) in that
 * order, each sequence's last tile (the one that sees the most keys)
 * first; then the prefill, chained by programmatic launch: a persistent
 * grid (two CTAs per SM) whose CTAs take (listed tile, KV head) work items
 * from the counter in that order.  So a long sequence never starts last, no
 * work is spent on tiles past a shorter sequence's new tokens, and a CTA
 * loads its next item while it computes the current one.
 * PA_ERR_UNSUPPORTED when the items would exceed 2^31 - 1.  The first kernel is itself
 * launched programmatically: it reads context_lens and query_start before
 * it waits for the kernel launched just before the call, so that kernel,
 * if it lets its dependents start early, must not be the one that writes
 * them. */
pa_status pa_prefill(void* out, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, const int32_t* query_start,
                     float scale, const pa_prefill_desc* desc,
                     void* workspace, size_t workspace_bytes,
                     int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------
 * Write new tokens' K and V into their cache slots.
 *
 * Defines ([Taming the Tail] "How the Architecture Works"; [KV-cache
 * chapter] "A one-paragraph recap": each step stores only the new token's K
 * and V): for token t with s = slot_mapping[t] >= 0,
 *     k_cache[s / block_size, :, s % block_size, :] = k[t, :, :]
 *     v_cache[s / block_size, :, s % block_size, :] = v[t, :, :]
 * a byte-exact copy.  slot_mapping[t] < 0 marks padding and is skipped.
 * Layouts: k, v [num_tokens, num_kv_heads, head_dim]; slot_mapping
 * [num_tokens] int64 on the device; caches as for pa_decode.
 * Slots must be distinct (two tokens writing one slot race).  A slot >=
 * num_blocks * block_size sets *dev_err = PA_ERR_DEVICE_OOB and is skipped.
 * ---------------------------------------------------------------------- */
pa_status pa_cache_write(void* k_cache, void* v_cache, const void* k,
                         const void* v, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------
 * Copy whole blocks for copy-on-write.
 *
 * Defines ([KV-cache chapter] "PagedAttention: borrowing virtual memory...";
 * [Taming the Tail] "Complex Memory Sharing"): for each pair i,
 *     k_cache[dst] = k_cache[src];  v_cache[dst] = v_cache[src]
 * (all KV heads, all slots of the block), byte-exact, where
 * (src, dst) = (pairs[2i], pairs[2i+1]).  pairs is device int32 [num_pairs][2]
 * as produced by pa_bm_append.  Destinations must be distinct and no
 * destination may also be a source in the same call.  An id outside
 * [0, num_blocks) sets *dev_err = PA_ERR_DEVICE_OOB and that pair is skipped.
 * ---------------------------------------------------------------------- */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs,
                         int num_pairs, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------
 * pa_swap_blocks -- move whole blocks between two pools for preemption by
 * swapping a request's KV cache to CPU RAM and back ([Taming the Tail]
 * "Infrastructure Scale"; the pairs come from pa_bm_swap_out / _swap_in).
 *   dst_*_cache, src_*_cache  [num_dst_blocks | num_src_blocks, num_kv_heads,
 *                 block_size, head_dim] of `dtype`, 16-byte aligned.  Each
 *                 may be memory of the current device or page-locked host
 *                 memory mapped into the device address space (e.g. from
 *                 cudaHostAlloc / cudaMallocHost, or registered); the kernel
 *                 reads and writes host pages directly over the host link.
 *                 Pageable memory or another device's memory -> INVALID_ARG.
 *   pairs         int32 [num_pairs][2] (source block, destination block),
 *                 device or mapped page-locked host memory.
 * One launch; K and V of every pair.  A pair outside [0, num_src_blocks) x
 * [0, num_dst_blocks) sets *dev_err = PA_ERR_DEVICE_OOB and is skipped.
 * Stream-ordered: run it before anything reuses the source blocks (swap-out
 * frees device blocks; swap-in frees host blocks).  The caller keeps host
 * buffers alive until the stream has passed the copy.
 * ---------------------------------------------------------------------- */
pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache,
                         const void* src_k_cache, const void* src_v_cache,
                         const int32_t* pairs, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size,
                         int num_src_blocks, int num_dst_blocks,
                         pa_dtype dtype, int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------
 * Host block manager: free block pool, per-sequence logical->physical block
 * tables, reference counts and copy-on-write ([Taming the Tail] "How the
 * Architecture Works", "Complex Memory Sharing"; [vLLM PagedAttention FAQ]
 * "Underlying Mechanism"; [KV-cache chapter] "PagedAttention: borrowing
 * virtual memory..." and answer A6).  Pure host code: it touches no device
 * memory and produces only integer arrays.  A handle is not thread-safe; its
 * memory is owned by the handle and released by pa_bm_destroy.
 * ---------------------------------------------------------------------- */

/* Create a pool of num_blocks blocks of block_size tokens.  free_order
 * (nullable, host int32[num_blocks]) is a permutation of 0..num_blocks-1
 * giving the order in which a fresh pool hands blocks out (NULL = ascending).
 * Blocks returned to the pool are handed out again before untouched ones
 * (most recently freed first). */
pa_status pa_bm_create(int num_blocks, int block_size,
                       const int32_t* free_order, void** bm);
void pa_bm_destroy(void* bm);

/* Register an empty sequence.  INVALID_ARG if the id exists. */
pa_status pa_bm_add_seq(void* bm, int64_t seq_id);

/* The child shares every block of the parent (each reference count + 1) and
 * starts with the parent's length ([vLLM PagedAttention FAQ] "Zero-Copy
 * Forking & Parallel Sampling"). */
pa_status pa_bm_fork(void* bm, int64_t parent_id, int64_t child_id);

/* Reserve n_tokens new token slots at the end of seq_id.
 * A new block is taken only when the last block is full; the first write
 * into a block whose reference count is above one first moves the sequence
 * to a private copy (count of the old block - 1).
 *   slots_out      host int64[n_tokens]: slot = block * block_size + offset
 *                  for each new token, in order (pass to pa_cache_write).
 *   cow_pairs_out  host int32[2 * max_cow]: (src, dst) blocks to copy with
 *                  pa_copy_blocks BEFORE writing the slots.  At most one pair
 *                  per call.  Nullable only if max_cow == 0 and no copy is
 *                  needed.
 *   num_cow_out    number of pairs written.
 * If the pool cannot supply every block the call needs, returns
 * PA_ERR_NO_FREE_BLOCKS and changes nothing. */
pa_status pa_bm_append(void* bm, int64_t seq_id, int n_tokens,
                       int64_t* slots_out, int32_t* cow_pairs_out,
                       int max_cow, int* num_cow_out);

/* Batched form of pa_bm_append for one decode step: appends n_tokens[i]
 * tokens to seq_ids[i] for i = 0..n-1, in order.
 *   slots_out      host int64[sum(n_tokens)], the sequences' slots in order.
 *   cow_pairs_out  host int32[2 * max_cow] (max_cow >= number of sequences
 *                  whose last block is shared suffices); pairs in order.
 *   num_cow_out    pairs written.   num_done_out  sequences fully appended.
 * If the pool runs out at sequence i, returns PA_ERR_NO_FREE_BLOCKS with
 * *num_done_out = i: appends 0..i-1 stand (their slots and pairs are
 * written), sequence i and later are unchanged. */
pa_status pa_bm_append_batch(void* bm, const int64_t* seq_ids,
                             const int32_t* n_tokens, int n,
                             int64_t* slots_out, int32_t* cow_pairs_out,
                             int max_cow, int* num_cow_out, int* num_done_out);

/* Drop the sequence: each of its blocks' counts - 1; blocks at zero return
 * to the pool ([KV-cache chapter] answer A6). */
pa_status pa_bm_free_seq(void* bm, int64_t seq_id);

/* Keep the first new_len tokens and release the blocks past them, e.g. to
 * discard rejected speculative tokens ([Taming the Tail] "The Future:
 * Speculative Decoding and Beyond").  new_len <= current length. */
pa_status pa_bm_truncate(void* bm, int64_t seq_id, int64_t new_len);

/* Fill host table_out[n][max_blocks] (int32, unused entries -1) and
 * lens_out[n] (int32) for the listed sequences.  INVALID_ARG if a sequence
 * holds more than max_blocks blocks or is longer than INT32_MAX tokens. */
pa_status pa_bm_block_table(void* bm, const int64_t* seq_ids, int n,
                            int max_blocks, int32_t* table_out,
                            int32_t* lens_out);

/* ---- Prefix cache ([KV-cache chapter] "RadixAttention: caching, not just
 * packing, the prefix") ------------------------------------------------------
 * Cached token sequences form a radix tree with one node per FULL block,
 * keyed by that block's block_size tokens under its parent; the partly filled
 * last block of a sequence is never cached.  The cache holds one reference
 * on every block it stores (pa_bm_refcount counts it).  A cached block that
 * only the cache references and that has no cached children is an evictable
 * leaf.  A logical clock stamps every node on the path of each match and
 * insert; when pa_bm_append / pa_bm_append_batch need more blocks than the
 * pool has free, evictable leaves are evicted oldest stamp first (a parent
 * can become an evictable leaf in turn).  If even evicting all of them would
 * not supply the append, the append fails with PA_ERR_NO_FREE_BLOCKS and the
 * cache is left exactly as it was.  Blocks a sequence uses are never
 * evicted.  Token ids are opaque int32 values compared for equality. */

/* Attach to the new, EMPTY sequence seq_id the longest run of cached full
 * blocks that starts tokens[0 .. n_tokens) (host int32): those blocks are
 * referenced, not copied, and the sequence's length becomes *matched_out,
 * a multiple of block_size.  Only tokens past it need a prefill; append them
 * with pa_bm_append (which opens a fresh block: no copy-on-write).
 * INVALID_ARG if the sequence is unknown or not empty. */
pa_status pa_bm_match_prefix(void* bm, int64_t seq_id, const int32_t* tokens,
                             int64_t n_tokens, int64_t* matched_out);

/* Cache the full blocks among the first n_tokens tokens of seq_id, whose
 * token ids are tokens[0 .. n_tokens) (host int32; n_tokens <= the
 * sequence's length).  Call it once their K/V are written.  A block whose
 * tokens are already cached at that place keeps the cached node (the
 * sequence's duplicate stays outside the cache).  INVALID_ARG, changing
 * nothing, if one of the sequence's blocks is cached under different
 * tokens. */
pa_status pa_bm_cache_insert(void* bm, int64_t seq_id, const int32_t* tokens,
                             int64_t n_tokens);

/* Evict up to max_blocks evictable leaves, oldest stamp first; their blocks
 * return to the pool.  *evicted_out = how many. */
pa_status pa_bm_cache_evict(void* bm, int max_blocks, int* evicted_out);

/* Number of cached blocks (-1 for a NULL handle). */
int pa_bm_num_cached(void* bm);

/* Dump the tree breadth-first (every parent before its children):
 * parent_out[i] = index of node i's parent in this dump (-1 under the root),
 * block_out[i] = its physical block, tokens_out[i * block_size ..] = its
 * tokens (host arrays sized max_nodes, max_nodes * block_size).  INVALID_ARG
 * if more than max_nodes blocks are cached. */
pa_status pa_bm_cache_nodes(void* bm, int max_nodes, int32_t* parent_out,
                            int32_t* block_out, int32_t* tokens_out,
                            int* n_out);

/* ---- Swapping to a host pool ([Taming the Tail] "Infrastructure Scale":
 * pause a request and move its KV cache to CPU RAM) --------------------------
 * A second pool of host blocks; a swapped-out sequence keeps its table but
 * its entries name host blocks.  A group of sequences is swapped at once so
 * blocks the group shares cross the link once: each distinct block of the
 * group's tables (in order of first use: sequences as listed, logical blocks
 * in order) gets one block in the other pool holding the group's references
 * to it; the old block keeps the references other tables or the prefix cache
 * hold and returns to its pool when none are left.  pairs_out receives the
 * (source, destination) copies for pa_swap_blocks, which must run before the
 * freed blocks are written again.  All or nothing: PA_ERR_NO_FREE_BLOCKS (the
 * target pool, after evicting cache leaves for a swap-in, cannot supply every
 * block) or INVALID_ARG (unknown / repeated sequence, wrong swap state,
 * max_pairs too small: the distinct block count suffices) change nothing.
 * A swapped-out sequence can only be swapped in or freed: append, fork,
 * truncate, block_table, match_prefix and cache_insert refuse it. */

/* Size the host pool (ids 0..num_host_blocks-1).  INVALID_ARG while any host
 * block is in use. */
pa_status pa_bm_set_host_blocks(void* bm, int num_host_blocks);

/* Swap the n sequences out: pairs_out (host int32 [2 * max_pairs]) gets
 * (device block, host block) pairs, *num_pairs_out their number. */
pa_status pa_bm_swap_out(void* bm, const int64_t* seq_ids, int n,
                         int32_t* pairs_out, int max_pairs,
                         int* num_pairs_out);

/* Swap the n sequences back in: (host block, device block) pairs. */
pa_status pa_bm_swap_in(void* bm, const int64_t* seq_ids, int n,
                        int32_t* pairs_out, int max_pairs,
                        int* num_pairs_out);

/* Free host blocks; a host block's reference count (-1 if out of range);
 * 1 if the sequence is swapped out, 0 if not, -1 if unknown. */
int pa_bm_num_free_host(void* bm);
int pa_bm_host_refcount(void* bm, int host_block);
int pa_bm_is_swapped(void* bm, int64_t seq_id);

/* The sequence's table entries in logical order (device block ids, or host
 * block ids while it is swapped out) into blocks_out (host int32
 * [max_blocks]); *n_out = how many. */
pa_status pa_bm_seq_blocks(void* bm, int64_t seq_id, int32_t* blocks_out,
                           int max_blocks, int* n_out);

/* Pool sizing: how many blocks of block_size tokens fit in `bytes` for a
 * model of num_layers layers, each holding K and V of num_kv_heads heads of
 * head_dim 2-byte elements per token (a block id then names the same slot
 * range in every layer's cache).  Per token and layer that is
 * 2 * num_kv_heads * head_dim * 2 bytes ([Taming the Tail] "The Math of the
 * Cache" counts 2 x layers x hidden x bytes; with grouped-query attention
 * the per-layer width is num_kv_heads * head_dim).  Pass the share of free
 * device memory the cache may take (a serving engine's memory-utilisation
 * setting).  -1 (INVALID_ARG) for a non-positive shape or another dtype. */
int64_t pa_pool_blocks(uint64_t bytes, int num_layers, int num_kv_heads,
                       int head_dim, int block_size, pa_dtype dtype);

/* Kernel launches this library has issued in this process (all devices,
 * all threads): lets a caller count the GPU work a timed region contained. */
int64_t pa_launch_count(void);

/* Measurement helper (no counterpart in the pages): read `bytes` (rounded
 * down to 16) of the device buffer `buf` once with streaming 128-bit loads
 * on `stream`; `sink` is a device word the kernel may write.  Timed on a
 * buffer far larger than L2 it gives the read bandwidth the GPU sustains,
 * the roofline the decode's bandwidth is compared with. */
pa_status pa_read_probe(const void* buf, size_t bytes, uint32_t* sink,
                        void* stream);

/* Self-test of the kernels' bounded waits (no counterpart in the pages): one
 * warp allocates 32 tensor-memory columns and waits on an mbarrier that
 * nothing arrives at.  After the wait limit (1 s of device time) it sets
 * *dev_err = PA_ERR_DEVICE_TIMEOUT (if still 0), frees the tensor memory and
 * returns, which is what the decode and prefill kernels do when a copy
 * never lands.  dev_err: a device int32, required (PA_ERR_INVALID_ARG
 * otherwise).  Asynchronous on `stream`. */
pa_status pa_wait_probe(int32_t* dev_err, void* stream);

/* Pool and sequence queries (-1 for an unknown handle / sequence / block).
 * pa_bm_num_used = blocks referenced by a table or by the prefix cache
 * (num_blocks - pa_bm_num_free). */
int pa_bm_num_free(void* bm);
int pa_bm_num_used(void* bm);
int pa_bm_refcount(void* bm, int block);
int64_t pa_bm_seq_len(void* bm, int64_t seq_id);
int pa_bm_num_seq_blocks(void* bm, int64_t seq_id);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* PAGEDKV_H */
