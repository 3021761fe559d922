// Host block manager: free pool, per-sequence block tables, reference counts,
// fork and copy-on-write.
//
// Semantics follow [Taming the Tail] "How the Architecture Works" (free block
// pool; a new block only when the last one is full), [vLLM PagedAttention FAQ]
// "Underlying Mechanism" (on-demand allocation, zero-copy forking with
// copy-on-write) and [KV-cache chapter] "PagedAttention: borrowing virtual
// memory..." and answer A6 (reference counts; a block rejoins the pool only at
// count zero; a private copy before the first write into a shared block).
//
// Design: everything is flat integer arrays.  The pool is a LIFO stack so a
// block freed a moment ago (likely still in L2) is reused first; the first
// fill follows the caller's free_order.  Appends are all-or-nothing: the
// number of blocks an append needs is computed before anything changes.
#include <cstdint>
#include <limits>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"
#include "status.h"

namespace pagedkv {
namespace {

struct Sequence {
  std::vector<int32_t> blocks;  // logical block i -> physical block
  int64_t len = 0;              // tokens stored
};

struct BlockManager {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<int32_t> ref;         // tables pointing at each block
  std::unordered_map<int64_t, Sequence> seqs;

  int32_t take() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }
  void drop(int32_t b) {
    if (--ref[b] == 0) free_stack.push_back(b);
  }
  int64_t blocks_for(int64_t len) const {
    return (len + block_size - 1) / block_size;
  }
};

BlockManager* as_bm(void* p) { return static_cast<BlockManager*>(p); }

}  // namespace
}  // namespace pagedkv

using pagedkv::BlockManager;
using pagedkv::Sequence;
using pagedkv::as_bm;
using pagedkv::fail;

extern "C" {

pa_status pa_bm_create(int num_blocks, int block_size,
                       const int32_t* free_order, void** out) {
  pagedkv::clear_error();
  if (!out) return fail(PA_ERR_INVALID_ARG, "pa_bm_create: bm is NULL");
  *out = nullptr;
  if (num_blocks < 0 || block_size <= 0)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_create: num_blocks=%d block_size=%d", num_blocks,
                block_size);
  BlockManager* bm = new (std::nothrow) BlockManager();
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_create: out of host memory");
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  bm->free_stack.resize(num_blocks);
  if (free_order) {
    std::vector<uint8_t> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return fail(PA_ERR_INVALID_ARG,
                    "pa_bm_create: free_order is not a permutation "
                    "(entry %d = %d)", i, b);
      }
      seen[b] = 1;
      bm->free_stack[num_blocks - 1 - i] = b;  // first handed out = [0]
    }
  } else {
    for (int i = 0; i < num_blocks; ++i)
      bm->free_stack[num_blocks - 1 - i] = i;
  }
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(void* bm) { delete as_bm(bm); }

pa_status pa_bm_add_seq(void* p, int64_t seq_id) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_add_seq: bm is NULL");
  if (!bm->seqs.emplace(seq_id, Sequence{}).second)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_add_seq: sequence %lld exists",
                static_cast<long long>(seq_id));
  return PA_OK;
}

pa_status pa_bm_fork(void* p, int64_t parent_id, int64_t child_id) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_fork: bm is NULL");
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_fork: no parent %lld",
                static_cast<long long>(parent_id));
  if (bm->seqs.count(child_id))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_fork: child %lld exists",
                static_cast<long long>(child_id));
  Sequence child = it->second;  // copy of table and length
  for (int32_t b : child.blocks) ++bm->ref[b];
  bm->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

pa_status pa_bm_append(void* p, int64_t seq_id, int n_tokens,
                       int64_t* slots_out, int32_t* cow_pairs_out, int max_cow,
                       int* num_cow_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_append: bm is NULL");
  if (n_tokens < 0 || (n_tokens > 0 && !slots_out) || !num_cow_out)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_append: n_tokens=%d slots_out=%p num_cow_out=%p",
                n_tokens, static_cast<void*>(slots_out),
                static_cast<void*>(num_cow_out));
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_append: no sequence %lld",
                static_cast<long long>(seq_id));
  Sequence& s = it->second;
  const int bs = bm->block_size;
  *num_cow_out = 0;
  if (n_tokens == 0) return PA_OK;

  // Blocks this append takes from the pool, decided before any change.
  const bool shared_partial =
      (s.len % bs) != 0 && bm->ref[s.blocks.back()] > 1;
  const int64_t fresh =
      bm->blocks_for(s.len + n_tokens) - static_cast<int64_t>(s.blocks.size());
  const int64_t need = fresh + (shared_partial ? 1 : 0);
  if (shared_partial && (max_cow < 1 || !cow_pairs_out))
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_append: sequence %lld needs a copy-on-write pair but "
                "max_cow=%d", static_cast<long long>(seq_id), max_cow);
  if (need > static_cast<int64_t>(bm->free_stack.size()))
    return fail(PA_ERR_NO_FREE_BLOCKS,
                "pa_bm_append: sequence %lld needs %lld blocks, %zu free",
                static_cast<long long>(seq_id), static_cast<long long>(need),
                bm->free_stack.size());

  if (shared_partial) {  // private copy of the shared, partly filled block
    int32_t src = s.blocks.back();
    int32_t dst = bm->take();
    bm->drop(src);
    s.blocks.back() = dst;
    cow_pairs_out[0] = src;
    cow_pairs_out[1] = dst;
    *num_cow_out = 1;
  }
  for (int i = 0; i < n_tokens; ++i) {
    const int64_t pos = s.len + i;
    const int64_t logical = pos / bs;
    if (logical == static_cast<int64_t>(s.blocks.size()))
      s.blocks.push_back(bm->take());
    slots_out[i] = static_cast<int64_t>(s.blocks[logical]) * bs + pos % bs;
  }
  s.len += n_tokens;
  return PA_OK;
}

pa_status pa_bm_append_batch(void* p, const int64_t* seq_ids,
                             const int32_t* n_tokens, int n,
                             int64_t* slots_out, int32_t* cow_pairs_out,
                             int max_cow, int* num_cow_out, int* num_done_out) {
  pagedkv::clear_error();
  if (!p || n < 0 || !num_cow_out || !num_done_out ||
      (n > 0 && (!seq_ids || !n_tokens)))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_append_batch: bad arguments");
  *num_cow_out = 0;
  *num_done_out = 0;
  int64_t offset = 0;
  for (int i = 0; i < n; ++i) {
    int ncow = 0;
    const int room = max_cow - *num_cow_out;
    pa_status st = pa_bm_append(
        p, seq_ids[i], n_tokens[i], slots_out ? slots_out + offset : nullptr,
        cow_pairs_out ? cow_pairs_out + 2 * *num_cow_out : nullptr,
        room > 0 ? room : 0, &ncow);
    if (st != PA_OK) return st;  // pa_bm_append changed nothing for seq i
    *num_cow_out += ncow;
    offset += n_tokens[i];
    *num_done_out = i + 1;
  }
  return PA_OK;
}

pa_status pa_bm_free_seq(void* p, int64_t seq_id) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_free_seq: bm is NULL");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_free_seq: no sequence %lld",
                static_cast<long long>(seq_id));
  for (int32_t b : it->second.blocks) bm->drop(b);
  bm->seqs.erase(it);
  return PA_OK;
}

pa_status pa_bm_truncate(void* p, int64_t seq_id, int64_t new_len) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_truncate: bm is NULL");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_truncate: no sequence %lld",
                static_cast<long long>(seq_id));
  Sequence& s = it->second;
  if (new_len < 0 || new_len > s.len)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_truncate: new_len %lld outside [0, %lld]",
                static_cast<long long>(new_len),
                static_cast<long long>(s.len));
  const int64_t keep = bm->blocks_for(new_len);
  while (static_cast<int64_t>(s.blocks.size()) > keep) {
    bm->drop(s.blocks.back());
    s.blocks.pop_back();
  }
  s.len = new_len;
  return PA_OK;
}

pa_status pa_bm_block_table(void* p, const int64_t* seq_ids, int n,
                            int max_blocks, int32_t* table_out,
                            int32_t* lens_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || n < 0 || max_blocks < 0 ||
      (n > 0 && (!seq_ids || !table_out || !lens_out)))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_block_table: bad arguments");
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end())
      return fail(PA_ERR_INVALID_ARG, "pa_bm_block_table: no sequence %lld",
                  static_cast<long long>(seq_ids[i]));
    const Sequence& s = it->second;
    if (static_cast<int64_t>(s.blocks.size()) > max_blocks ||
        s.len > std::numeric_limits<int32_t>::max())
      return fail(PA_ERR_INVALID_ARG,
                  "pa_bm_block_table: sequence %lld holds %zu blocks, "
                  "table has %d columns", static_cast<long long>(seq_ids[i]),
                  s.blocks.size(), max_blocks);
    int32_t* row = table_out + static_cast<int64_t>(i) * max_blocks;
    const int nb = static_cast<int>(s.blocks.size());
    for (int j = 0; j < nb; ++j) row[j] = s.blocks[j];
    for (int j = nb; j < max_blocks; ++j) row[j] = -1;
    lens_out[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

int pa_bm_num_free(void* p) {
  BlockManager* bm = as_bm(p);
  return bm ? static_cast<int>(bm->free_stack.size()) : -1;
}

int pa_bm_refcount(void* p, int block) {
  BlockManager* bm = as_bm(p);
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->ref[block];
}

int64_t pa_bm_seq_len(void* p, int64_t seq_id) {
  BlockManager* bm = as_bm(p);
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

int pa_bm_num_seq_blocks(void* p, int64_t seq_id) {
  BlockManager* bm = as_bm(p);
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : static_cast<int>(it->second.blocks.size());
}

}  // extern "C"
