// Host block manager: free pool, per-sequence block tables, reference counts,
// fork, copy-on-write, and a radix-tree prefix cache.
//
// Semantics follow [Taming the Tail] "How the Architecture Works" (free block
// pool; a new block only when the last one is full), [vLLM PagedAttention FAQ]
// "Underlying Mechanism" (on-demand allocation, zero-copy forking with
// copy-on-write) and [KV-cache chapter] "PagedAttention: borrowing virtual
// memory..." and answer A6 (reference counts; a block rejoins the pool only at
// count zero; a private copy before the first write into a shared block).
//
// Prefix cache ([KV-cache chapter] "RadixAttention: caching, not just packing,
// the prefix"): cached token sequences form a tree with one node per full
// block, keyed by that block's tokens under its parent.  A request walks the
// tree and references every matched block instead of recomputing it.  The
// cache holds one reference per cached block; a cached block that only the
// cache references and that has no cached children is an evictable leaf.
// When an append needs more blocks than the pool has, evictable leaves go
// least recently used first (a logical clock stamps each match / insert
// walk), and a leaf's parent may become evictable in turn.  Reference counts
// keep every block a sequence still uses out of reach.
//
// Swap ([Taming the Tail] "Infrastructure Scale", preemption by moving a
// request's KV cache to CPU RAM): a second pool of host blocks.  A group of
// sequences is swapped at once, so a block the group shares crosses the link
// once: each distinct device block of the group gets one host block carrying
// the group's references, and the device block keeps the references other
// tables (or the cache) hold.  Swap-in is the mirror image and allocates
// device blocks like an append (evicting cache leaves).  Both are all or
// nothing and return the (source, destination) pairs pa_swap_blocks copies.
//
// Design: everything is flat integer arrays.  The pool is a LIFO stack so a
// block freed a moment ago (likely still in L2) is reused first; the first
// fill follows the caller's free_order.  Appends are all-or-nothing: the
// number of blocks an append needs is computed before anything changes, and
// an append that eviction cannot satisfy puts back what it evicted.  Cache
// nodes live in one array; children are found through a hash map keyed by
// (parent node, block tokens); evictable leaves sit in an ordered set by
// stamp, kept current whenever a count, a stamp or a child count changes.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <limits>
#include <new>
#include <set>
#include <unordered_map>
#include <utility>
#include <vector>

#include "pagedkv.h"
#include "status.h"

namespace pagedkv {
namespace {

struct Sequence {
  std::vector<int32_t> blocks;  // logical block i -> physical block
  int64_t len = 0;              // tokens stored
  bool swapped = false;         // blocks name host-pool blocks
};

struct Node {
  int32_t block = -1;   // -1: the root, or a released node
  int32_t parent = -1;
  int32_t n_children = 0;
  int64_t last = 0;     // stamp of the last walk through this node
  uint64_t hash = 0;    // of (parent, tokens)
  bool in_lru = false;
  int64_t lru_stamp = 0;
  std::vector<int32_t> tokens;
};

uint64_t mix(uint64_t h, uint64_t v) {
  // splitmix64 finaliser over the running value
  h ^= v + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
  h ^= h >> 30;
  h *= 0xbf58476d1ce4e5b9ull;
  h ^= h >> 27;
  h *= 0x94d049bb133111ebull;
  return h ^ (h >> 31);
}

uint64_t key_hash(int32_t parent, const int32_t* tokens, int n) {
  uint64_t h = mix(0x2545f4914f6cdd1dull, static_cast<uint32_t>(parent));
  for (int i = 0; i < n; ++i) h = mix(h, static_cast<uint32_t>(tokens[i]));
  return h;
}

struct BlockManager {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<int32_t> ref;         // tables (+1 if cached) per block
  std::unordered_map<int64_t, Sequence> seqs;

  // prefix cache
  std::vector<Node> nodes{Node{}};  // [0] = root
  std::vector<int32_t> free_nodes;
  std::vector<int32_t> node_of;     // block -> cache node or -1
  std::unordered_multimap<uint64_t, int32_t> children;
  std::set<std::pair<int64_t, int32_t>> lru;  // evictable leaves by stamp
  int64_t clock = 0;
  int num_cached = 0;

  // host pool for swapped-out sequences
  int num_host_blocks = 0;
  std::vector<int32_t> host_free;  // top = back()
  std::vector<int32_t> host_ref;

  int32_t take() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }
  void drop(int32_t b) {
    if (--ref[b] == 0)
      free_stack.push_back(b);
    else if (node_of[b] >= 0)
      refresh(node_of[b]);
  }
  void add_ref(int32_t b) {
    ++ref[b];
    if (node_of[b] >= 0) refresh(node_of[b]);
  }
  int64_t blocks_for(int64_t len) const {
    return (len + block_size - 1) / block_size;
  }

  // Keep node n's membership of the evictable-leaf set current.
  void refresh(int32_t n) {
    Node& x = nodes[n];
    const bool want = x.block >= 0 && x.n_children == 0 && ref[x.block] == 1;
    if (x.in_lru && (!want || x.lru_stamp != x.last)) {
      lru.erase({x.lru_stamp, n});
      x.in_lru = false;
    }
    if (want && !x.in_lru) {
      lru.insert({x.last, n});
      x.lru_stamp = x.last;
      x.in_lru = true;
    }
  }
  void touch(int32_t n, int64_t now) {
    nodes[n].last = now;
    refresh(n);
  }

  int32_t find_child(int32_t parent, const int32_t* tokens) const {
    const uint64_t h = key_hash(parent, tokens, block_size);
    auto range = children.equal_range(h);
    for (auto it = range.first; it != range.second; ++it) {
      const Node& c = nodes[it->second];
      if (c.parent == parent &&
          std::memcmp(c.tokens.data(), tokens, sizeof(int32_t) * block_size) ==
              0)
        return it->second;
    }
    return -1;
  }

  // New node for block b (the cache takes a reference) under parent.
  int32_t add_node(int32_t parent, const int32_t* tokens, int32_t b,
                   int64_t now) {
    int32_t n;
    if (!free_nodes.empty()) {
      n = free_nodes.back();
      free_nodes.pop_back();
    } else {
      n = static_cast<int32_t>(nodes.size());
      nodes.emplace_back();
    }
    Node& x = nodes[n];
    x.block = b;
    x.parent = parent;
    x.n_children = 0;
    x.last = now;
    x.in_lru = false;
    x.tokens.assign(tokens, tokens + block_size);
    x.hash = key_hash(parent, tokens, block_size);
    children.emplace(x.hash, n);
    ++nodes[parent].n_children;
    if (parent != 0) refresh(parent);
    node_of[b] = n;
    ++num_cached;
    add_ref(b);
    return n;
  }

  // Remove evictable leaf n from the tree; its block returns to the pool.
  // The node keeps its fields so relink() can undo this.
  void unlink(int32_t n) {
    Node& x = nodes[n];
    lru.erase({x.lru_stamp, n});
    x.in_lru = false;
    auto range = children.equal_range(x.hash);
    for (auto it = range.first; it != range.second; ++it)
      if (it->second == n) {
        children.erase(it);
        break;
      }
    --nodes[x.parent].n_children;
    if (x.parent != 0) refresh(x.parent);
    node_of[x.block] = -1;
    --num_cached;
    drop(x.block);  // 1 -> 0: back to the pool
  }
  void relink(int32_t n) {  // exact inverse of the last unlink()
    Node& x = nodes[n];
    free_stack.pop_back();  // x.block, pushed by unlink
    ref[x.block] = 1;
    node_of[x.block] = n;
    ++num_cached;
    children.emplace(x.hash, n);
    ++nodes[x.parent].n_children;
    if (x.parent != 0) refresh(x.parent);
    refresh(n);
  }
  void release_node(int32_t n) {
    nodes[n].block = -1;
    nodes[n].tokens.clear();
    free_nodes.push_back(n);
  }

  // Make at least `need` blocks free by evicting leaves, oldest first.  All
  // or nothing: if the cache cannot supply enough, nothing is evicted.
  bool ensure_free(int64_t need) {
    if (need <= static_cast<int64_t>(free_stack.size())) return true;
    std::vector<int32_t> evicted;
    while (static_cast<int64_t>(free_stack.size()) < need && !lru.empty()) {
      const int32_t n = lru.begin()->second;
      unlink(n);
      evicted.push_back(n);
    }
    if (static_cast<int64_t>(free_stack.size()) >= need) {
      for (int32_t n : evicted) release_node(n);
      return true;
    }
    for (auto it = evicted.rbegin(); it != evicted.rend(); ++it) relink(*it);
    return false;
  }
};

BlockManager* as_bm(void* p) { return static_cast<BlockManager*>(p); }

}  // namespace
}  // namespace pagedkv

using pagedkv::BlockManager;
using pagedkv::Node;
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
  bm->node_of.assign(num_blocks, -1);
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
  if (it->second.swapped)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_fork: parent %lld is swapped out",
                static_cast<long long>(parent_id));
  Sequence child = it->second;  // copy of table and length
  for (int32_t b : child.blocks) bm->add_ref(b);
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
  if (s.swapped)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_append: sequence %lld is swapped out",
                static_cast<long long>(seq_id));
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
  if (!bm->ensure_free(need))
    return fail(PA_ERR_NO_FREE_BLOCKS,
                "pa_bm_append: sequence %lld needs %lld blocks, %zu free "
                "after evicting every evictable cached block",
                static_cast<long long>(seq_id), static_cast<long long>(need),
                bm->free_stack.size() + bm->lru.size());

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
  if (it->second.swapped) {
    for (int32_t h : it->second.blocks)
      if (--bm->host_ref[h] == 0) bm->host_free.push_back(h);
  } else {
    for (int32_t b : it->second.blocks) bm->drop(b);
  }
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
  if (s.swapped)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_truncate: sequence %lld is swapped out",
                static_cast<long long>(seq_id));
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
    if (s.swapped)
      return fail(PA_ERR_INVALID_ARG,
                  "pa_bm_block_table: sequence %lld is swapped out",
                  static_cast<long long>(seq_ids[i]));
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

int pa_bm_num_used(void* p) {
  BlockManager* bm = as_bm(p);
  return bm ? bm->num_blocks - static_cast<int>(bm->free_stack.size()) : -1;
}

int64_t pa_pool_blocks(uint64_t bytes, int num_layers, int num_kv_heads,
                       int head_dim, int block_size, pa_dtype dtype) {
  pagedkv::clear_error();
  if (num_layers <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || (dtype != PA_F16 && dtype != PA_BF16)) {
    fail(PA_ERR_INVALID_ARG,
         "pa_pool_blocks: num_layers=%d num_kv_heads=%d head_dim=%d "
         "block_size=%d dtype=%d", num_layers, num_kv_heads, head_dim,
         block_size, static_cast<int>(dtype));
    return -1;
  }
  // K and V, every layer, every KV head, block_size tokens, 2-byte elements.
  const uint64_t per_block = 2ull * num_layers * num_kv_heads * head_dim *
                             block_size * 2ull;
  return static_cast<int64_t>(bytes / per_block);
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

pa_status pa_bm_match_prefix(void* p, int64_t seq_id, const int32_t* tokens,
                             int64_t n_tokens, int64_t* matched_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || n_tokens < 0 || (n_tokens > 0 && !tokens) || !matched_out)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_match_prefix: bad arguments");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_match_prefix: no sequence %lld",
                static_cast<long long>(seq_id));
  Sequence& s = it->second;
  if (s.len != 0 || !s.blocks.empty() || s.swapped)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_match_prefix: sequence %lld is not empty or is "
                "swapped out",
                static_cast<long long>(seq_id));
  const int bs = bm->block_size;
  const int64_t now = ++bm->clock;
  int32_t node = 0;
  for (int64_t i = 0; i < n_tokens / bs; ++i) {
    const int32_t c = bm->find_child(node, tokens + i * bs);
    if (c < 0) break;
    bm->touch(c, now);
    s.blocks.push_back(bm->nodes[c].block);
    bm->add_ref(bm->nodes[c].block);
    node = c;
  }
  s.len = static_cast<int64_t>(s.blocks.size()) * bs;
  *matched_out = s.len;
  return PA_OK;
}

pa_status pa_bm_cache_insert(void* p, int64_t seq_id, const int32_t* tokens,
                             int64_t n_tokens) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || n_tokens < 0 || (n_tokens > 0 && !tokens))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_cache_insert: bad arguments");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_cache_insert: no sequence %lld",
                static_cast<long long>(seq_id));
  const Sequence& s = it->second;
  if (s.swapped)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_cache_insert: sequence %lld is swapped out",
                static_cast<long long>(seq_id));
  if (n_tokens > s.len)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_cache_insert: %lld tokens, sequence %lld holds %lld",
                static_cast<long long>(n_tokens),
                static_cast<long long>(seq_id), static_cast<long long>(s.len));
  const int bs = bm->block_size;
  const int64_t n_full = n_tokens / bs;
  // Check first, so a refused insert changes nothing: a block may sit in the
  // tree only under its own tokens.
  int32_t node = 0;
  bool creating = false;
  for (int64_t i = 0; i < n_full; ++i) {
    const int32_t c = creating ? -1 : bm->find_child(node, tokens + i * bs);
    const int32_t placed = bm->node_of[s.blocks[i]];
    if (c < 0) {
      creating = true;
      if (placed >= 0)
        return fail(PA_ERR_INVALID_ARG,
                    "pa_bm_cache_insert: block %d of sequence %lld is cached "
                    "under other tokens", s.blocks[i],
                    static_cast<long long>(seq_id));
    } else {
      if (placed >= 0 && placed != c)
        return fail(PA_ERR_INVALID_ARG,
                    "pa_bm_cache_insert: block %d of sequence %lld is cached "
                    "under other tokens", s.blocks[i],
                    static_cast<long long>(seq_id));
      node = c;
    }
  }
  const int64_t now = ++bm->clock;
  node = 0;
  for (int64_t i = 0; i < n_full; ++i) {
    int32_t c = bm->find_child(node, tokens + i * bs);
    if (c < 0)
      c = bm->add_node(node, tokens + i * bs, s.blocks[i], now);
    else
      bm->touch(c, now);
    node = c;
  }
  return PA_OK;
}

pa_status pa_bm_cache_evict(void* p, int max_blocks, int* evicted_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || max_blocks < 0 || !evicted_out)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_cache_evict: bad arguments");
  int done = 0;
  while (done < max_blocks && !bm->lru.empty()) {
    const int32_t n = bm->lru.begin()->second;
    bm->unlink(n);
    bm->release_node(n);
    ++done;
  }
  *evicted_out = done;
  return PA_OK;
}

int pa_bm_num_cached(void* p) {
  BlockManager* bm = as_bm(p);
  return bm ? bm->num_cached : -1;
}

pa_status pa_bm_cache_nodes(void* p, int max_nodes, int32_t* parent_out,
                            int32_t* block_out, int32_t* tokens_out,
                            int* n_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || max_nodes < 0 || !n_out ||
      (max_nodes > 0 && (!parent_out || !block_out || !tokens_out)))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_cache_nodes: bad arguments");
  if (bm->num_cached > max_nodes)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_cache_nodes: %d cached blocks, room for %d",
                bm->num_cached, max_nodes);
  // Breadth-first from the root, so every parent precedes its children.
  std::vector<std::vector<int32_t>> kids(bm->nodes.size());
  for (size_t n = 1; n < bm->nodes.size(); ++n)
    if (bm->nodes[n].block >= 0 && bm->node_of[bm->nodes[n].block] ==
                                       static_cast<int32_t>(n))
      kids[bm->nodes[n].parent].push_back(static_cast<int32_t>(n));
  std::vector<int32_t> index(bm->nodes.size(), -1);
  std::vector<int32_t> queue{0};
  int out = 0;
  for (size_t q = 0; q < queue.size(); ++q) {
    for (int32_t c : kids[queue[q]]) {
      const Node& x = bm->nodes[c];
      index[c] = out;
      parent_out[out] = x.parent == 0 ? -1 : index[x.parent];
      block_out[out] = x.block;
      std::memcpy(tokens_out + static_cast<int64_t>(out) * bm->block_size,
                  x.tokens.data(), sizeof(int32_t) * bm->block_size);
      ++out;
      queue.push_back(c);
    }
  }
  *n_out = out;
  return PA_OK;
}

pa_status pa_bm_set_host_blocks(void* p, int num_host_blocks) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || num_host_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_set_host_blocks: bad arguments");
  if (static_cast<int>(bm->host_free.size()) != bm->num_host_blocks)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_set_host_blocks: %d host blocks are in use",
                bm->num_host_blocks -
                    static_cast<int>(bm->host_free.size()));
  bm->num_host_blocks = num_host_blocks;
  bm->host_ref.assign(num_host_blocks, 0);
  bm->host_free.resize(num_host_blocks);
  for (int i = 0; i < num_host_blocks; ++i)
    bm->host_free[num_host_blocks - 1 - i] = i;  // first handed out = 0
  return PA_OK;
}

}  // extern "C"

namespace {

// Distinct blocks of the group's tables in order of first use, with the
// group's reference count of each.  `seen` is indexed by block id.
void group_uses(const std::vector<Sequence*>& group, int pool_size,
                std::vector<int32_t>* order, std::vector<int32_t>* count) {
  count->assign(pool_size, 0);
  order->clear();
  for (const Sequence* s : group)
    for (int32_t b : s->blocks)
      if ((*count)[b]++ == 0) order->push_back(b);
}

// Validate the group: known, distinct, and swapped (or not) as required.
pa_status collect_group(BlockManager* bm, const int64_t* seq_ids, int n,
                        bool want_swapped, const char* fn,
                        std::vector<Sequence*>* group) {
  group->clear();
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end())
      return fail(PA_ERR_INVALID_ARG, "%s: no sequence %lld", fn,
                  static_cast<long long>(seq_ids[i]));
    if (it->second.swapped != want_swapped)
      return fail(PA_ERR_INVALID_ARG, "%s: sequence %lld is %s", fn,
                  static_cast<long long>(seq_ids[i]),
                  want_swapped ? "not swapped out" : "already swapped out");
    for (const Sequence* g : *group)
      if (g == &it->second)
        return fail(PA_ERR_INVALID_ARG, "%s: sequence %lld listed twice", fn,
                    static_cast<long long>(seq_ids[i]));
    group->push_back(&it->second);
  }
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_bm_swap_out(void* p, const int64_t* seq_ids, int n,
                         int32_t* pairs_out, int max_pairs,
                         int* num_pairs_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || n < 0 || (n > 0 && !seq_ids) || !num_pairs_out ||
      max_pairs < 0 || (max_pairs > 0 && !pairs_out))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_swap_out: bad arguments");
  *num_pairs_out = 0;
  std::vector<Sequence*> group;
  pa_status st = collect_group(bm, seq_ids, n, false, "pa_bm_swap_out",
                               &group);
  if (st != PA_OK) return st;
  std::vector<int32_t> order, count;
  group_uses(group, bm->num_blocks, &order, &count);
  const int distinct = static_cast<int>(order.size());
  if (distinct > max_pairs)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_swap_out: %d pairs, room for %d", distinct, max_pairs);
  if (distinct > static_cast<int>(bm->host_free.size()))
    return fail(PA_ERR_NO_FREE_BLOCKS,
                "pa_bm_swap_out: %d host blocks needed, %zu free", distinct,
                bm->host_free.size());
  std::vector<int32_t> to_host(bm->num_blocks, -1);
  for (int i = 0; i < distinct; ++i) {
    const int32_t d = order[i];
    const int32_t h = bm->host_free.back();
    bm->host_free.pop_back();
    bm->host_ref[h] = count[d];
    to_host[d] = h;
    pairs_out[2 * i] = d;
    pairs_out[2 * i + 1] = h;
  }
  for (int32_t d : order)
    for (int r = 0; r < count[d]; ++r) bm->drop(d);
  for (Sequence* s : group) {
    for (int32_t& b : s->blocks) b = to_host[b];
    s->swapped = true;
  }
  *num_pairs_out = distinct;
  return PA_OK;
}

pa_status pa_bm_swap_in(void* p, const int64_t* seq_ids, int n,
                        int32_t* pairs_out, int max_pairs,
                        int* num_pairs_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || n < 0 || (n > 0 && !seq_ids) || !num_pairs_out ||
      max_pairs < 0 || (max_pairs > 0 && !pairs_out))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_swap_in: bad arguments");
  *num_pairs_out = 0;
  std::vector<Sequence*> group;
  pa_status st = collect_group(bm, seq_ids, n, true, "pa_bm_swap_in",
                               &group);
  if (st != PA_OK) return st;
  std::vector<int32_t> order, count;
  group_uses(group, bm->num_host_blocks, &order, &count);
  const int distinct = static_cast<int>(order.size());
  if (distinct > max_pairs)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_swap_in: %d pairs, room for %d", distinct, max_pairs);
  if (!bm->ensure_free(distinct))
    return fail(PA_ERR_NO_FREE_BLOCKS,
                "pa_bm_swap_in: %d device blocks needed, %zu free after "
                "evicting every evictable cached block", distinct,
                bm->free_stack.size() + bm->lru.size());
  std::vector<int32_t> to_dev(bm->num_host_blocks, -1);
  for (int i = 0; i < distinct; ++i) {
    const int32_t h = order[i];
    const int32_t d = bm->take();
    bm->ref[d] = count[h];
    to_dev[h] = d;
    pairs_out[2 * i] = h;
    pairs_out[2 * i + 1] = d;
  }
  for (int32_t h : order) {
    bm->host_ref[h] -= count[h];
    if (bm->host_ref[h] == 0) bm->host_free.push_back(h);
  }
  for (Sequence* s : group) {
    for (int32_t& b : s->blocks) b = to_dev[b];
    s->swapped = false;
  }
  *num_pairs_out = distinct;
  return PA_OK;
}

int pa_bm_num_free_host(void* p) {
  BlockManager* bm = as_bm(p);
  return bm ? static_cast<int>(bm->host_free.size()) : -1;
}

int pa_bm_host_refcount(void* p, int block) {
  BlockManager* bm = as_bm(p);
  if (!bm || block < 0 || block >= bm->num_host_blocks) return -1;
  return bm->host_ref[block];
}

int pa_bm_is_swapped(void* p, int64_t seq_id) {
  BlockManager* bm = as_bm(p);
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : (it->second.swapped ? 1 : 0);
}

pa_status pa_bm_seq_blocks(void* p, int64_t seq_id, int32_t* blocks_out,
                           int max_blocks, int* n_out) {
  pagedkv::clear_error();
  BlockManager* bm = as_bm(p);
  if (!bm || !n_out || max_blocks < 0 || (max_blocks > 0 && !blocks_out))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_seq_blocks: bad arguments");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end())
    return fail(PA_ERR_INVALID_ARG, "pa_bm_seq_blocks: no sequence %lld",
                static_cast<long long>(seq_id));
  const std::vector<int32_t>& b = it->second.blocks;
  if (static_cast<int64_t>(b.size()) > max_blocks)
    return fail(PA_ERR_INVALID_ARG,
                "pa_bm_seq_blocks: %zu blocks, room for %d", b.size(),
                max_blocks);
  std::copy(b.begin(), b.end(), blocks_out);
  *n_out = static_cast<int>(b.size());
  return PA_OK;
}

}  // extern "C"
