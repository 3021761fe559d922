"""Reference model of a radix-tree prefix cache over paged KV blocks.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What it models ([KV-cache chapter] "RadixAttention: caching, not just
packing, the prefix"): all cached token sequences form a radix tree, in which
sequences with a common prefix share the path from the root down to where
they diverge.  A new request walks the tree with its tokens; every matched
token already has its K/V in GPU memory and is referenced, not recomputed;
only the tokens past the divergence need a prefill pass.  When memory runs
low, leaves are trimmed least recently used first, and reference counts keep
any branch still referenced by a running request from being evicted.

Readings where the pages leave a step open (each stated so a reader can check
them):

* Granularity.  K/V live in blocks of ``block_size`` tokens, and a block is
  the unit that can be referenced by several tables.  The tree therefore
  holds whole blocks: one node per full block, keyed by that block's tokens
  under its parent.  A chain of single-child nodes is the radix tree's
  compressed edge written out block by block; matching and eviction give the
  same result either way when a block is the smallest thing freed.  The last,
  partly filled block of a sequence is never cached.
* References.  The cache holds one reference on every block it stores, on
  top of the tables that point at it ([KV-cache chapter] "PagedAttention:
  borrowing virtual memory ..." reference counts).  A cached block whose only
  reference is the cache's, and that has no cached children, is an
  evictable leaf.
* Recency.  A logical clock advances once per match and once per insert; the
  walk stamps every node on its path with the new time.  Eviction removes the
  evictable leaf with the oldest stamp; its parent may then become a leaf.
  Two leaves never share a stamp (nodes stamped in one walk form one chain),
  so the order is unique.
* When.  Blocks are evicted only when an append needs more blocks than the
  pool has free (or on an explicit ``evict``).  An append that could not be
  satisfied even after evicting every evictable block raises ``NoFreeBlocks``
  and changes nothing, cache included.
* Duplicates.  If a request computed a block whose tokens are already cached
  at that place in the tree, the cached node is kept and the request keeps
  its own copy outside the cache; the walk continues below the cached node.
"""
from __future__ import annotations

from .block_model import BlockModel, NoFreeBlocks


class _Node:
    __slots__ = ("key", "block", "parent", "children", "last")

    def __init__(self, key, block, parent, last):
        self.key = key
        self.block = block
        self.parent = parent
        self.children = {}
        self.last = last


class PrefixCacheModel(BlockModel):
    """BlockModel plus the radix-tree prefix cache described above."""

    def __init__(self, num_blocks: int, block_size: int):
        super().__init__(num_blocks, block_size)
        self.root = _Node(None, None, None, 0)
        self.clock = 0
        self.node_of = {}          # cached block -> its node

    # -- helpers --------------------------------------------------------------
    def _tick(self) -> int:
        self.clock += 1
        return self.clock

    def _key(self, tokens, i):
        bs = self.block_size
        return tuple(int(t) for t in tokens[i * bs:(i + 1) * bs])

    def _nodes(self):
        stack, out = list(self.root.children.values()), []
        while stack:
            n = stack.pop()
            out.append(n)
            stack.extend(n.children.values())
        return out

    def num_cached(self) -> int:
        return len(self.node_of)

    def cached_paths(self):
        """Every cached block as the tuple of token keys from the root."""
        paths = set()
        for n in self._nodes():
            keys, m = [], n
            while m is not self.root:
                keys.append(m.key)
                m = m.parent
            paths.add(tuple(reversed(keys)))
        return paths

    def num_evictable(self) -> int:
        """Blocks that evicting leaf after leaf could free: cached nodes
        whose own block and whole subtree are held by the cache alone."""
        def count(node):
            total, all_free = 0, True
            for c in node.children.values():
                sub, free = count(c)
                total += sub
                all_free &= free
            if node is self.root:
                return total, all_free
            mine = all_free and self.ref[node.block] == 1
            return total + (1 if mine else 0), mine
        return count(self.root)[0]

    # -- cache operations ---------------------------------------------------------
    def match(self, seq, tokens) -> int:
        """Attach the longest cached run of full blocks that starts
        ``tokens`` to the new, empty sequence ``seq``; returns the number of
        tokens it covers (a multiple of the block size)."""
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        if self.lens[seq] or self.tables[seq]:
            raise ValueError("match needs an empty sequence")
        now = self._tick()
        node = self.root
        for i in range(len(tokens) // self.block_size):
            child = node.children.get(self._key(tokens, i))
            if child is None:
                break
            child.last = now
            self.tables[seq].append(child.block)
            self.ref[child.block] += 1
            node = child
        self.lens[seq] = len(self.tables[seq]) * self.block_size
        return self.lens[seq]

    def insert(self, seq, tokens) -> None:
        """Cache the full blocks among the first ``len(tokens)`` tokens of
        ``seq`` (``tokens`` are that sequence's tokens)."""
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        if len(tokens) > self.lens[seq]:
            raise ValueError("more tokens than the sequence holds")
        table = self.tables[seq]
        n_full = len(tokens) // self.block_size
        # check first, so a refused insert changes nothing: a block may sit
        # in the tree only under its own tokens
        node, creating = self.root, False
        for i in range(n_full):
            child = None if creating else node.children.get(
                self._key(tokens, i))
            placed = self.node_of.get(table[i])
            if child is None:
                creating = True
                if placed is not None:
                    raise ValueError("block is cached under other tokens")
            else:
                if placed is not None and placed is not child:
                    raise ValueError("block is cached under other tokens")
                node = child
        now = self._tick()
        node = self.root
        for i in range(n_full):
            key = self._key(tokens, i)
            child = node.children.get(key)
            if child is None:
                blk = table[i]
                child = _Node(key, blk, node, now)
                node.children[key] = child
                self.node_of[blk] = child
                self.ref[blk] += 1
            child.last = now
            node = child

    def _evict_one(self) -> bool:
        best = None
        for n in self._nodes():
            if n.children or self.ref[n.block] != 1:
                continue
            if best is None or n.last < best.last:
                best = n
        if best is None:
            return False
        del best.parent.children[best.key]
        del self.node_of[best.block]
        self._drop(best.block)
        return True

    def evict(self, n_blocks: int) -> int:
        """Evict up to ``n_blocks`` leaves, least recently used first;
        returns how many were evicted."""
        done = 0
        while done < n_blocks and self._evict_one():
            done += 1
        return done

    # -- allocation with eviction ------------------------------------------------
    def append(self, seq, n_tokens: int):
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        if n_tokens < 0:
            raise ValueError("negative token count")
        short = self.blocks_needed(seq, n_tokens) - len(self.free)
        if short > 0:
            if short > self.num_evictable():
                raise NoFreeBlocks(f"sequence {seq} needs more blocks")
            evicted = self.evict(short)
            assert evicted == short
        return super().append(seq, n_tokens)
