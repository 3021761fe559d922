"""Reference model of swapping sequences' KV blocks to host memory and back.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What it models ([Taming the Tail] "Infrastructure Scale", preemption
policy): when the GPU runs out of physical blocks, a request can be paused
and its KV cache moved to CPU RAM, to be brought back later.  The pages pose
the choice (swap or recompute) and fix nothing else, so every step below is
a reading, stated so it can be checked:

* A second pool of ``num_host_blocks`` blocks lives in host memory.  A
  swapped-out sequence keeps its table, but its entries name host blocks.
* Swapping works on a group of sequences at once, so blocks the group shares
  cross the link once: for every distinct device block the group's tables
  use, one host block is taken, holding as many references as the group has
  to it; the device block loses those references and returns to the pool
  when none are left (a block another sequence, or the prefix cache, still
  holds stays on the device).  The copies to run are (device, host) pairs in
  order of first use (sequences in the order given, logical blocks in
  order).  Swapping back in is the mirror image with (host, device) pairs;
  device blocks come from the pool, evicting prefix-cache leaves like any
  other allocation.
* All or nothing: if the target pool cannot supply every block, the call
  raises ``NoFreeBlocks`` and changes nothing.
* A swapped-out sequence can only be swapped in or freed; appending to,
  forking, truncating, caching or reading its table is refused.
* The copies run in stream order before any later write into the freed
  blocks, so the data moved is exactly the bytes of the source blocks.
"""
from __future__ import annotations

from .block_model import NoFreeBlocks
from .prefix_cache import PrefixCacheModel


class SwapModel(PrefixCacheModel):
    def __init__(self, num_blocks: int, block_size: int,
                 num_host_blocks: int = 0):
        super().__init__(num_blocks, block_size)
        self.num_host_blocks = num_host_blocks
        self.host_free = set(range(num_host_blocks))
        self.host_ref = {}
        self.swapped = set()

    def num_free_host(self) -> int:
        return len(self.host_free)

    def host_refcount(self, blk: int) -> int:
        return self.host_ref.get(blk, 0)

    def _check_resident(self, seq):
        if seq in self.swapped:
            raise ValueError(f"sequence {seq} is swapped out")

    # refuse the operations a swapped sequence cannot take
    def append(self, seq, n_tokens: int):
        self._check_resident(seq)
        return super().append(seq, n_tokens)

    def fork(self, parent, child) -> None:
        self._check_resident(parent)
        super().fork(parent, child)

    def truncate(self, seq, new_len: int) -> None:
        self._check_resident(seq)
        super().truncate(seq, new_len)

    def insert(self, seq, tokens) -> None:
        self._check_resident(seq)
        super().insert(seq, tokens)

    def match(self, seq, tokens) -> int:
        self._check_resident(seq)
        return super().match(seq, tokens)

    def free_seq(self, seq) -> None:
        if seq in self.swapped:
            for blk in self.tables.pop(seq):
                self.host_ref[blk] -= 1
                if self.host_ref[blk] == 0:
                    del self.host_ref[blk]
                    self.host_free.add(blk)
            del self.lens[seq]
            self.swapped.discard(seq)
            return
        super().free_seq(seq)

    @staticmethod
    def _group_uses(tables, seqs):
        """Distinct blocks of the group in order of first use, with the
        number of the group's references to each."""
        order, count = [], {}
        for s in seqs:
            for blk in tables[s]:
                if blk not in count:
                    order.append(blk)
                    count[blk] = 0
                count[blk] += 1
        return order, count

    def swap_out(self, seqs):
        seqs = list(seqs)
        if len(set(seqs)) != len(seqs):
            raise ValueError("a sequence is listed twice")
        for s in seqs:
            if s not in self.tables:
                raise KeyError(f"no sequence {s}")
            self._check_resident(s)
        order, count = self._group_uses(self.tables, seqs)
        if len(order) > len(self.host_free):
            raise NoFreeBlocks("host pool cannot take the group")
        to_host, pairs = {}, []
        for blk in order:
            h = min(self.host_free)
            self.host_free.remove(h)
            self.host_ref[h] = count[blk]
            to_host[blk] = h
            pairs.append((blk, h))
        for blk in order:                 # drop after every copy is decided
            for _ in range(count[blk]):
                self._drop(blk)
        for s in seqs:
            self.tables[s] = [to_host[b] for b in self.tables[s]]
            self.swapped.add(s)
        return pairs

    def swap_in(self, seqs):
        seqs = list(seqs)
        if len(set(seqs)) != len(seqs):
            raise ValueError("a sequence is listed twice")
        for s in seqs:
            if s not in self.swapped:
                raise ValueError(f"sequence {s} is not swapped out")
        order, count = self._group_uses(self.tables, seqs)
        short = len(order) - len(self.free)
        if short > 0:
            if short > self.num_evictable():
                raise NoFreeBlocks("device pool cannot take the group")
            assert self.evict(short) == short
        to_dev, pairs = {}, []
        for h in order:
            d = self._take()
            self.ref[d] = count[h]
            to_dev[h] = d
            pairs.append((h, d))
        for h in order:
            self.host_ref[h] -= count[h]
            if self.host_ref[h] == 0:
                del self.host_ref[h]
                self.host_free.add(h)
        for s in seqs:
            self.tables[s] = [to_dev[h] for h in self.tables[s]]
            self.swapped.discard(s)
        return pairs
