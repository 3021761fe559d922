"""Reference model of the paged KV-cache block manager, in plain Python.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Semantics, each taken from the pages:

* Pool and tables -- [Taming the Tail] "How the Architecture Works": a free
  block pool, per-sequence logical blocks mapped to physical blocks anywhere
  in the pool through a block table.
* On-demand allocation -- [Taming the Tail] same section and [vLLM
  PagedAttention FAQ] "Dynamic On-Demand Page Allocation": a new block is taken
  from the pool only when the current last block is full (with block size 16,
  the 17th token opens the second block).
* Reference counts -- [KV-cache chapter] "PagedAttention: borrowing virtual
  memory from the operating system" and answer A6: a block shared by several
  tables carries a count of the tables pointing at it, and goes back to the
  pool only when that count reaches zero.
* Copy-on-write -- [KV-cache chapter] same section, [Taming the Tail]
  "Complex Memory Sharing" and [vLLM PagedAttention FAQ] "Zero-Copy Forking &
  Parallel Sampling": a sequence about to write into a block that other
  tables also point at first gets a private copy of it.
* Fork -- [vLLM PagedAttention FAQ] "Zero-Copy Forking": a child shares all
  of its parent's blocks.
* Discarding speculative blocks -- [Taming the Tail] "The Future: Speculative
  Decoding and Beyond": on rejection the blocks past the kept length are
  simply dropped (``truncate``).

Which physical id a request receives is not fixed by the pages; this model
hands out the smallest free id.  Tests therefore compare the library's block
manager with this model up to a relabelling of block ids: what is unique is
the number of blocks per sequence, which (sequence, logical block) pairs share
one physical block, every reference count, the free count, the copy pairs per
append and each token's offset inside its block.

An append that would need more blocks than the pool has raises
``NoFreeBlocks`` and changes nothing (reading: the pages leave what happens on
exhaustion to a preemption policy, [Taming the Tail] "Infrastructure Scale").
"""
from __future__ import annotations


class NoFreeBlocks(RuntimeError):
    """The pool cannot supply the blocks an append needs."""


class BlockModel:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad pool shape")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = set(range(num_blocks))
        self.ref = {}                  # physical block -> number of tables
        self.tables = {}               # seq id -> list of physical blocks
        self.lens = {}                 # seq id -> tokens stored

    # -- pool ---------------------------------------------------------------
    def _take(self) -> int:
        blk = min(self.free)
        self.free.remove(blk)
        self.ref[blk] = 1
        return blk

    def _drop(self, blk: int) -> None:
        self.ref[blk] -= 1
        if self.ref[blk] == 0:
            del self.ref[blk]
            self.free.add(blk)

    def num_free(self) -> int:
        return len(self.free)

    def refcount(self, blk: int) -> int:
        return self.ref.get(blk, 0)

    # -- sequences ----------------------------------------------------------
    def add_seq(self, seq) -> None:
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        self.tables[seq] = []
        self.lens[seq] = 0

    def fork(self, parent, child) -> None:
        """Child starts as an exact sharer of every block of the parent."""
        if parent not in self.tables or child in self.tables:
            raise KeyError("fork needs an existing parent and a new child")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for blk in self.tables[child]:
            self.ref[blk] += 1

    def blocks_needed(self, seq, n_tokens: int) -> int:
        """Blocks an append of ``n_tokens`` would take from the pool."""
        L = self.lens[seq]
        table = self.tables[seq]
        bs = self.block_size
        fresh = -(-(L + n_tokens) // bs) - len(table)
        partial_shared = (n_tokens > 0 and L % bs != 0
                          and self.ref[table[-1]] > 1)
        return fresh + (1 if partial_shared else 0)

    def append(self, seq, n_tokens: int):
        """Store ``n_tokens`` new tokens at the end of ``seq``.

        Returns ``(placements, copies)``: ``placements[i]`` is the
        ``(physical_block, offset)`` of the i-th new token and ``copies`` the
        ``(src, dst)`` blocks whose contents must be copied before any token
        is written (copy-on-write of a shared, partly filled last block).
        """
        if seq not in self.tables:
            raise KeyError(f"no sequence {seq}")
        if n_tokens < 0:
            raise ValueError("negative token count")
        if self.blocks_needed(seq, n_tokens) > len(self.free):
            raise NoFreeBlocks(f"sequence {seq} needs more blocks")
        table = self.tables[seq]
        bs = self.block_size
        placements, copies = [], []
        for _ in range(n_tokens):
            pos = self.lens[seq]
            logical, offset = divmod(pos, bs)
            if logical == len(table):          # last block full: open a new one
                table.append(self._take())
            elif self.ref[table[logical]] > 1:  # first write into a shared block
                src = table[logical]
                dst = self._take()
                self._drop(src)
                table[logical] = dst
                copies.append((src, dst))
            placements.append((table[logical], offset))
            self.lens[seq] = pos + 1
        return placements, copies

    def free_seq(self, seq) -> None:
        """Tear down a sequence's table; blocks at count zero rejoin the pool."""
        for blk in self.tables.pop(seq):
            self._drop(blk)
        del self.lens[seq]

    def truncate(self, seq, new_len: int) -> None:
        """Keep the first ``new_len`` tokens; release whole blocks past them."""
        if not 0 <= new_len <= self.lens[seq]:
            raise ValueError("truncate can only shorten a sequence")
        table = self.tables[seq]
        keep = -(-new_len // self.block_size)
        while len(table) > keep:
            self._drop(table.pop())
        self.lens[seq] = new_len
