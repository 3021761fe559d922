"""Pins of the swap model (oracle/swap_model.py).

The pages only pose the choice to pause a request and move its KV cache to
CPU RAM ([Taming the Tail] "Infrastructure Scale"), so the pins are closed
forms and invariants of that reading:

* a round trip leaves every sequence reading the same bytes, with the same
  sharing structure, lengths and reference counts (checked by moving actual
  block contents with the returned pairs, so a wrong direction, a dropped
  pair or a wrong order fails);
* host blocks taken = distinct device blocks of the group (shared blocks
  cross the link once); device blocks freed = those held only by the group;
* refusals change nothing; a swapped sequence takes no other operation.
"""
import random

import numpy as np
import pytest

from oracle.block_model import NoFreeBlocks
from oracle.swap_model import SwapModel


class Pools:
    """Block contents: every appended token slot gets a unique value."""

    def __init__(self, model, width=3):
        self.dev = np.full((model.num_blocks, model.block_size, width), -1)
        self.host = np.full((model.num_host_blocks, model.block_size, width),
                            -1)
        self.next = 0

    def write(self, placements):
        for blk, off in placements:
            self.dev[blk, off] = self.next
            self.next += 1

    def copy(self, pairs, to_host):
        for src, dst in pairs:
            if to_host:
                self.host[dst] = self.dev[src]
            else:
                self.dev[dst] = self.host[src]

    def read(self, model, seq, on_host=False):
        pool = self.host if on_host else self.dev
        bs = model.block_size
        return np.array([pool[model.tables[seq][t // bs], t % bs]
                         for t in range(model.lens[seq])])


def build(m, pools, rnd, n_seqs=6):
    m.add_seq(0)
    pools.write(m.append(0, 37)[0])
    for s in range(1, n_seqs):
        if rnd.random() < 0.5:
            m.fork(rnd.randrange(s), s)
        else:
            m.add_seq(s)
        placements, copies = m.append(s, rnd.randint(1, 20))
        pools.dev[[d for _, d in copies]] = pools.dev[[c for c, _ in copies]]
        pools.write(placements)


def sharing(m, seqs):
    """Which (sequence, logical block) pairs share a physical block."""
    first, out = {}, []
    for s in seqs:
        for i, blk in enumerate(m.tables[s]):
            out.append(first.setdefault(blk, (s, i)))
    return out


@pytest.mark.parametrize("seed", range(8))
def test_round_trip_restores_contents_and_structure(seed):
    rnd = random.Random(seed)
    m = SwapModel(64, 4, num_host_blocks=64)
    pools = Pools(m)
    build(m, pools, rnd)
    seqs = sorted(m.tables)
    group = rnd.sample(seqs, rnd.randint(1, len(seqs)))
    before = {s: pools.read(m, s) for s in seqs}
    share_before = sharing(m, group)
    lens_before = dict(m.lens)
    distinct = len({b for s in group for b in m.tables[s]})
    held_only = sum(1 for b in {b for s in group for b in m.tables[s]}
                    if m.refcount(b) == sum(t.count(b) for x, t in
                                             m.tables.items() if x in group))
    free0 = m.num_free()
    out_pairs = m.swap_out(group)
    assert len(out_pairs) == distinct == 64 - m.num_free_host()
    assert m.num_free() == free0 + held_only
    pools.copy(out_pairs, to_host=True)
    for s in group:
        assert (pools.read(m, s, on_host=True) == before[s]).all()
    freed = [d for d, _ in out_pairs if d in m.free]
    assert len(freed) == held_only
    pools.dev[freed] = -7             # freed blocks get reused meanwhile
    in_pairs = m.swap_in(group)
    pools.copy(in_pairs, to_host=False)
    for s in seqs:
        assert (pools.read(m, s) == before[s]).all(), s
    assert sharing(m, group) == share_before
    assert m.lens == lens_before
    assert m.num_free_host() == 64


def test_shared_prefix_crosses_once():
    m = SwapModel(64, 4, num_host_blocks=64)
    m.add_seq(0)
    m.append(0, 40)                   # 10 full prefix blocks
    for s in range(1, 4):
        m.fork(0, s)
    for s in range(4):
        m.append(s, 12)               # 3 own blocks each
    assert len(m.swap_out(range(4))) == 10 + 4 * 3
    assert m.num_free() == 64
    assert {m.host_refcount(h) for h in m.tables[0][:10]} == {4}
    pairs = m.swap_in([2])            # one member comes back alone
    assert len(pairs) == 13
    assert {m.host_refcount(h) for h in m.tables[0][:10]} == {3}
    assert all(m.refcount(b) == 1 for b in m.tables[2])


def test_partial_group_copies_shared_blocks_and_keeps_them():
    m = SwapModel(32, 4, num_host_blocks=32)
    m.add_seq(0)
    m.append(0, 8)
    m.fork(0, 1)
    pairs = m.swap_out([1])
    assert len(pairs) == 2
    assert [m.refcount(b) for b in m.tables[0]] == [1, 1]
    assert m.num_free() == 30


def test_refusals_change_nothing():
    m = SwapModel(16, 4, num_host_blocks=2)
    m.add_seq(0)
    m.append(0, 12)
    with pytest.raises(NoFreeBlocks):
        m.swap_out([0])
    assert 0 not in m.swapped and m.num_free_host() == 2
    m.num_host_blocks = 3
    m.host_free = {0, 1, 2}
    m.swap_out([0])
    for op in (lambda: m.append(0, 1), lambda: m.fork(0, 5),
               lambda: m.truncate(0, 1), lambda: m.insert(0, [1] * 4),
               lambda: m.swap_out([0])):
        with pytest.raises(ValueError):
            op()
    m.add_seq(1)
    m.append(1, 64)                   # device pool now full
    with pytest.raises(NoFreeBlocks):
        m.swap_in([0])
    assert 0 in m.swapped and m.num_free_host() == 0
    m.free_seq(1)
    m.swap_in([0])
    m.free_seq(0)
    assert m.num_free() == 16 and m.num_free_host() == 3


def test_swap_in_evicts_cached_leaves():
    m = SwapModel(8, 2, num_host_blocks=8)
    m.add_seq(0)
    m.append(0, 4)
    m.insert(0, [1, 2, 3, 4])
    m.free_seq(0)                     # 2 blocks cached only
    m.add_seq(1)
    m.append(1, 8)
    m.swap_out([1])
    m.add_seq(2)
    m.append(2, 8)                    # 2 free left
    m.swap_in([1])                    # needs 4: evicts both cached blocks
    assert m.num_cached() == 0 and m.num_free() == 0
