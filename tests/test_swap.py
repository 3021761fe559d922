"""The library's swap (C++ block manager) against the oracle swap model.

Both see the same operations: appends, forks, frees, prefix-cache traffic
and group swaps both ways.  Block ids are compared up to one relabelling per
pool (device, host), consistent across all tables, the cache and every
returned pair: tables, swap state, lengths, reference counts on both pools,
free counts, cached paths, the pairs themselves and every refusal.
"""
import random

import numpy as np
import pytest

from oracle.block_model import NoFreeBlocks
from oracle.swap_model import SwapModel


class Relabel:
    def __init__(self):
        self.maps = {"dev": {}, "host": {}}

    def same(self, pool, lib_id, model_id):
        m = self.maps[pool]
        assert m.setdefault(int(lib_id), model_id) == model_id, (pool, lib_id)
        assert len(set(m.values())) == len(m)


def assert_same(bm, model):
    """Compare the states; returns the relabelling they define."""
    rl = Relabel()
    for s in sorted(model.tables):
        swapped = s in model.swapped
        assert bm.is_swapped(s) == swapped
        assert bm.seq_len(s) == model.lens[s]
        lib = bm.seq_blocks(s)
        assert len(lib) == len(model.tables[s])
        for x, y in zip(lib, model.tables[s]):
            rl.same("host" if swapped else "dev", x, y)
    for x, y in rl.maps["dev"].items():
        assert bm.refcount(x) == model.refcount(y)
    for x, y in rl.maps["host"].items():
        assert bm.host_refcount(x) == model.host_refcount(y)
    assert bm.num_free() == model.num_free()
    assert bm.num_free_host() == model.num_free_host()
    assert bm.cached_paths() == model.cached_paths()
    return rl


def same_pairs(before, after, lib_pairs, model_pairs, src_pool, dst_pool):
    """Sources are named by the state before the swap, destinations by the
    state after it."""
    assert len(lib_pairs) == len(model_pairs)
    for (a, b), (c, d) in zip(lib_pairs, model_pairs):
        before.same(src_pool, a, c)
        after.same(dst_pool, b, d)


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_model(pkv, seed):
    rnd = random.Random(seed)
    nb, nh, bs = rnd.choice([(32, 24, 4), (48, 64, 2), (40, 16, 4)])
    bm = pkv.BlockManager(nb, bs, free_order=np.random.default_rng(seed)
                          .permutation(nb).astype(np.int32))
    bm.set_host_blocks(nh)
    model = SwapModel(nb, bs, num_host_blocks=nh)
    live, nxt = [], 0
    before = assert_same(bm, model)
    for _ in range(600):
        op = rnd.random()
        swap = None
        resident = [s for s in live if s not in model.swapped]
        swapped = [s for s in live if s in model.swapped]
        if op < 0.2 or not live:
            bm.add_seq(nxt)
            model.add_seq(nxt)
            toks = [rnd.randint(0, 1) for _ in range(rnd.randint(0, 4 * bs))]
            assert bm.match_prefix(nxt, toks) == model.match(nxt, toks)
            try:
                model.append(nxt, len(toks) - model.lens[nxt])
            except NoFreeBlocks:
                with pytest.raises(pkv.NoFreeBlocksError):
                    bm.append(nxt, len(toks) - bm.seq_len(nxt))
            else:
                bm.append(nxt, len(toks) - bm.seq_len(nxt))
                bm.cache_insert(nxt, toks)
                model.insert(nxt, toks)
            live.append(nxt)
            nxt += 1
        elif op < 0.3 and resident:
            p = rnd.choice(resident)
            bm.fork(p, nxt)
            model.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif op < 0.45 and resident:
            s = rnd.choice(resident)
            n = rnd.randint(1, 2 * bs)
            try:
                model.append(s, n)
            except NoFreeBlocks:
                with pytest.raises(pkv.NoFreeBlocksError):
                    bm.append(s, n)
            else:
                bm.append(s, n)
        elif op < 0.55:
            s = rnd.choice(live)
            bm.free_seq(s)
            model.free_seq(s)
            live.remove(s)
        elif op < 0.75 and resident:
            group = rnd.sample(resident, rnd.randint(1, min(4, len(resident))))
            try:
                mp = model.swap_out(group)
            except NoFreeBlocks:
                with pytest.raises(pkv.NoFreeBlocksError):
                    bm.swap_out(group)
            else:
                swap = (bm.swap_out(group), mp, "dev", "host")
        elif swapped:
            group = rnd.sample(swapped, rnd.randint(1, min(4, len(swapped))))
            try:
                mp = model.swap_in(group)
            except NoFreeBlocks:
                with pytest.raises(pkv.NoFreeBlocksError):
                    bm.swap_in(group)
            else:
                swap = (bm.swap_in(group), mp, "host", "dev")
        after = assert_same(bm, model)
        if swap is not None:
            same_pairs(before, after, *swap)
        before = after


def test_swapped_sequence_refuses_other_operations(pkv):
    bm = pkv.BlockManager(16, 4)
    bm.set_host_blocks(8)
    bm.add_seq(0)
    bm.append(0, 9)
    pairs = bm.swap_out([0])
    assert len(pairs) == 3 and bm.is_swapped(0)
    for op in (lambda: bm.append(0, 1), lambda: bm.fork(0, 1),
               lambda: bm.truncate(0, 1), lambda: bm.block_table([0], 4),
               lambda: bm.cache_insert(0, [1] * 4), lambda: bm.swap_out([0]),
               lambda: bm.set_host_blocks(4)):
        with pytest.raises(pkv.PagedKVError):
            op()
    with pytest.raises(pkv.PagedKVError):
        bm.swap_in([0, 0])
    back = bm.swap_in([0])
    assert [h for h, _ in back] == [d for _, d in pairs]
    assert bm.num_free_host() == 8
    table, lens = bm.block_table([0], 4)
    assert lens[0] == 9 and (table[0][:3] >= 0).all()


def test_max_pairs_too_small_changes_nothing(pkv):
    bm = pkv.BlockManager(16, 4)
    bm.set_host_blocks(8)
    bm.add_seq(0)
    bm.append(0, 9)
    with pytest.raises(pkv.PagedKVError):
        bm.swap_out([0], pairs_out=np.empty((2, 2), dtype=np.int32))
    assert not bm.is_swapped(0) and bm.num_free_host() == 8
