"""The library's prefix cache (C++ block manager) against the oracle model.

Both see the same operations.  Physical ids are not unique, so states are
compared up to a relabelling of block ids that must be consistent across the
sequences' tables and the cache: tables, lengths, reference counts, free
count, the set of cached token paths, the block behind each path, every
match length and every refusal -- all exact.
"""
import random

import numpy as np
import pytest

from oracle.block_model import NoFreeBlocks
from oracle.prefix_cache import PrefixCacheModel

from test_block_manager import assert_same_state


def assert_same_cache(bm, model):
    relabel = assert_same_state(bm, model)
    parent, block, toks = bm.cache_nodes()
    paths = []
    for i in range(len(parent)):
        key = tuple(int(t) for t in toks[i])
        paths.append((key,) if parent[i] < 0 else paths[parent[i]] + (key,))
    assert set(paths) == model.cached_paths()
    assert bm.num_cached() == model.num_cached()
    # the block behind each path, through the same relabelling
    by_path = {}
    for n in model._nodes():
        keys, m = [], n
        while m is not model.root:
            keys.append(m.key)
            m = m.parent
        by_path[tuple(reversed(keys))] = n.block
    for p, b in zip(paths, block):
        assert relabel.setdefault(int(b), by_path[p]) == by_path[p], p
        assert bm.refcount(int(b)) == model.refcount(by_path[p])
    assert len(set(relabel.values())) == len(relabel)


def serve_both(pkv, bm, model, seq, tokens):
    """match -> append the rest -> insert, on both; returns the match, or
    None if both refused the append."""
    bm.add_seq(seq)
    model.add_seq(seq)
    hit = bm.match_prefix(seq, tokens)
    assert hit == model.match(seq, tokens)
    try:
        model.append(seq, len(tokens) - hit)
    except NoFreeBlocks:
        with pytest.raises(pkv.NoFreeBlocksError):
            bm.append(seq, len(tokens) - hit)
        return None
    bm.append(seq, len(tokens) - hit)
    bm.cache_insert(seq, tokens)
    model.insert(seq, tokens)
    return hit


@pytest.mark.parametrize("prompt_len,expected", [(384, 3024), (380, 3523)])
def test_worked_example_2_through_the_library(pkv, prompt_len, expected):
    bs, requests, question = 16, 500, 90
    bm = pkv.BlockManager(16000, bs)
    prompt = list(range(10_000, 10_000 + prompt_len))
    hits = []
    for r in range(requests):
        q = [100_000 + r * question + i for i in range(question)]
        bm.add_seq(r)
        hits.append(bm.match_prefix(r, prompt + q))
        bm.append(r, len(prompt) + question - hits[-1])
        bm.cache_insert(r, prompt + q)
    assert 16000 - bm.num_free() == expected
    assert hits[0] == 0 and set(hits[1:]) == {bs * (prompt_len // bs)}


def test_hand_worked_lru_order(pkv):
    bm = pkv.BlockManager(8, 2)
    for seq, toks in ((0, [1, 2, 3, 4]), (1, [1, 2, 5, 6]), (2, [7, 8])):
        bm.add_seq(seq)
        assert bm.match_prefix(seq, toks) == (2 if seq == 1 else 0)
        bm.append(seq, len(toks) - (2 if seq == 1 else 0))
        bm.cache_insert(seq, toks)
        bm.free_seq(seq)
    bm.add_seq(3)
    assert bm.match_prefix(3, [1, 2, 3, 4, 9]) == 4
    bm.free_seq(3)
    order = []
    while True:
        before = bm.cached_paths()
        if not bm.cache_evict(1):
            break
        (gone,) = before - bm.cached_paths()
        order.append(gone[-1])
    assert order == [(5, 6), (7, 8), (3, 4), (1, 2)]
    assert bm.num_free() == 8 and bm.num_cached() == 0


def test_refused_append_leaves_cache_intact(pkv):
    bm = pkv.BlockManager(6, 2)
    model = PrefixCacheModel(6, 2)
    serve_both(pkv, bm, model, 0, [1, 2, 3, 4])
    serve_both(pkv, bm, model, 1, [5, 6, 7, 8])
    for s in (0, 1):
        bm.free_seq(s)
        model.free_seq(s)
    bm.add_seq(2)
    model.add_seq(2)
    before = bm.cached_paths()
    with pytest.raises(pkv.NoFreeBlocksError):
        bm.append(2, 13)             # 7 blocks: more than free + evictable
    assert bm.cached_paths() == before and bm.num_free() == 2
    bm.append(2, 6)
    model.append(2, 6)
    assert_same_cache(bm, model)


def test_insert_refuses_inconsistent_tokens(pkv):
    bm = pkv.BlockManager(16, 2)
    bm.add_seq(0)
    bm.append(0, 4)
    bm.cache_insert(0, [1, 2, 3, 4])
    bm.fork(0, 1)
    with pytest.raises(pkv.PagedKVError):
        bm.cache_insert(1, [9, 9, 3, 4])
    assert bm.cached_paths() == {((1, 2),), ((1, 2), (3, 4))}


def test_match_needs_an_empty_sequence(pkv):
    bm = pkv.BlockManager(16, 2)
    bm.add_seq(0)
    bm.append(0, 1)
    with pytest.raises(pkv.PagedKVError):
        bm.match_prefix(0, [1, 2])
    with pytest.raises(pkv.PagedKVError):
        bm.match_prefix(7, [1, 2])


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_model(pkv, seed):
    rnd = random.Random(seed)
    nb, bs = rnd.choice([(24, 2), (40, 4), (64, 4)])
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    bm = pkv.BlockManager(nb, bs, free_order=order)
    model = PrefixCacheModel(nb, bs)
    vocab = [0, 1] if seed % 2 else [0, 1, 2]
    live, nxt = {}, 0
    for step in range(500):
        op = rnd.random()
        if op < 0.35 or not live:
            toks = [rnd.choice(vocab) for _ in range(rnd.randint(0, 5 * bs))]
            if serve_both(pkv, bm, model, nxt, toks) is None:
                bm.free_seq(nxt)
                model.free_seq(nxt)
            else:
                live[nxt] = toks
            nxt += 1
        elif op < 0.55:
            s = rnd.choice(list(live))
            bm.free_seq(s)
            model.free_seq(s)
            del live[s]
        elif op < 0.62:
            s = rnd.choice(list(live))
            bm.fork(s, nxt)
            model.fork(s, nxt)
            live[nxt] = list(live[s])
            nxt += 1
        elif op < 0.70:
            s = rnd.choice(list(live))
            n = rnd.randint(0, len(live[s]))
            bm.truncate(s, n)
            model.truncate(s, n)
            live[s] = live[s][:n]
        elif op < 0.85:
            # a decode step or a chunk: more tokens, then cache them
            s = rnd.choice(list(live))
            extra = [rnd.choice(vocab) for _ in range(rnd.randint(1, 2 * bs))]
            try:
                _, copies = model.append(s, len(extra))
            except NoFreeBlocks:
                with pytest.raises(pkv.NoFreeBlocksError):
                    bm.append(s, len(extra))
            else:
                _, pairs = bm.append(s, len(extra))
                assert len(pairs) == len(copies)
                live[s] = live[s] + extra
                k = rnd.randint(0, len(live[s]))
                try:
                    model.insert(s, live[s][:k])
                except ValueError:
                    with pytest.raises(pkv.PagedKVError):
                        bm.cache_insert(s, live[s][:k])
                else:
                    bm.cache_insert(s, live[s][:k])
        else:
            k = rnd.randint(1, 4)
            assert bm.cache_evict(k) == model.evict(k)
        assert_same_cache(bm, model)
