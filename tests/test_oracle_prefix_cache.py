"""Pins of the prefix-cache model (oracle/prefix_cache.py) against the pages.

* [KV-cache chapter] Worked Example 2: a shared system prompt stored once
  and only the question blocks allocated per request -- 15,000 blocks without
  sharing, 3,024 with it, a factor of about 4.96.  The page counts 24 prompt
  blocks, which is the block-aligned prompt of 384 tokens; the 380-token
  prompt it names shares 23 full blocks (its 24th block is partly filled and
  is never cached), giving 23 + 500 x 7 = 3,523.
* [KV-cache chapter] "RadixAttention: caching, not just packing, the
  prefix": matched tokens are referenced, not recomputed; leaves are evicted
  least recently used first; a branch referenced by a running request is
  never evicted.  A hand-worked tree fixes the eviction order.
"""
import random

import pytest

from oracle.block_model import NoFreeBlocks
from oracle.prefix_cache import PrefixCacheModel


def serve(model, seq, tokens):
    """One request: match, allocate the rest, (prefill), cache, keep live."""
    model.add_seq(seq)
    hit = model.match(seq, tokens)
    model.append(seq, len(tokens) - hit)
    model.insert(seq, tokens)
    return hit


@pytest.mark.parametrize("prompt_len,expected", [(384, 3024), (380, 3523)])
def test_worked_example_2_shared_system_prompt(prompt_len, expected):
    bs, requests, question = 16, 500, 90
    model = PrefixCacheModel(16000, bs)
    prompt = list(range(10_000, 10_000 + prompt_len))
    hits = []
    for r in range(requests):
        q = [100_000 + r * question + i for i in range(question)]
        hits.append(serve(model, r, prompt + q))
    in_use = model.num_blocks - model.num_free()
    assert in_use == expected
    assert hits[0] == 0
    assert set(hits[1:]) == {bs * (prompt_len // bs)}
    without = requests * -(-(prompt_len + question) // bs)
    assert without == 15000
    if prompt_len == 384:
        assert round(without / in_use, 2) == 4.96


def test_hand_worked_lru_order():
    # block size 2; A = [1 2 | 3 4], B = [1 2 | 5 6], C = [7 8], D touches A.
    # Stamps: A insert 2, B match 3 / insert 4, C insert 6, D match 7.
    # Leaves then: [3 4] @7, [5 6] @4, [7 8] @6 -> evict [5 6], [7 8],
    # [3 4], and finally [1 2] once it has become a leaf.
    m = PrefixCacheModel(8, 2)
    for seq, toks in ((0, [1, 2, 3, 4]), (1, [1, 2, 5, 6]), (2, [7, 8])):
        serve(m, seq, toks)
        m.free_seq(seq)
    assert m.num_cached() == 4 and m.num_free() == 4
    m.add_seq(3)
    assert m.match(3, [1, 2, 3, 4, 9]) == 4
    m.free_seq(3)
    order = []
    while True:
        before = m.cached_paths()
        if not m.evict(1):
            break
        (gone,) = before - m.cached_paths()
        order.append(gone[-1])
    assert order == [(5, 6), (7, 8), (3, 4), (1, 2)]
    assert m.num_free() == 8


def test_live_branches_are_not_evicted():
    m = PrefixCacheModel(8, 2)
    for seq, toks in ((0, [1, 2, 3, 4]), (1, [1, 2, 5, 6]), (2, [7, 8])):
        serve(m, seq, toks)
        m.free_seq(seq)
    m.add_seq(3)
    m.match(3, [1, 2, 3, 4])          # a running request holds [1 2][3 4]
    assert m.num_evictable() == 2
    assert m.evict(10) == 2
    assert m.cached_paths() == {((1, 2),), ((1, 2), (3, 4))}
    assert m.refcount(m.tables[3][0]) == 2
    m.free_seq(3)
    assert m.num_evictable() == 2 and m.evict(10) == 2
    assert m.num_free() == 8 and m.num_cached() == 0


def test_matched_blocks_are_shared_not_copied():
    m = PrefixCacheModel(16, 4)
    toks = list(range(11))
    serve(m, 0, toks)                 # blocks [0..3] [4..7] cached, 3 tokens left
    m.add_seq(1)
    assert m.match(1, toks) == 8
    assert m.tables[1] == m.tables[0][:2]
    assert [m.refcount(b) for b in m.tables[1]] == [3, 3]  # 2 tables + cache
    # appending to a sequence that ends on a cached full block opens a new one
    placements, copies = m.append(1, 3)
    assert copies == [] and placements[0][1] == 0
    assert m.tables[1][2] != m.tables[0][2]


def test_append_evicts_lru_and_refuses_without_change():
    m = PrefixCacheModel(6, 2)
    serve(m, 0, [1, 2, 3, 4])
    serve(m, 1, [5, 6, 7, 8])
    m.free_seq(0)
    m.free_seq(1)                     # 4 cached, 2 free
    m.add_seq(2)
    m.append(2, 6)                    # needs 3: evicts the oldest leaf [3 4]
    assert m.cached_paths() == {((1, 2),), ((5, 6),), ((5, 6), (7, 8))}
    m.add_seq(3)
    with pytest.raises(NoFreeBlocks):
        m.append(3, 8)                # needs 4, only 3 evictable
    assert m.num_cached() == 3 and m.lens[3] == 0
    m.append(3, 6)
    assert m.num_cached() == 0 and m.num_free() == 0


def test_duplicate_blocks_stay_outside_the_cache():
    m = PrefixCacheModel(16, 2)
    m.add_seq(0)
    m.add_seq(1)
    m.append(0, 4)
    m.append(1, 4)                    # both computed [1 2 | 3 4] themselves
    m.insert(0, [1, 2, 3, 4])
    m.insert(1, [1, 2, 3, 4])
    assert m.num_cached() == 2
    assert all(m.refcount(b) == 1 for b in m.tables[1])
    assert all(m.refcount(b) == 2 for b in m.tables[0])


def test_insert_refuses_inconsistent_tokens():
    m = PrefixCacheModel(16, 2)
    serve(m, 0, [1, 2, 3, 4])
    m.fork(0, 1)                      # shares the cached blocks
    with pytest.raises(ValueError):
        m.insert(1, [9, 9, 3, 4])     # block 0 is cached under [1 2]
    assert m.cached_paths() == {((1, 2),), ((1, 2), (3, 4))}


def test_random_ops_keep_invariants():
    rnd = random.Random(5)
    m = PrefixCacheModel(40, 4)
    vocab = [0, 1]
    live, nxt = [], 0
    for _ in range(2000):
        op = rnd.random()
        if op < 0.3 or not live:
            toks = [rnd.choice(vocab) for _ in range(rnd.randint(1, 14))]
            try:
                serve(m, nxt, toks)
            except NoFreeBlocks:
                m.free_seq(nxt)
                continue
            live.append((nxt, toks))
            nxt += 1
        elif op < 0.6:
            s, _ = live.pop(rnd.randrange(len(live)))
            m.free_seq(s)
        else:
            m.evict(rnd.randint(1, 3))
        # invariants: every cached block is referenced by the cache, counts
        # add up, and the pool plus live blocks cover everything
        refs = {}
        for s in m.tables.values():
            for b in s:
                refs[b] = refs.get(b, 0) + 1
        for b in m.node_of:
            refs[b] = refs.get(b, 0) + 1
        assert refs == m.ref
        assert len(refs) + m.num_free() == m.num_blocks
        # every live request still reads its own tokens' cached prefix
        for s, toks in live:
            assert m.lens[s] == len(toks)
