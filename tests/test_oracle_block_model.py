"""Pins of the block-manager reference model (oracle/block_model.py).

Expected values come from the pages (tests/golden/worked_examples.json) or
from invariants every state must satisfy: reference counts equal the number
of table entries pointing at a block, and the pool holds exactly the blocks
nobody points at.
"""
import random

import pytest

from oracle import fragmentation as fr
from oracle.block_model import BlockModel, NoFreeBlocks


def check_invariants(m: BlockModel):
    counts = {}
    for seq, table in m.tables.items():
        assert len(table) == fr.blocks_for(m.lens[seq], m.block_size)
        for blk in table:
            counts[blk] = counts.get(blk, 0) + 1
    assert counts == m.ref
    assert set(counts).isdisjoint(m.free)
    assert len(counts) + len(m.free) == m.num_blocks


def test_answer_6_refcount_keeps_shared_block(golden):
    g = golden["answer_6"]
    m = BlockModel(8, 16)
    m.add_seq("A")
    m.append("A", 10)
    m.fork("A", "B")
    p0 = m.tables["A"][0]
    assert m.refcount(p0) == g["refcount_before"]
    m.free_seq("A")
    assert m.refcount(p0) == g["refcount_after_one_teardown"]
    assert (p0 in m.free) == g["returned_to_pool_after_one_teardown"]
    m.free_seq("B")
    assert p0 in m.free and m.refcount(p0) == 0
    check_invariants(m)


def test_token_17_opens_a_block(golden):
    g = golden["token_17"]
    m = BlockModel(4, g["block_size"])
    m.add_seq(0)
    m.append(0, 16)
    assert len(m.tables[0]) == g["blocks_after_16_tokens"]
    placements, copies = m.append(0, 1)
    assert len(m.tables[0]) == g["blocks_after_17_tokens"]
    assert placements == [(m.tables[0][1], 0)] and copies == []


def test_worked_example_1_through_appends(golden):
    g = golden["worked_example_1"]
    m = BlockModel(256, g["block_size"])
    for i, L in enumerate(g["lengths"]):
        m.add_seq(i)
        # tokens arrive one decode step at a time
        for _ in range(L):
            m.append(i, 1)
    assert [len(m.tables[i]) for i in range(4)] == g["blocks_per_seq"]
    assert 256 - m.num_free() == g["total_blocks"]
    waste = [len(m.tables[i]) * 16 - m.lens[i] for i in range(4)]
    assert sum(waste) == g["paged_waste_slots"]
    assert all(w < golden["waste_bound"]["max_waste_per_seq_exclusive"]
               for w in waste)
    check_invariants(m)


def test_placements_are_token_order():
    m = BlockModel(16, 16)
    m.add_seq(0)
    placements, _ = m.append(0, 40)
    t = m.tables[0]
    assert placements == [(t[p // 16], p % 16) for p in range(40)]


def test_fork_then_write_copies_partial_block():
    m = BlockModel(16, 16)
    m.add_seq("p")
    m.append("p", 20)                 # block 0 full, block 1 holds 4 tokens
    m.fork("p", "c")
    shared_last = m.tables["p"][1]
    placements, copies = m.append("c", 1)
    assert len(copies) == 1 and copies[0][0] == shared_last
    dst = copies[0][1]
    assert m.tables["c"] == [m.tables["p"][0], dst]
    assert placements == [(dst, 4)]
    assert m.refcount(shared_last) == 1 and m.refcount(dst) == 1
    assert m.refcount(m.tables["p"][0]) == 2
    # the parent now writes in place: no second copy
    _, copies = m.append("p", 1)
    assert copies == []
    check_invariants(m)


def test_fork_at_block_boundary_needs_no_copy():
    m = BlockModel(8, 16)
    m.add_seq(0)
    m.append(0, 32)
    m.fork(0, 1)
    placements, copies = m.append(1, 3)
    assert copies == [] and len(m.tables[1]) == 3
    assert placements[0][1] == 0


def test_exhaustion_changes_nothing():
    m = BlockModel(3, 16)
    m.add_seq(0)
    m.append(0, 40)                   # 3 blocks
    snapshot = (dict(m.ref), set(m.free), {k: list(v) for k, v in
                                           m.tables.items()}, dict(m.lens))
    with pytest.raises(NoFreeBlocks):
        m.append(0, 9)
    assert snapshot == (m.ref, m.free, m.tables, m.lens)
    m.append(0, 8)                    # fills the last block exactly: fine
    check_invariants(m)


def test_copy_on_write_needs_a_free_block():
    m = BlockModel(2, 16)
    m.add_seq(0)
    m.append(0, 20)
    m.fork(0, 1)
    with pytest.raises(NoFreeBlocks):
        m.append(1, 1)                # copy needs a third block
    assert m.lens[1] == 20 and m.refcount(m.tables[0][1]) == 2


def test_shared_prefix_mix_copy_count():
    # 2056-token prefix = 128 full blocks + 8 tokens; 128 sharers append in
    # index order; every writer but the last sees a count above one.
    m = BlockModel(128 * 64 + 200, 16)
    m.add_seq(0)
    m.append(0, 2056)
    for s in range(1, 128):
        m.fork(0, s)
    assert all(m.refcount(b) == 128 for b in m.tables[0])
    total_copies = 0
    for s in range(128):
        _, copies = m.append(s, 16 + s)
        total_copies += len(copies)
    assert total_copies == 127
    check_invariants(m)


def test_worked_example_2_with_a_real_block_manager(golden):
    # Worked Example 2 prints 3024 blocks assuming the 380-token prompt ends
    # on a block boundary; it does not (380 = 23*16 + 12).  Run through the
    # model, the 23 whole blocks are shared, the partial one is copied by
    # every writer but the last, and each request then needs 6 more blocks.
    g = golden["worked_example_2"]
    m = BlockModel(20000, g["block_size"])
    m.add_seq(0)
    m.append(0, g["prompt_len"])
    for s in range(1, g["num_requests"]):
        m.fork(0, s)
    for s in range(g["num_requests"]):
        m.append(s, g["suffix_len"])
    used = m.num_blocks - m.num_free()
    shareable = fr.shareable_prompt_blocks(g["prompt_len"], 16)["blocks"]
    per_req_new = fr.blocks_for(g["suffix_len"] - (16 - g["prompt_len"] % 16),
                                16)
    assert per_req_new == 6
    expect = shareable + 1 + (g["num_requests"] - 1) + \
        g["num_requests"] * per_req_new
    assert used == expect == 3523
    check_invariants(m)


def test_truncate_releases_tail_blocks():
    m = BlockModel(8, 16)
    m.add_seq(0)
    m.append(0, 50)                   # 4 blocks
    m.truncate(0, 17)
    assert len(m.tables[0]) == 2 and m.num_free() == 6
    placements, _ = m.append(0, 1)
    assert placements == [(m.tables[0][1], 1)]
    check_invariants(m)


def test_random_operations_keep_invariants():
    rnd = random.Random(1234)
    m = BlockModel(64, 16)
    live, nxt = [], 0
    for _ in range(2000):
        op = rnd.random()
        if op < 0.15 or not live:
            m.add_seq(nxt)
            live.append(nxt)
            nxt += 1
        elif op < 0.25:
            m.fork(rnd.choice(live), nxt)
            live.append(nxt)
            nxt += 1
        elif op < 0.35:
            s = rnd.choice(live)
            m.free_seq(s)
            live.remove(s)
        elif op < 0.40:
            s = rnd.choice(live)
            m.truncate(s, rnd.randint(0, m.lens[s]))
        else:
            s = rnd.choice(live)
            try:
                m.append(s, rnd.randint(1, 40))
            except NoFreeBlocks:
                pass
        check_invariants(m)
