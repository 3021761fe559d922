"""The library's C++ block manager against the oracle's block model.

Both see the same operations.  Physical ids are not unique (the pages fix no
allocation order), so states are compared up to a relabelling of block ids:
number of blocks and length per sequence, which (sequence, logical block)
pairs share a physical block, each reference count, the free count, copy
pairs and every token's offset -- all bit-exact.
"""
import random

import numpy as np
import pytest

from oracle import fragmentation as fr
from oracle.block_model import BlockModel, NoFreeBlocks


def tables_of(bm, seqs, max_blocks=4096):
    if not seqs:
        return {}
    table, lens = bm.block_table(seqs, max_blocks)
    return {s: (list(table[i][table[i] >= 0]), int(lens[i]))
            for i, s in enumerate(seqs)}


def assert_same_state(bm, model):
    seqs = sorted(model.tables)
    lib_tables = tables_of(bm, seqs)
    relabel = {}
    for s in seqs:
        lib_blocks, lib_len = lib_tables[s]
        assert lib_len == model.lens[s]
        assert len(lib_blocks) == len(model.tables[s])
        for lb, (x, y) in enumerate(zip(lib_blocks, model.tables[s])):
            assert relabel.setdefault(x, y) == y, (s, lb)
    assert len(set(relabel.values())) == len(relabel)   # injective
    for x, y in relabel.items():
        assert bm.refcount(x) == model.refcount(y)
    assert bm.num_free() == model.num_free()
    return relabel


def test_random_operations_match_model(pkv):
    for seed in range(4):
        rnd = random.Random(seed)
        nb, bs = 48, rnd.choice([4, 16])
        order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
        bm = pkv.BlockManager(nb, bs, free_order=order)
        model = BlockModel(nb, bs)
        live, nxt = [], 0
        for _ in range(600):
            op = rnd.random()
            n, slots, placements = 0, [], []
            before = tables_of(bm, live)
            if op < 0.12 or not live:
                bm.add_seq(nxt)
                model.add_seq(nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.22:
                p = rnd.choice(live)
                bm.fork(p, nxt)
                model.fork(p, nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.32:
                s = rnd.choice(live)
                bm.free_seq(s)
                model.free_seq(s)
                live.remove(s)
            elif op < 0.37:
                s = rnd.choice(live)
                n = rnd.randint(0, model.lens[s])
                bm.truncate(s, n)
                model.truncate(s, n)
            else:
                s = rnd.choice(live)
                n = rnd.randint(0, 3 * bs)
                try:
                    placements, copies = model.append(s, n)
                except NoFreeBlocks:
                    with pytest.raises(pkv.NoFreeBlocksError):
                        bm.append(s, n)
                    assert tables_of(bm, live) == before
                    continue
                start = model.lens[s] - n
                slots, pairs = bm.append(s, n)
                assert len(pairs) == len(copies)
                after = tables_of(bm, live)[s][0]
                for i, slot in enumerate(slots):
                    pos = start + i
                    assert slot % bs == placements[i][1] == pos % bs
                    assert slot // bs == after[pos // bs]
                for (src, dst) in pairs:
                    old = before[s][0]
                    assert src == old[-1] and dst == after[len(old) - 1]
            relabel = assert_same_state(bm, model)
            # placements agree with the relabelled tables
            if placements:
                for i, slot in enumerate(slots):
                    assert relabel[int(slot // bs)] == placements[i][0]
        bm.close()


def test_worked_example_1_block_counts(pkv, golden):
    g = golden["worked_example_1"]
    bm = pkv.BlockManager(256, g["block_size"])
    for i, L in enumerate(g["lengths"]):
        bm.add_seq(i)
        bm.append(i, L)
    table, lens = bm.block_table(list(range(4)), 128)
    per_seq = [int((row >= 0).sum()) for row in table]
    assert per_seq == g["blocks_per_seq"]
    assert 256 - bm.num_free() == g["total_blocks"]
    waste = [n * 16 - L for n, L in zip(per_seq, g["lengths"])]
    assert all(0 <= w < 16 for w in waste)
    assert sum(waste) == g["paged_waste_slots"]
    assert list(lens) == g["lengths"]


def test_free_order_is_followed(pkv):
    order = np.random.default_rng(0).permutation(64).astype(np.int32)
    bm = pkv.BlockManager(64, 16, free_order=order)
    bm.add_seq(7)
    slots, pairs = bm.append(7, 16 * 5)
    assert len(pairs) == 0
    table, _ = bm.block_table([7], 8)
    assert list(table[0][:5]) == list(order[:5])
    assert list(slots) == [order[p // 16] * 16 + p % 16 for p in range(80)]


def test_token_17_and_answer_6(pkv, golden):
    bm = pkv.BlockManager(8, 16)
    bm.add_seq(0)
    bm.append(0, 16)
    assert bm.num_seq_blocks(0) == golden["token_17"]["blocks_after_16_tokens"]
    bm.append(0, 1)
    assert bm.num_seq_blocks(0) == golden["token_17"]["blocks_after_17_tokens"]
    g = golden["answer_6"]
    bm.fork(0, 1)
    table, _ = bm.block_table([0], 4)
    p0 = int(table[0][0])
    assert bm.refcount(p0) == g["refcount_before"]
    bm.free_seq(0)
    assert bm.refcount(p0) == g["refcount_after_one_teardown"]
    assert bm.num_free() == 6   # nothing returned yet
    bm.free_seq(1)
    assert bm.refcount(p0) == 0 and bm.num_free() == 8


def test_shared_prefix_mix_gives_127_copies(pkv):
    bm = pkv.BlockManager(128 * 70, 16)
    bm.add_seq(0)
    bm.append(0, 2056)
    for s in range(1, 128):
        bm.fork(0, s)
    table, _ = bm.block_table([0], 200)
    assert all(bm.refcount(int(b)) == 128 for b in table[0][table[0] >= 0])
    total = 0
    for s in range(128):
        _, pairs = bm.append(s, 16 + s)
        total += len(pairs)
    assert total == 127


def test_worked_example_2_real_count(pkv, golden):
    g = golden["worked_example_2"]
    bm = pkv.BlockManager(20000, 16)
    bm.add_seq(0)
    bm.append(0, g["prompt_len"])
    for s in range(1, g["num_requests"]):
        bm.fork(0, s)
    for s in range(g["num_requests"]):
        bm.append(s, g["suffix_len"])
    assert 20000 - bm.num_free() == 3523   # see oracle test: not 3024


def test_exhaustion_is_atomic(pkv):
    bm = pkv.BlockManager(3, 16)
    bm.add_seq(0)
    bm.append(0, 40)
    before = bm.block_table([0], 4)
    with pytest.raises(pkv.NoFreeBlocksError):
        bm.append(0, 9)
    after = bm.block_table([0], 4)
    assert np.array_equal(before[0], after[0]) and before[1][0] == after[1][0]
    bm.append(0, 8)
    assert bm.num_free() == 0


def test_errors(pkv):
    bm = pkv.BlockManager(4, 16)
    bm.add_seq(1)
    with pytest.raises(pkv.PagedKVError, match="exists"):
        bm.add_seq(1)
    with pytest.raises(pkv.PagedKVError):
        bm.append(99, 1)
    with pytest.raises(pkv.PagedKVError):
        bm.fork(99, 2)
    with pytest.raises(pkv.PagedKVError):
        bm.truncate(1, 5)
    bm.append(1, 40)
    with pytest.raises(pkv.PagedKVError, match="columns"):
        bm.block_table([1], 2)
    with pytest.raises(pkv.PagedKVError, match="permutation"):
        pkv.BlockManager(4, 16, free_order=[0, 1, 1, 2])
    assert bm.seq_len(1) == 40 and bm.seq_len(5) == -1


def test_append_batch_matches_single_appends(pkv):
    order = np.random.default_rng(3).permutation(200).astype(np.int32)
    a = pkv.BlockManager(200, 16, free_order=order)
    b = pkv.BlockManager(200, 16, free_order=order)
    for bm in (a, b):
        bm.add_seq(0)
        bm.append(0, 20)
        for s in (1, 2, 3):
            bm.fork(0, s)
    ids, n = [0, 1, 2, 3], [3, 17, 1, 40]
    slots, pairs = a.append_batch(ids, n)
    exp_slots, exp_pairs = [], []
    for s, k in zip(ids, n):
        sl, pr = b.append(s, k)
        exp_slots += list(sl)
        exp_pairs += [tuple(x) for x in pr]
    assert list(slots) == exp_slots
    assert [tuple(x) for x in pairs] == exp_pairs and len(pairs) == 3
    assert a.block_table(ids, 8)[0].tolist() == b.block_table(ids, 8)[0].tolist()


def test_append_batch_partial_failure(pkv):
    bm = pkv.BlockManager(4, 16)
    for s in range(3):
        bm.add_seq(s)
    with pytest.raises(pkv.NoFreeBlocksError) as ei:
        bm.append_batch([0, 1, 2], [16, 50, 1])
    assert ei.value.num_done == 1
    assert bm.seq_len(0) == 16 and bm.seq_len(1) == 0 and bm.seq_len(2) == 0


def test_num_used_counts_tables_and_cache(pkv):
    bm = pkv.BlockManager(32, 4)
    assert bm.num_used() == 0
    bm.add_seq(0)
    bm.append(0, 9)                       # 3 blocks
    bm.fork(0, 1)                         # shared: still 3
    assert bm.num_used() == 3
    bm.cache_insert(0, list(range(8)))    # 2 full blocks cached
    bm.free_seq(0)
    bm.free_seq(1)
    assert bm.num_used() == 2             # the cache still holds them
    assert bm.num_used() + bm.num_free() == 32


def test_pool_blocks_from_bytes(pkv):
    import torch
    # Llama-3-70B shape: 80 layers, 8 KV heads of 128 dims, bf16.  Per token
    # 2 (K, V) x 80 x 8 x 128 x 2 B = 327,680 B (the pages' 2 x layers x
    # hidden x bytes with the grouped-query width 8 x 128); 8,192 tokens
    # take 2.68 GB.
    per_token = 2 * 80 * 8 * 128 * 2
    assert per_token == 327_680
    assert per_token * 8192 == 2_684_354_560
    n = pkv.pa_pool_blocks(per_token * 16 * 1000, 80, 8, 128, 16,
                           torch.bfloat16)
    assert n == 1000
    assert pkv.pa_pool_blocks(per_token * 16 * 1000 - 1, 80, 8, 128, 16,
                              torch.float16) == 999
    # one layer, the batch-256 mix's pool: 4,096 B per token, block 16
    assert pkv.pa_pool_blocks(64 << 30, 1, 8, 128, 16, torch.bfloat16) == \
        (64 << 30) // (4096 * 16)
    with pytest.raises(pkv.PagedKVError):
        pkv.pa_pool_blocks(1 << 30, 0, 8, 128, 16, torch.bfloat16)
    with pytest.raises(TypeError):
        pkv.pa_pool_blocks(1 << 30, 1, 8, 128, 16, torch.float32)
