"""Pins of the fragmentation / sharing oracle to the pages' printed numbers.

Every expected value comes from tests/golden/worked_examples.json, which
records what the KV-cache chapter and the other pages print, with the section.
"""
import pytest

from oracle import fragmentation as fr


def _check_report(rep, g):
    assert list(rep.blocks_per_seq) == g["blocks_per_seq"]
    assert rep.total_blocks == g["total_blocks"]
    assert rep.paged_slots == g["paged_slots"]
    assert rep.paged_slots - sum(g["lengths"]) == g["paged_waste_slots"]
    r = rep.rounded(2)
    assert r["paged_waste_pct"] == pytest.approx(g["paged_waste_pct"], abs=0)


def test_worked_example_1(golden):
    g = golden["worked_example_1"]
    rep = fr.fragmentation(g["lengths"], g["block_size"], g["max_seq_len"])
    _check_report(rep, g)
    assert rep.actual_tokens == g["actual_tokens"]
    assert rep.contiguous_slots == g["contiguous_slots"]
    assert rep.contiguous_slots - rep.actual_tokens == \
        g["contiguous_waste_slots"]
    r = rep.rounded(2)
    assert r["contiguous_waste_pct"] == g["contiguous_waste_pct"]
    assert r["reduction_factor"] == g["reduction_factor"]


def test_worked_example_1_waste_below_one_block(golden):
    g = golden["worked_example_1"]
    bound = golden["waste_bound"]["max_waste_per_seq_exclusive"]
    rep = fr.fragmentation(g["lengths"], g["block_size"], g["max_seq_len"])
    assert all(0 <= w < bound for w in rep.waste_per_seq)
    assert sum(rep.waste_per_seq) == g["paged_waste_slots"]


def test_answer_2(golden):
    g = golden["answer_2"]
    rep = fr.fragmentation(g["lengths"], g["block_size"], g["max_seq_len"])
    _check_report(rep, g)
    assert list(rep.waste_per_seq) == g["waste_per_seq"]
    assert rep.actual_tokens == g["actual_tokens"]
    assert rep.contiguous_slots - rep.actual_tokens == \
        g["contiguous_waste_slots"]
    r = rep.rounded(2)
    assert r["contiguous_waste_pct"] == g["contiguous_waste_pct"]
    assert r["reduction_factor"] == g["reduction_factor"]


def test_answer_3_block_size_tradeoff(golden):
    g = golden["answer_3"]
    rep = fr.fragmentation(g["lengths"], g["block_size"], g["max_seq_len"])
    _check_report(rep, g)
    assert list(rep.waste_per_seq) == g["waste_per_seq"]
    # table entries at the two block sizes
    rep16 = fr.fragmentation(g["lengths"], 16, g["max_seq_len"])
    assert rep16.total_blocks == g["table_entries_bs16"]
    assert rep.total_blocks == g["table_entries_bs64"]
    # whole (shareable) blocks of the 380-token prompt
    s16 = fr.shareable_prompt_blocks(g["shared_prompt_len"], 16)
    s64 = fr.shareable_prompt_blocks(g["shared_prompt_len"], 64)
    assert (s16["blocks"], s16["tokens"]) == (g["shareable_blocks_bs16"],
                                              g["shareable_tokens_bs16"])
    assert (s64["blocks"], s64["tokens"]) == (g["shareable_blocks_bs64"],
                                              g["shareable_tokens_bs64"])
    assert round(100 * s16["fraction"], 1) == g["shareable_pct_bs16"]
    assert round(100 * s64["fraction"], 1) == g["shareable_pct_bs64"]


@pytest.mark.parametrize("key", ["worked_example_2", "answer_5"])
def test_prefix_sharing_arithmetic(golden, key):
    g = golden[key]
    r = fr.sharing_blocks(g["prompt_len"], g["suffix_len"],
                          g["num_requests"], g["block_size"])
    assert r["prompt_blocks"] == g["prompt_blocks"]
    assert r["suffix_blocks"] == g["suffix_blocks"]
    assert r["without_sharing"] == g["without_sharing"]
    assert r["with_sharing"] == g["with_sharing"]
    assert round(r["reduction_factor"], 2) == g["reduction_factor"]


def test_worked_example_2_unshared_equals_whole_request(golden):
    # Worked Example 2 also counts the unshared request directly as
    # ceil(470/16) = 30 blocks.
    g = golden["worked_example_2"]
    assert fr.blocks_for(g["prompt_len"] + g["suffix_len"], 16) == \
        g["blocks_per_request_unshared"]


def test_blocks_for_edges():
    assert fr.blocks_for(0, 16) == 0
    assert fr.blocks_for(1, 16) == 1
    assert fr.blocks_for(16, 16) == 1
    assert fr.blocks_for(17, 16) == 2
    assert fr.waste_slots(16, 16) == 0
    assert fr.waste_slots(17, 16) == 15
    with pytest.raises(ValueError):
        fr.fragmentation([3000], 16, 2048)
