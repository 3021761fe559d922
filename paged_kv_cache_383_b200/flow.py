"""Host orchestration of one decode step over the library's calls.

Order on one stream, as the pages require a private copy before the first
write into a shared block ([KV-cache chapter] "PagedAttention: borrowing
virtual memory..."): block manager append (host) -> pa_copy_blocks ->
pa_cache_write -> pa_decode.  Only argument marshalling and host<->device
copies of the integer arrays happen here.
"""
from __future__ import annotations

import numpy as np

from . import BlockManager, pa_cache_write, pa_copy_blocks


def write_tokens(bm: BlockManager, k_cache, v_cache, seq_ids, n_tokens, k, v,
                 dev_err=None, stream=None):
    """Append ``n_tokens[i]`` tokens to ``seq_ids[i]`` in the block manager,
    copy any shared partial block first, then scatter the tokens' K/V rows
    (``k``, ``v``: [sum(n_tokens), Hkv, D], sequences in order) into their
    slots.  Returns (slots, cow_pairs) as host arrays."""
    import torch
    slots, pairs = bm.append_batch(seq_ids, n_tokens)
    dev = k_cache.device
    if len(pairs):
        pa_copy_blocks(k_cache, v_cache,
                       torch.from_numpy(pairs).to(dev, non_blocking=True),
                       dev_err=dev_err, stream=stream)
    if len(slots):
        pa_cache_write(k_cache, v_cache, k, v,
                       torch.from_numpy(slots).to(dev, non_blocking=True),
                       dev_err=dev_err, stream=stream)
    return slots, pairs


def shared_prefix_batch(bm: BlockManager, k_cache, v_cache, prefix_k,
                        prefix_v, num_seqs: int, dev_err=None):
    """Sequence 0 takes the prefix tokens and writes their K/V; sequences
    1..num_seqs-1 fork from it, so every prefix block has reference count
    num_seqs."""
    bm.add_seq(0)
    write_tokens(bm, k_cache, v_cache, [0], [prefix_k.shape[0]], prefix_k,
                 prefix_v, dev_err=dev_err)
    for s in range(1, num_seqs):
        bm.fork(0, s)


def tables_on_device(bm: BlockManager, seq_ids, max_blocks: int, device):
    import torch
    table, lens = bm.block_table(seq_ids, max_blocks)
    return (torch.from_numpy(table).to(device),
            torch.from_numpy(lens).to(device), lens.astype(np.int64))
