"""fp64 oracle for single-query (decode) attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What it computes.  [vLLM PagedAttention FAQ], "Does PagedAttention change the
mathematical attention output?" and the "Common Misconceptions" list, and
[KV-cache chapter], "Common misconception: PagedAttention makes attention
faster", state that paging changes only where K and V sit and how they are
found; every query attends to every cached key with the same scores and the
same softmax as contiguous multi-head attention.  So the oracle is that plain
definition: first undo the paging (``depage``), then run textbook softmax
attention of one query vector over the sequence's contiguous K/V in float64.

Layout of the paged cache (the interface the library and this oracle both
read; the pages fix only that K/V live in fixed-size blocks reached through a
per-sequence block table, [Taming the Tail] "How the Architecture Works" and
"Under the Hood: The CUDA Kernel Engineering"):

* ``k_cache``, ``v_cache``: ``[num_blocks, num_kv_heads, block_size, head_dim]``
* ``block_tables``: ``[num_seqs, max_blocks_per_seq]`` physical block ids;
  entry ``i`` of row ``b`` holds logical block ``i`` of sequence ``b``
  ([KV-cache chapter] "PagedAttention: borrowing virtual memory from the
  operating system": logical block 0, 1, 2, ... mapped through a small
  per-request table to free physical blocks anywhere in the pool).
* ``context_lens``: ``[num_seqs]`` tokens of each sequence, the new token
  included (the single query sits at the last position, so no causal mask).
* ``q``: ``[num_seqs, num_q_heads, head_dim]``.

Readings where the pages are silent:

* Grouped-query attention: query head ``h`` reads KV head ``h // G`` with
  ``G = num_q_heads // num_kv_heads`` (consecutive grouping).  [Taming the
  Tail] "The Math of the Cache" names a model with 8 KV heads and grouped
  query attention but no mapping.
* A sequence with no tokens attends over an empty set; its output is the
  empty weighted sum, a zero vector.
* Inputs arrive as float32/float64 arrays that hold the exact fp16/bf16
  values; the oracle upcasts to float64 and never rounds its result.
"""
from __future__ import annotations

import numpy as np


def depage(cache: np.ndarray, table_row: np.ndarray, context_len: int,
           kv_head: int, block_size: int) -> np.ndarray:
    """Rows ``0..context_len-1`` of one sequence's K (or V) for one KV head.

    Token ``t`` lives in logical block ``t // block_size`` at offset
    ``t % block_size``; the block table row maps that logical block to a
    physical block ([Taming the Tail] "How the Architecture Works": logical
    blocks are contiguous from the model's view, physical ones are scattered,
    and the table translates one into the other).

    Returns a float64 array ``[context_len, head_dim]``.
    """
    t = np.arange(int(context_len))
    logical_block = t // block_size
    offset = t % block_size
    physical_block = np.asarray(table_row)[logical_block].astype(np.int64)
    if context_len and (physical_block.min() < 0
                        or physical_block.max() >= cache.shape[0]):
        raise IndexError("block table entry outside the physical pool")
    return np.asarray(cache[physical_block, kv_head, offset, :],
                      dtype=np.float64)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray,
           scale: float) -> np.ndarray:
    """softmax(scale * K q) V for one query vector, in float64.

    ``q`` is ``[head_dim]``, ``K`` and ``V`` are ``[L, head_dim]``.  The
    largest score is subtracted before exponentiating (it cancels between
    numerator and denominator, so the result is the textbook softmax).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    scores = float(scale) * (K @ q)
    weights = np.exp(scores - scores.max())
    weights /= weights.sum()
    return weights @ V


def kv_head_of(q_head: int, num_q_heads: int, num_kv_heads: int) -> int:
    """KV head serving query head ``q_head`` (consecutive GQA grouping)."""
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    return q_head // (num_q_heads // num_kv_heads)


def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 block_tables: np.ndarray, context_lens: np.ndarray,
                 scale: float, seqs=None) -> np.ndarray:
    """Decode attention for every (sequence, query head), in float64.

    De-pages each sequence's K and V for the KV head its query head reads,
    then applies ``attend``.  ``seqs`` optionally restricts the work to a
    subset of sequence indices (rows of the result for other sequences are
    NaN); the bench uses it to time a bounded sample.

    Returns ``[num_seqs, num_q_heads, head_dim]`` float64.
    """
    num_seqs, num_q_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[1]
    block_size = k_cache.shape[2]
    out = np.full((num_seqs, num_q_heads, head_dim), np.nan)
    for b in (range(num_seqs) if seqs is None else seqs):
        L = int(context_lens[b])
        for kvh in range(num_kv_heads):
            K = depage(k_cache, block_tables[b], L, kvh, block_size)
            V = depage(v_cache, block_tables[b], L, kvh, block_size)
            for h in range(num_q_heads):
                if kv_head_of(h, num_q_heads, num_kv_heads) == kvh:
                    out[b, h] = attend(q[b, h], K, V, scale)
    return out


def contiguous_decode(q: np.ndarray, K_seqs, V_seqs, scale: float,
                      seqs=None) -> np.ndarray:
    """Decode attention over contiguous per-sequence K/V (no paging at all).

    ``K_seqs[b]`` and ``V_seqs[b]`` are ``[L_b, num_kv_heads, head_dim]``:
    the sequence's logical tokens in order.  This is the contiguous
    multi-head attention the paged result must equal; tests of the full
    append / copy-on-write / write / decode flow compare against it, so the
    expected values never depend on how the blocks were laid out.
    """
    num_seqs, num_q_heads, head_dim = q.shape
    out = np.full((num_seqs, num_q_heads, head_dim), np.nan)
    for b in (range(num_seqs) if seqs is None else seqs):
        Kb = np.asarray(K_seqs[b], dtype=np.float64)
        Vb = np.asarray(V_seqs[b], dtype=np.float64)
        num_kv_heads = Kb.shape[1]
        for h in range(num_q_heads):
            kvh = kv_head_of(h, num_q_heads, num_kv_heads)
            out[b, h] = attend(q[b, h], Kb[:, kvh, :], Vb[:, kvh, :], scale)
    return out


def paged_prefill(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                  block_tables: np.ndarray, context_lens: np.ndarray,
                  query_start: np.ndarray, scale: float,
                  seqs=None) -> np.ndarray:
    """Causal attention of each sequence's newest tokens over its paged K/V.

    Sequence b holds ``context_lens[b]`` = L tokens in the cache, of which the
    last ``q_len = query_start[b+1] - query_start[b]`` are new and have query
    vectors ``q[query_start[b] + i]`` (i = 0 .. q_len-1).  New token i sits
    at position ``p = L - q_len + i`` and attends to positions 0 .. p (the
    tokens before it and itself), with the same scores and softmax as
    contiguous attention.  Decode is the case q_len = 1; prefilling a whole
    prompt is q_len = L; anything between is a chunk of a longer prompt, or
    several speculative tokens checked at once ([Taming the Tail] "The
    Future: Speculative Decoding and Beyond": the verifying model processes
    the draft tokens in one pass).

    ``q`` is ``[total_q, num_q_heads, head_dim]``; returns the same shape in
    float64 (NaN rows for sequences not in ``seqs``).
    """
    total_q, num_q_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[1]
    block_size = k_cache.shape[2]
    out = np.full((total_q, num_q_heads, head_dim), np.nan)
    B = len(context_lens)
    for b in (range(B) if seqs is None else seqs):
        L = int(context_lens[b])
        q0, q1 = int(query_start[b]), int(query_start[b + 1])
        q_len = q1 - q0
        if q_len > L:
            raise ValueError("more new tokens than the context holds")
        for kvh in range(num_kv_heads):
            K = depage(k_cache, block_tables[b], L, kvh, block_size)
            V = depage(v_cache, block_tables[b], L, kvh, block_size)
            for h in range(num_q_heads):
                if kv_head_of(h, num_q_heads, num_kv_heads) != kvh:
                    continue
                for i in range(q_len):
                    p = L - q_len + i
                    out[q0 + i, h] = attend(q[q0 + i, h], K[:p + 1],
                                            V[:p + 1], scale)
    return out
