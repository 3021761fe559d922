"""Seeded synthetic inputs for the five decode workloads.

This module only draws random inputs and lays out their structure (lengths,
which physical blocks each sequence owns, random values).  It holds none of
the attention arithmetic and none of the block manager's logic, so both the
CUDA path and the CPU oracle can take their inputs from it.

Workloads (shapes from the serving mixes the pages describe; the pages name no
public dataset):

* ``tiny_mha_d64``       -- 4 sequences of 47, 612, 130, 1900 tokens (the
  KV-cache chapter's Worked Example 1), block 16, a 256-block pool handed out
  by random permutation, 8 query = 8 KV heads, head_dim 64, fp16, scale 1/8.
* ``llama3_8b_gqa4``     -- 64 sequences, lengths uniform in [128, 4096],
  32 query / 8 KV heads, head_dim 128, bf16, block 16, pool 1.2x the need,
  plus one new token per sequence written through a slot mapping.
* ``llama3_70b_gqa8``    -- 256 sequences, lengths log-normal with median 1024
  (sigma 1.0 on ln tokens) clamped to [1, 8192], 64 query / 8 KV heads,
  head_dim 128, bf16, block 16 (``..._bs32``: block 32, same lengths/values).
* ``shared_prefix_cow``  -- 128 sequences sharing a 2056-token prefix, own
  suffix uniform in [16, 1024], 32 query / 8 KV heads, head_dim 128, bf16,
  block 16 (the prefix/suffix K/V are drawn here; tables come from the block
  manager).
* ``long_context_split`` -- 8 sequences, lengths uniform in [32768, 131072],
  64 query / 8 KV heads, head_dim 128, fp16, block 32, 512-token partitions.

Random draws: lengths and block permutations from ``numpy.random.
default_rng(seed)``; tensor values N(0, 1) from ``torch.Generator`` seeded
with the same seed on the target device (so values on a GPU differ from a CPU
draw with the same seed; each test or bench run takes its inputs from one
draw).  Unused pool blocks are filled with N(0, 1) noise too, so a stray read
changes the result.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                 # "float16" | "bfloat16"
    lengths: str               # "fixed" | "uniform" | "lognormal" | "prefix"
    fixed_lengths: tuple = ()
    low: int = 0
    high: int = 0
    median: float = 0.0
    sigma: float = 0.0
    cap: int = 0
    prefix_len: int = 0
    num_blocks: int = 0        # 0 -> ceil(pool_factor * need)
    pool_factor: float = 1.2
    partition_size: int = 0    # 0 -> library's automatic choice
    scale: float = 0.0         # 0 -> 1/sqrt(head_dim)
    new_token: bool = False    # one new token per sequence via cache write

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale else 1.0 / math.sqrt(self.head_dim)

    def scaled(self, num_seqs=None, cap=None, low=None, high=None,
               prefix_len=None, fixed_lengths=None) -> "Workload":
        """Same structure, smaller sizes (for oracle-sized parity runs)."""
        kw = {}
        if num_seqs is not None:
            kw["num_seqs"] = num_seqs
        if cap is not None:
            kw["cap"] = cap
        if low is not None:
            kw["low"] = low
        if high is not None:
            kw["high"] = high
        if prefix_len is not None:
            kw["prefix_len"] = prefix_len
        if fixed_lengths is not None:
            kw["fixed_lengths"] = tuple(fixed_lengths)
            kw["num_seqs"] = len(fixed_lengths)
        return replace(self, **kw)


WORKLOADS = {
    "tiny_mha_d64": Workload(
        "tiny_mha_d64", 383001, 4, 8, 8, 64, 16, "float16", "fixed",
        fixed_lengths=(47, 612, 130, 1900), num_blocks=256, scale=0.125),
    "llama3_8b_gqa4": Workload(
        "llama3_8b_gqa4", 383002, 64, 32, 8, 128, 16, "bfloat16", "uniform",
        low=128, high=4096, new_token=True),
    "llama3_70b_gqa8": Workload(
        "llama3_70b_gqa8", 383003, 256, 64, 8, 128, 16, "bfloat16",
        "lognormal", median=1024.0, sigma=1.0, cap=8192),
    "llama3_70b_gqa8_bs32": Workload(
        "llama3_70b_gqa8_bs32", 383003, 256, 64, 8, 128, 32, "bfloat16",
        "lognormal", median=1024.0, sigma=1.0, cap=8192),
    "shared_prefix_cow": Workload(
        "shared_prefix_cow", 383004, 128, 32, 8, 128, 16, "bfloat16",
        "prefix", low=16, high=1024, prefix_len=2056),
    "long_context_split": Workload(
        "long_context_split", 383005, 8, 64, 8, 128, 32, "float16", "uniform",
        low=32768, high=131072, partition_size=512),
}


def draw_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """Context length of every sequence (the newest token included)."""
    if w.lengths == "fixed":
        return np.array(w.fixed_lengths, dtype=np.int64)
    if w.lengths == "uniform":
        return rng.integers(w.low, w.high + 1, size=w.num_seqs).astype(np.int64)
    if w.lengths == "lognormal":
        x = np.exp(rng.normal(math.log(w.median), w.sigma, size=w.num_seqs))
        return np.clip(np.rint(x), 1, w.cap).astype(np.int64)
    if w.lengths == "prefix":
        suffix = rng.integers(w.low, w.high + 1, size=w.num_seqs)
        return (w.prefix_len + suffix).astype(np.int64)
    raise ValueError(w.lengths)


def blocks_needed(lengths, block_size: int) -> np.ndarray:
    """Blocks each sequence occupies when its tokens fill blocks in order."""
    lengths = np.asarray(lengths, dtype=np.int64)
    return (lengths + block_size - 1) // block_size


@dataclass
class PagedInputs:
    """Host-side structure of one decode batch plus device/CPU tensors."""
    workload: Workload
    lengths: np.ndarray        # int64 [B]
    block_tables: np.ndarray   # int32 [B, max_blocks], -1 padded
    num_blocks: int
    q: object                  # torch [B, Hq, D]
    k_cache: object            # torch [NB, Hkv, bs, D]
    v_cache: object
    k_new: object = None       # torch [B, Hkv, D] (new-token workloads)
    v_new: object = None
    new_slots: np.ndarray = None  # int64 [B]: slot of position L-1

    @property
    def max_blocks(self) -> int:
        return self.block_tables.shape[1]


def torch_dtype(name: str):
    import torch
    return {"float16": torch.float16, "bfloat16": torch.bfloat16}[name]


def make_paged(w: Workload, device="cpu", values=True) -> PagedInputs:
    """Random lengths, a random assignment of physical blocks (a permutation
    of the pool, handed out to the sequences' logical blocks in order, as a
    fresh pool would), and N(0, 1) values for q and the whole pool."""
    import torch
    rng = np.random.default_rng(w.seed)
    lengths = draw_lengths(w, rng)
    nblk = blocks_needed(lengths, w.block_size)
    need = int(nblk.sum())
    num_blocks = w.num_blocks or int(math.ceil(w.pool_factor * need))
    if num_blocks < need:
        raise ValueError("pool smaller than the blocks needed")
    perm = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = max(int(nblk.max()), 1)
    tables = np.full((w.num_seqs, max_blocks), -1, dtype=np.int32)
    start = 0
    for b in range(w.num_seqs):
        tables[b, : nblk[b]] = perm[start: start + nblk[b]]
        start += nblk[b]
    new_slots = None
    if w.new_token:
        pos = lengths - 1
        new_slots = (tables[np.arange(w.num_seqs), pos // w.block_size]
                     .astype(np.int64) * w.block_size + pos % w.block_size)
    if not values:
        return PagedInputs(w, lengths, tables, num_blocks, None, None, None,
                           new_slots=new_slots)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    shape_c = (num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    q = torch.randn(w.num_seqs, w.num_q_heads, w.head_dim, generator=g,
                    device=device, dtype=torch.float32).to(dt)
    k_cache = _randn(shape_c, g, device, dt)
    v_cache = _randn(shape_c, g, device, dt)
    out = PagedInputs(w, lengths, tables, num_blocks, q, k_cache, v_cache,
                      new_slots=new_slots)
    if w.new_token:
        shape_t = (w.num_seqs, w.num_kv_heads, w.head_dim)
        out.k_new = _randn(shape_t, g, device, dt)
        out.v_new = _randn(shape_t, g, device, dt)
    return out


def _randn(shape, g, device, dt):
    """N(0, 1) in the target dtype, drawn in fp32 chunks (bounded temp)."""
    import torch
    out = torch.empty(shape, device=device, dtype=dt)
    flat = out.view(-1)
    chunk = 1 << 26
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i: i + n] = torch.randn(n, generator=g, device=device,
                                     dtype=torch.float32).to(dt)
    return out


@dataclass
class PrefixInputs:
    """Shared-prefix workload: logical K/V of the prefix and each suffix."""
    workload: Workload
    lengths: np.ndarray        # int64 [B] = prefix + suffix
    suffix_lens: np.ndarray    # int64 [B]
    num_blocks: int
    free_order: np.ndarray     # int32 permutation of the pool
    q: object                  # [B, Hq, D]
    prefix_k: object           # [P, Hkv, D]
    prefix_v: object
    suffix_k: object           # [sum(suffix), Hkv, D], sequences in order
    suffix_v: object
    pool_fill_seed: int = 0


def make_prefix(w: Workload, device="cpu") -> PrefixInputs:
    """Prefix K/V shared by every sequence, per-sequence suffix K/V, q, and a
    random hand-out order of a pool 1.2x the blocks the batch needs once the
    prefix is shared (plus one private copy of the partial prefix block per
    sequence)."""
    import torch
    rng = np.random.default_rng(w.seed)
    lengths = draw_lengths(w, rng)
    suffix = lengths - w.prefix_len
    bs = w.block_size
    shared = int(blocks_needed([w.prefix_len], bs)[0])
    own = int(blocks_needed(lengths, bs).sum()) - w.num_seqs * (
        w.prefix_len // bs)
    need = shared + own + w.num_seqs
    num_blocks = w.num_blocks or int(math.ceil(w.pool_factor * need))
    free_order = rng.permutation(num_blocks).astype(np.int32)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    H, D = w.num_kv_heads, w.head_dim
    q = torch.randn(w.num_seqs, w.num_q_heads, D, generator=g, device=device,
                    dtype=torch.float32).to(dt)
    pk = _randn((w.prefix_len, H, D), g, device, dt)
    pv = _randn((w.prefix_len, H, D), g, device, dt)
    total = int(suffix.sum())
    sk = _randn((total, H, D), g, device, dt)
    sv = _randn((total, H, D), g, device, dt)
    return PrefixInputs(w, lengths, suffix, num_blocks, free_order, q, pk, pv,
                        sk, sv)


@dataclass
class PrefillInputs:
    """A paged batch plus query rows for each sequence's newest tokens."""
    paged: PagedInputs
    q_lens: np.ndarray         # int64 [B]: new tokens per sequence (<= L)
    query_start: np.ndarray    # int32 [B+1]
    q: object                  # torch [sum(q_lens), Hq, D]


def make_prefill(w: Workload, q_lens, device="cpu",
                 seed_offset: int = 17) -> PrefillInputs:
    """``make_paged`` for the cache, plus N(0, 1) query rows for the last
    ``q_lens[b]`` tokens of every sequence (clipped to its length)."""
    import torch
    inp = make_paged(w, device=device)
    q_lens = np.minimum(np.asarray(q_lens, dtype=np.int64), inp.lengths)
    start = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + seed_offset)
    q = torch.randn(int(start[-1]), w.num_q_heads, w.head_dim, generator=g,
                    device=device, dtype=torch.float32).to(
                        torch_dtype(w.dtype))
    return PrefillInputs(inp, q_lens, start, q)


# Prefill workloads (tensor-core bound): Llama-3-70B heads, block 16, bf16.
# chunked: the last 512 tokens of 16 contexts uniform in [2048, 8192]
# (a chunk of a long prompt appended to what is cached); prompt: 8 whole
# prompts uniform in [1024, 8192] (every token new).
WORKLOADS["chunked_prefill_gqa8"] = Workload(
    "chunked_prefill_gqa8", 383006, 16, 64, 8, 128, 16, "bfloat16",
    "uniform", low=2048, high=8192)
WORKLOADS["prompt_prefill_gqa8"] = Workload(
    "prompt_prefill_gqa8", 383007, 8, 64, 8, 128, 16, "bfloat16",
    "uniform", low=1024, high=8192)
