"""GPU: whole decode steps against the oracle's contiguous attention.

* shared-prefix mix: fork, append (copy-on-write of the shared partial block),
  pa_copy_blocks, pa_cache_write, pa_decode -- compared with attention over
  each sequence's logical tokens (prefix then its own suffix), so the expected
  values do not depend on any table or slot the library produced;
* new-token step of the 64-sequence workload: the new token's K/V written
  through its slot, then decode over all tokens.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import flow
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_decode, sample_seqs, to_np

pytestmark = pytest.mark.gpu


def _noise_pool(nb, w, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dt = wl.torch_dtype(w.dtype)
    shape = (nb, w.num_kv_heads, w.block_size, w.head_dim)
    return (torch.randn(shape, generator=g, device="cuda").to(dt),
            torch.randn(shape, generator=g, device="cuda").to(dt))


def _prefix_step(pkv, w, seqs_to_check):
    inp = wl.make_prefix(w, device="cuda")
    kc, vc = _noise_pool(inp.num_blocks, w, w.seed + 1)
    bm = pkv.BlockManager(inp.num_blocks, w.block_size,
                          free_order=inp.free_order)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flow.shared_prefix_batch(bm, kc, vc, inp.prefix_k, inp.prefix_v,
                             w.num_seqs, dev_err=err)
    ids = list(range(w.num_seqs))
    slots, pairs = flow.write_tokens(bm, kc, vc, ids, inp.suffix_lens,
                                     inp.suffix_k, inp.suffix_v, dev_err=err)
    max_blocks = int(wl.blocks_needed(inp.lengths, w.block_size).max())
    bt, cl, lens = flow.tables_on_device(bm, ids, max_blocks, "cuda")
    assert np.array_equal(lens, inp.lengths)
    out = torch.empty_like(inp.q)
    pkv.pa_decode(out, inp.q, kc, vc, bt, cl, w.softmax_scale,
                  max_context_len=int(lens.max()), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    starts = np.concatenate([[0], np.cumsum(inp.suffix_lens)])
    K = [torch.cat([inp.prefix_k, inp.suffix_k[starts[b]:starts[b + 1]]])
         for b in range(w.num_seqs)]
    V = [torch.cat([inp.prefix_v, inp.suffix_v[starts[b]:starts[b + 1]]])
         for b in range(w.num_seqs)]
    seqs = seqs_to_check(inp.lengths)
    ref = oa.contiguous_decode(to_np(inp.q), [to_np(k) for k in K],
                               [to_np(v) for v in V], w.softmax_scale,
                               seqs=seqs)
    for b in seqs:
        check_decode(to_np(out[b]), ref[b], inp.q.dtype, f"prefix seq {b}")
    return pairs, bm


def test_shared_prefix_small(pkv):
    w = wl.WORKLOADS["shared_prefix_cow"].scaled(num_seqs=6, prefix_len=200,
                                                 low=16, high=100)
    pairs, bm = _prefix_step(pkv, w, lambda L: list(range(len(L))))
    assert len(pairs) == 5          # every writer but the last copies


def test_shared_prefix_full_size(pkv):
    w = wl.WORKLOADS["shared_prefix_cow"]
    pairs, bm = _prefix_step(pkv, w, lambda L: sample_seqs(L, k=6))
    assert len(pairs) == 127
    assert all(bm.refcount(int(s)) == 1 for s, _ in pairs[-1:])


@pytest.mark.parametrize("scale", ["small", "full"])
def test_new_token_step(pkv, scale):
    w = wl.WORKLOADS["llama3_8b_gqa4"]
    if scale == "small":
        w = w.scaled(num_seqs=5, low=30, high=600)
    inp = wl.make_paged(w, device="cuda")
    seqs = list(range(w.num_seqs)) if scale == "small" else \
        sample_seqs(inp.lengths, k=6)
    # logical K/V of the checked sequences, taken before the write
    K, V = {}, {}
    for b in seqs:
        L = int(inp.lengths[b])
        nblk = -(-L // w.block_size)
        idx = torch.from_numpy(inp.block_tables[b, :nblk].astype(np.int64))
        kc = to_np(inp.k_cache[idx.cuda()])
        vc = to_np(inp.v_cache[idx.cuda()])
        sub = np.arange(nblk)
        K[b] = np.concatenate([np.stack(
            [oa.depage(kc, sub, L - 1, h, w.block_size)
             for h in range(w.num_kv_heads)], axis=1),
            to_np(inp.k_new[b])[None]])
        V[b] = np.concatenate([np.stack(
            [oa.depage(vc, sub, L - 1, h, w.block_size)
             for h in range(w.num_kv_heads)], axis=1),
            to_np(inp.v_new[b])[None]])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_cache_write(inp.k_cache, inp.v_cache, inp.k_new, inp.v_new,
                       torch.from_numpy(inp.new_slots).cuda(), dev_err=err)
    out = torch.empty_like(inp.q)
    pkv.pa_decode(out, inp.q, inp.k_cache, inp.v_cache,
                  torch.from_numpy(inp.block_tables).cuda(),
                  torch.from_numpy(inp.lengths.astype(np.int32)).cuda(),
                  w.softmax_scale, max_context_len=int(inp.lengths.max()),
                  dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    qn = to_np(inp.q)
    for b in seqs:
        ref = oa.contiguous_decode(qn[b:b + 1], [K[b]], [V[b]],
                                   w.softmax_scale)[0]
        check_decode(to_np(out[b]), ref, inp.q.dtype, f"new-token seq {b}")
