"""GPU tests of pa_swap_blocks with the block manager's swap: sequences are
swapped out to a pinned host pool, their device blocks are reused (and
overwritten), and after swapping back in the decode output is bit-identical
to the output before the swap and within tolerance of the oracle.  The copy
itself is checked byte for byte."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_decode, to_np

pytestmark = pytest.mark.gpu


def _decode(pkv, inp, bt, cl, kc, vc):
    out = torch.empty_like(inp.q)
    pkv.pa_decode(out, inp.q, kc, vc, bt, cl, inp.workload.softmax_scale,
                  max_context_len=int(inp.lengths.max()))
    torch.cuda.synchronize()
    return out


def _setup(pkv, bs=16, n=12, seed=31):
    w = wl.WORKLOADS["llama3_8b_gqa4"].scaled(num_seqs=n, low=20, high=700)
    w = wl.replace(w, seed=seed, block_size=bs, new_token=False)
    inp = wl.make_paged(w, device="cuda")
    # the block manager reproduces the tables: one sequence per row, blocks
    # taken in the order the workload assigned them
    order = np.concatenate([inp.block_tables[b][inp.block_tables[b] >= 0]
                            for b in range(n)])
    rest = np.setdiff1d(np.arange(inp.num_blocks), order)
    bm = pkv.BlockManager(inp.num_blocks, bs,
                          free_order=np.concatenate([order, rest])
                          .astype(np.int32))
    for b in range(n):
        bm.add_seq(b)
        bm.append(b, int(inp.lengths[b]))
    table, lens = bm.block_table(list(range(n)), inp.max_blocks)
    assert (table == inp.block_tables).all()
    return w, inp, bm


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("pairs_on_host", [False, True])
def test_swap_round_trip_bit_exact(pkv, bs, pairs_on_host):
    w, inp, bm = _setup(pkv, bs)
    n = w.num_seqs
    kc, vc = inp.k_cache, inp.v_cache
    bt = torch.from_numpy(inp.block_tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    before = _decode(pkv, inp, bt, cl, kc, vc)
    group = [1, 4, 5, 9]
    ref = oa.paged_decode(to_np(inp.q), to_np(kc), to_np(vc),
                          inp.block_tables, inp.lengths, w.softmax_scale,
                          seqs=group)
    nh = inp.num_blocks
    bm.set_host_blocks(nh)
    hk = torch.empty((nh,) + tuple(kc.shape[1:]), dtype=kc.dtype,
                     pin_memory=True)
    hv = torch.empty_like(hk, pin_memory=True)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def as_pairs(p):
        t = torch.from_numpy(np.ascontiguousarray(p))
        return t.pin_memory() if pairs_on_host else t.cuda()

    out_pairs = bm.swap_out(group)
    pairs = as_pairs(out_pairs)
    pkv.pa_swap_blocks(hk, hv, kc, vc, pairs, dev_err=err)
    torch.cuda.synchronize()
    src = torch.from_numpy(out_pairs[:, 0].astype(np.int64))
    dst = torch.from_numpy(out_pairs[:, 1].astype(np.int64))
    assert torch.equal(hk[dst], kc.cpu()[src])
    assert torch.equal(hv[dst], vc.cpu()[src])
    # the freed device blocks get new contents before the swap-in
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    freed = src.cuda()
    kc[freed] = torch.randn(kc[freed].shape, generator=g,
                            device="cuda").to(kc.dtype)
    vc[freed] = torch.randn(vc[freed].shape, generator=g,
                            device="cuda").to(vc.dtype)
    # other requests take blocks meanwhile, in reverse order of release
    bm.add_seq(100)
    bm.append(100, 3 * bs)
    in_pairs = bm.swap_in(group[::-1])
    pkv.pa_swap_blocks(kc, vc, hk, hv, as_pairs(in_pairs), dev_err=err)
    table, lens = bm.block_table(list(range(n)), inp.max_blocks)
    assert list(lens) == list(inp.lengths)
    moved = [b for b in range(n) if b in group]
    assert all((table[b] != inp.block_tables[b]).any() for b in moved
               if inp.lengths[b] > 3 * bs)
    after = _decode(pkv, inp, torch.from_numpy(table).cuda(), cl, kc, vc)
    assert err.item() == 0
    assert torch.equal(after, before)
    check_decode(to_np(after)[group], ref[group], inp.q.dtype, "swapped")


def test_bad_pair_is_flagged_and_skipped(pkv):
    w, inp, bm = _setup(pkv)
    kc, vc = inp.k_cache, inp.v_cache
    hk = torch.zeros((4,) + tuple(kc.shape[1:]), dtype=kc.dtype,
                     pin_memory=True)
    hv = torch.zeros_like(hk, pin_memory=True)
    pairs = torch.tensor([[0, 0], [1, 9], [2, 2]], dtype=torch.int32,
                         device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_swap_blocks(hk, hv, kc, vc, pairs, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    assert torch.equal(hk[0], kc[0].cpu()) and torch.equal(hk[2], kc[2].cpu())
    assert not hk[1].any() and not hk[3].any()


def test_pageable_host_memory_is_refused(pkv):
    w, inp, bm = _setup(pkv)
    kc, vc = inp.k_cache, inp.v_cache
    hk = torch.zeros((4,) + tuple(kc.shape[1:]), dtype=kc.dtype)
    pairs = torch.tensor([[0, 0]], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        pkv.pa_swap_blocks(hk, hk.clone(), kc, vc, pairs)
    # the library's own check, reached without the binding's
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    hv = hk.clone()
    before = pkv.pa_launch_count()
    st = lib.pa_swap_blocks(hk.data_ptr(), hv.data_ptr(), kc.data_ptr(),
                            vc.data_ptr(), pairs.data_ptr(), 1,
                            kc.shape[1], kc.shape[3], kc.shape[2],
                            kc.shape[0], 4, _lib.PA_BF16, None,
                            torch.cuda.current_stream().cuda_stream)
    assert st == _lib.PA_ERR_INVALID_ARG
    assert "page-locked" in lib.pa_last_error().decode()
    assert pkv.pa_launch_count() == before
