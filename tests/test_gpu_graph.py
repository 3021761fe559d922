"""A decode step (cache write of the new tokens, then pa_decode) captured in a
CUDA graph replays with the same results as eager calls.  Capture records
the library's launches (the prep kernel, the decode, the reduce) with their
programmatic-launch edges; replays read whatever the captured input buffers
hold at replay time."""
import numpy as np
import pytest
import torch

from paged_kv_cache_383_b200 import workloads as wl

from oracle import attention as oa

from helpers import check_decode, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,ps", [("llama3_8b_gqa4", 0),
                                     ("llama3_8b_gqa4", 64),
                                     ("tiny_mha_d64", 0)])
def test_captured_step_replays_like_eager(pkv, name, ps):
    w = wl.WORKLOADS[name]
    if name == "llama3_8b_gqa4":
        w = w.scaled(num_seqs=16, low=100, high=1500)
    w = wl.replace(w, new_token=True)
    inp = wl.make_paged(w, device="cuda")
    dev = inp.q.device
    bt = torch.from_numpy(inp.block_tables).to(dev)
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).to(dev)
    slots = torch.from_numpy(inp.new_slots).to(dev)
    q = inp.q.clone()
    k_new, v_new = inp.k_new.clone(), inp.v_new.clone()
    out = torch.empty_like(q)
    desc = pkv.make_desc(q, inp.k_cache, bt, partition_size=ps,
                         max_context_len=int(inp.lengths.max()))
    ws = torch.empty(pkv.pa_decode_workspace_bytes(desc), dtype=torch.uint8,
                     device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    k0, v0 = to_np(inp.k_cache), to_np(inp.v_cache)   # before any write

    def step():
        pkv.pa_cache_write(inp.k_cache, inp.v_cache, k_new, v_new, slots,
                           dev_err=err)
        pkv.pa_decode(out, q, inp.k_cache, inp.v_cache, bt, cl,
                      w.softmax_scale, desc=desc, workspace=ws, dev_err=err)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                      # first use configures the kernels
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    launches = pkv.pa_launch_count()
    with torch.cuda.graph(graph):
        step()
    captured = pkv.pa_launch_count() - launches

    g = torch.Generator(device=dev)
    for trial in range(2):
        g.manual_seed(100 + trial)
        q.copy_(torch.randn(q.shape, generator=g, device=dev).to(q.dtype))
        k_new.copy_(torch.randn(k_new.shape, generator=g,
                                device=dev).to(k_new.dtype))
        v_new.copy_(torch.randn(v_new.shape, generator=g,
                                device=dev).to(v_new.dtype))
        graph.replay()
        torch.cuda.synchronize()
        replayed = out.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(replayed, out), trial
    assert err.item() == 0
    assert captured >= 3            # write, prep, decode (+ reduce)
    # expected cache: the inputs with the last new tokens scattered on the
    # host into their slots (a byte copy), then the oracle
    bs = w.block_size
    for t, slot in enumerate(inp.new_slots):
        k0[slot // bs, :, slot % bs] = to_np(k_new[t])
        v0[slot // bs, :, slot % bs] = to_np(v_new[t])
    seqs = list(range(min(4, w.num_seqs)))
    ref = oa.paged_decode(to_np(q), k0, v0, inp.block_tables, inp.lengths,
                          w.softmax_scale, seqs=seqs)
    check_decode(to_np(replayed)[seqs], ref[seqs], q.dtype, "graph replay")
    del graph


def test_captured_copy_and_prefill_replay_like_eager(pkv):
    lens = (100, 300, 37)
    w = wl.Workload("graph_prefill", 77, len(lens), 32, 8, 128, 16,
                    "bfloat16", "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, (30, 120, 37), device="cuda")
    inp = pin.paged
    dev = inp.k_cache.device
    bt = torch.from_numpy(inp.block_tables).to(dev)
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).to(dev)
    qs = torch.from_numpy(pin.query_start).to(dev)
    free = np.setdiff1d(np.arange(inp.num_blocks), inp.block_tables)
    pairs = torch.tensor([[int(inp.block_tables[0, 0]), int(free[0])]],
                         dtype=torch.int32, device=dev)
    q = pin.q.clone()
    out = torch.empty_like(q)
    kw = dict(max_q_len=120, max_context_len=300)

    def step():
        pkv.pa_copy_blocks(inp.k_cache, inp.v_cache, pairs)
        pkv.pa_prefill(out, q, inp.k_cache, inp.v_cache, bt, cl, qs,
                       w.softmax_scale, **kw)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    g = torch.Generator(device=dev)
    for trial in range(2):
        g.manual_seed(200 + trial)
        q.copy_(torch.randn(q.shape, generator=g, device=dev).to(q.dtype))
        graph.replay()
        torch.cuda.synchronize()
        replayed = out.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(replayed, out), trial
    src, dst = int(pairs[0, 0]), int(pairs[0, 1])
    assert torch.equal(inp.k_cache[dst], inp.k_cache[src])
    del graph
