"""GPU: pa_decode_noalloc, the decode entry point that allocates nothing.

It exists for callers that cannot allocate device memory (a serving process
whose HBM is committed to the KV-cache pool, a C host program without a
device allocator): its workspace is a fixed scratch area inside the library.
This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must also pass on its own in a
fresh process.

Checked through the C ABI.  The no-alloc call runs the same kernels as
pa_decode with a caller workspace, so the outputs must be bit-identical, and
both must meet the decode tolerance against the fp64 oracle.  The area keeps
the previous call's contents, so the calls come in sequences that would let
a stale partial from an earlier call reach the output: two calls in a row,
and calls of different shapes queued back to back on one stream with no
synchronisation between them (many partitions through the reduce kernel,
then fewer through the fused combine, then a single partition).  A shape
whose scratch would not fit is refused.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_383_b200 import _lib
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_decode, oracle_paged_sample, to_np

pytestmark = pytest.mark.gpu


def _inputs(name, **scaled):
    w = wl.WORKLOADS[name].scaled(**scaled)
    inp = wl.make_paged(w, device="cuda")
    bt = torch.from_numpy(inp.block_tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    return w, inp, bt, cl


def _noalloc(lib, out, inp, bt, cl, scale, desc, err, stream):
    """One pa_decode_noalloc call through the C ABI (no synchronisation)."""
    st = lib.pa_decode_noalloc(
        out.data_ptr(), inp.q.data_ptr(), inp.k_cache.data_ptr(),
        inp.v_cache.data_ptr(), bt.data_ptr(), cl.data_ptr(),
        ctypes.c_float(scale), ctypes.byref(desc), err.data_ptr(), stream)
    assert st == _lib.PA_OK, lib.pa_last_error()


def _with_workspace(pkv, inp, bt, cl, scale, **kw):
    want = torch.empty_like(inp.q)
    pkv.pa_decode(want, inp.q, inp.k_cache, inp.v_cache, bt, cl, scale, **kw)
    return want


def _check_oracle(w, inp, out):
    seqs = list(range(len(inp.lengths)))
    ref = oracle_paged_sample(inp.q, inp.k_cache, inp.v_cache,
                              inp.block_tables, inp.lengths,
                              w.softmax_scale, seqs)
    got = to_np(out)
    check_decode(got[seqs], np.stack([ref[b] for b in seqs]), out.dtype,
                 "pa_decode_noalloc vs oracle")


@pytest.mark.parametrize("name,scaled,ps,reduce", [
    ("llama3_70b_gqa8", dict(num_seqs=12, cap=3000), 512, "auto"),
    ("long_context_split", dict(num_seqs=2, low=9000, high=12000), 512,
     "kernel"),
    ("llama3_8b_gqa4", dict(num_seqs=6, low=100, high=900), 1024, "auto"),
])
def test_noalloc_matches_workspace_path(pkv, name, scaled, ps, reduce):
    w, inp, bt, cl = _inputs(name, **scaled)
    max_ctx = int(inp.lengths.max())
    kw = dict(partition_size=ps, reduce=reduce, max_context_len=max_ctx)
    want = _with_workspace(pkv, inp, bt, cl, w.softmax_scale, **kw)
    desc = pkv.make_desc(inp.q, inp.k_cache, bt, **kw)
    assert 0 < pkv.pa_decode_workspace_bytes(desc) or ps >= max_ctx
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        got = torch.full_like(inp.q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        _noalloc(lib, got, inp, bt, cl, w.softmax_scale, desc, err, stream)
        torch.cuda.synchronize()
        assert err.item() == 0
        assert torch.equal(got, want), (call, name)
    _check_oracle(w, inp, got)


def test_noalloc_shapes_back_to_back_on_one_stream(pkv):
    """Three shapes, queued with no synchronisation: each call's prep kernel
    resets the counters and rewrites the order while the previous call's
    kernels may still be draining (programmatic launch), and a call with
    fewer partitions follows one that left more partials in the area."""
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [
        # 128-token partitions over up to 3000 tokens: 24 partitions, the
        # separate reduce kernel with one partition per consumer warp
        (("llama3_70b_gqa8", dict(num_seqs=16, cap=3000)), 128, "kernel"),
        # 512-token partitions: up to 6, the fused last-CTA combine
        (("llama3_70b_gqa8", dict(num_seqs=10, cap=2500)), 512, "auto"),
        # one partition covers every sequence: no partials at all
        (("llama3_8b_gqa4", dict(num_seqs=5, low=100, high=600)), 1024,
         "auto"),
    ]
    runs = []
    for (name, scaled), ps, reduce in cases:
        w, inp, bt, cl = _inputs(name, **scaled)
        kw = dict(partition_size=ps, reduce=reduce,
                  max_context_len=int(inp.lengths.max()))
        want = _with_workspace(pkv, inp, bt, cl, w.softmax_scale, **kw)
        desc = pkv.make_desc(inp.q, inp.k_cache, bt, **kw)
        runs.append((w, inp, bt, cl, desc, want))
    torch.cuda.synchronize()
    for rep in range(2):
        outs = []
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for w, inp, bt, cl, desc, _ in runs:
            got = torch.full_like(inp.q, float("nan"))
            _noalloc(lib, got, inp, bt, cl, w.softmax_scale, desc, err,
                     stream)
            outs.append(got)
        torch.cuda.synchronize()
        assert err.item() == 0
        for i, ((w, inp, _, _, _, want), got) in enumerate(zip(runs, outs)):
            assert torch.equal(got, want), (rep, i)
    for (w, inp, _, _, _, _), got in zip(runs, outs):
        _check_oracle(w, inp, got)


def test_noalloc_rejects_shapes_beyond_its_scratch(pkv):
    w, inp, bt, cl = _inputs("llama3_70b_gqa8", num_seqs=4, cap=3000)
    # 64 q heads x 4 seqs x 8192/16 partitions x 130 floats: far over 32 MiB
    desc = pkv.make_desc(inp.q, inp.k_cache, bt, partition_size=16,
                         max_context_len=8192)
    need = pkv.pa_decode_workspace_bytes(desc)
    assert need > _lib.PA_NOALLOC_SCRATCH_BYTES
    out = torch.empty_like(inp.q)
    with pytest.raises(pkv.PagedKVError, match="built-in area"):
        pkv.pa_decode_noalloc(out, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                              w.softmax_scale, desc=desc)
