"""GPU: pa_decode_noalloc, the decode entry point that allocates nothing.

It exists for callers that cannot allocate device memory (a serving process
whose HBM is committed to the KV-cache pool, a C host program without a
device allocator): its workspace is a fixed scratch area inside the library.
This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must also pass on its own in a
fresh process.

Checked through the C ABI, twice in a row (the area keeps the previous call's
contents): the output matches pa_decode with a caller workspace, within the
decode tolerance, for a fused combine, the separate reduce kernel and a
single-partition shape; a shape whose scratch would not fit is refused.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_383_b200 import _lib
from paged_kv_cache_383_b200 import workloads as wl

from helpers import ATOL

pytestmark = pytest.mark.gpu


def _inputs(name, **scaled):
    w = wl.WORKLOADS[name].scaled(**scaled)
    inp = wl.make_paged(w, device="cuda")
    bt = torch.from_numpy(inp.block_tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    return w, inp, bt, cl


@pytest.mark.parametrize("name,scaled,ps,reduce", [
    ("llama3_70b_gqa8", dict(num_seqs=12, cap=3000), 512, "auto"),
    ("long_context_split", dict(num_seqs=2, low=9000, high=12000), 512,
     "kernel"),
    ("llama3_8b_gqa4", dict(num_seqs=6, low=100, high=900), 1024, "auto"),
])
def test_noalloc_matches_workspace_path(pkv, name, scaled, ps, reduce):
    w, inp, bt, cl = _inputs(name, **scaled)
    max_ctx = int(inp.lengths.max())
    want = torch.empty_like(inp.q)
    pkv.pa_decode(want, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                  w.softmax_scale, partition_size=ps, reduce=reduce,
                  max_context_len=max_ctx)
    desc = pkv.make_desc(inp.q, inp.k_cache, bt, partition_size=ps,
                         max_context_len=max_ctx, reduce=reduce)
    assert 0 < pkv.pa_decode_workspace_bytes(desc) or ps >= max_ctx
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        got = torch.full_like(inp.q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = lib.pa_decode_noalloc(
            got.data_ptr(), inp.q.data_ptr(), inp.k_cache.data_ptr(),
            inp.v_cache.data_ptr(), bt.data_ptr(), cl.data_ptr(),
            ctypes.c_float(w.softmax_scale), ctypes.byref(desc),
            err.data_ptr(), stream)
        assert st == _lib.PA_OK, lib.pa_last_error()
        torch.cuda.synchronize()
        assert err.item() == 0
        diff = (got.float() - want.float()).abs().max().item()
        assert diff <= ATOL, (call, diff)


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
