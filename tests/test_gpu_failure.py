"""Failure path of the kernels' bounded waits, without a real fault.

pa_wait_probe runs one warp that holds tensor memory and waits on an
mbarrier nothing arrives at (a flag that nothing sets).  The wait gives up
after its limit, the error word reads PA_ERR_DEVICE_TIMEOUT, and the
context stays usable: a prefill (which allocates tensor memory again) and a
decode still match the oracle afterwards."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import _lib
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_decode, check_prefill, prefill_both, to_np

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_the_context_survives(pkv):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    pkv.pa_wait_probe(err)
    b.record()
    torch.cuda.synchronize()
    assert err.item() == _lib.PA_ERR_DEVICE_TIMEOUT
    assert 900.0 <= a.elapsed_time(b) <= 10_000.0   # the 1 s limit

    w = wl.WORKLOADS["llama3_70b_gqa8"].scaled(num_seqs=4, cap=700)
    lens = wl.make_paged(w, values=False).lengths
    pin = wl.make_prefill(w, np.minimum(lens, (5, 40, 1, 17)), device="cuda")
    inp = pin.paged
    bt = torch.from_numpy(inp.block_tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    qs = torch.from_numpy(pin.query_start).cuda()
    err.zero_()
    out = torch.empty_like(pin.q)
    out32 = prefill_both(pkv, out, pin.q, inp.k_cache, inp.v_cache, bt, cl,
                         qs, w.softmax_scale, max_q_len=int(pin.q_lens.max()),
                         max_context_len=int(inp.lengths.max()), dev_err=err)
    dq = torch.randn(4, w.num_q_heads, w.head_dim,
                     device="cuda").to(pin.q.dtype)
    dout = torch.empty_like(dq)
    pkv.pa_decode(dout, dq, inp.k_cache, inp.v_cache, bt, cl,
                  w.softmax_scale, max_context_len=int(inp.lengths.max()),
                  dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    kc, vc = to_np(inp.k_cache), to_np(inp.v_cache)
    ref = oa.paged_prefill(to_np(pin.q), kc, vc, inp.block_tables,
                           inp.lengths, pin.query_start, w.softmax_scale)
    check_prefill(out, out32, ref, "prefill after the timeout")
    ref = oa.paged_decode(to_np(dq), kc, vc, inp.block_tables, inp.lengths,
                          w.softmax_scale)
    check_decode(to_np(dout), ref, dq.dtype, "decode after the timeout")
