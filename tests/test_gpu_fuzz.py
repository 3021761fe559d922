"""GPU: seeded random shapes for pa_decode and pa_prefill against the fp64
oracle.

Each case draws its shape from a fixed seed: dtype, query group G, head_dim,
block size, batch, ragged context lengths (0 and 1 included, partly filled
last blocks), partition size and reduction (decode), new-token counts that
reach every prefill layout (a few rows per KV head, chunks, whole prompts)
and the precision of P.  Every output is compared with the oracle as the
other parity tests do: the float32 output with no carve-out, the dtype
output as its exact rounding (prefill) or within the tolerance (decode).
The result is the one of contiguous attention ([vLLM PagedAttention FAQ]
"Does PagedAttention change the mathematical attention output?").
"""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_decode, check_prefill, check_strict, prefill_both, to_np

pytestmark = pytest.mark.gpu

DTYPES = ("bfloat16", "float16")
GROUPS = (1, 2, 4, 8)


def _shape(rng, max_seqs, max_len):
    dtype = DTYPES[rng.integers(2)]
    g = int(GROUPS[rng.integers(4)])
    hkv = int(rng.choice((1, 2, 4, 8)))
    d = int(rng.choice((64, 128)))
    bs = int(rng.choice((16, 32)))
    n = int(rng.integers(1, max_seqs + 1))
    kind = rng.integers(3)
    if kind == 0:      # short, ragged, edge lengths
        lens = rng.choice([0, 1, 2, bs - 1, bs, bs + 1, 63, 64, 65, 127, 128,
                           129, 300], size=n)
    elif kind == 1:    # uniform
        lens = rng.integers(1, max_len + 1, size=n)
    else:              # one long, the rest short
        lens = rng.integers(1, 200, size=n)
        lens[rng.integers(n)] = max_len
    return dtype, g, hkv, d, bs, np.asarray(lens, dtype=np.int64)


@pytest.mark.parametrize("seed", range(32))
def test_decode_random_shapes(pkv, seed):
    rng = np.random.default_rng(1000 + seed)
    dtype, g, hkv, d, bs, lens = _shape(rng, 24, 3000)
    w = wl.Workload(f"fuzz_dec{seed}", 2000 + seed, len(lens), g * hkv, hkv,
                    d, bs, dtype, "fixed", fixed_lengths=tuple(lens))
    inp = wl.make_paged(w, device="cuda")
    ps = int(rng.choice((0, bs, 64, 128, 512, 1024)))
    kernel = ("auto", "simt", "mma")[int(rng.integers(3))]
    reduce = ("auto", "kernel")[int(rng.integers(2))]
    bt = torch.from_numpy(inp.block_tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    max_ctx = int(inp.lengths.max()) if len(lens) else 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(inp.q)
    out32 = torch.empty(inp.q.shape, dtype=torch.float32, device="cuda")
    for o in (out, out32):
        pkv.pa_decode(o, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                      w.softmax_scale, partition_size=ps, kernel=kernel,
                      reduce=reduce, max_context_len=max_ctx, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oa.paged_decode(to_np(inp.q), to_np(inp.k_cache),
                          to_np(inp.v_cache), inp.block_tables, inp.lengths,
                          w.softmax_scale)
    what = (f"seed {seed}: {dtype} G{g} Hkv{hkv} D{d} bs{bs} ps{ps} "
            f"{kernel}/{reduce} lens {lens.tolist()}")
    check_strict(to_np(out32), ref, what)
    check_decode(to_np(out), ref, inp.q.dtype, what)


# The oracle attends one (row, query head) at a time: each case is held to
# this many of them so the sweep stays within seconds per case.
ORACLE_ROWS = 60000


@pytest.mark.parametrize("seed", range(32))
def test_prefill_random_shapes(pkv, seed):
    rng = np.random.default_rng(3000 + seed)
    dtype, g, hkv, d, bs, lens = _shape(rng, 12, 1500)
    lens = np.maximum(lens, 1)
    hq = g * hkv
    mode = int(rng.integers(3))
    if mode == 0:      # a few new tokens: the few-row layouts
        q_lens = rng.integers(0, 64 // g + 1, size=len(lens))
    elif mode == 1:    # chunks
        q_lens = rng.integers(1, 300, size=len(lens))
    else:              # whole prompts
        q_lens = lens.copy()
    q_lens = np.minimum(q_lens, lens)
    while len(lens) > 1 and int(q_lens.sum()) * hq > ORACLE_ROWS:
        lens, q_lens = lens[:-1], q_lens[:-1]
    if int(q_lens.sum()) * hq > ORACLE_ROWS:
        q_lens = np.minimum(q_lens, ORACLE_ROWS // hq)
        if mode == 2:
            lens = q_lens.copy()
    pv = ("auto", "split", "single")[int(rng.integers(3))]
    w = wl.Workload(f"fuzz_pf{seed}", 4000 + seed, len(lens), g * hkv, hkv,
                    d, bs, dtype, "fixed", fixed_lengths=tuple(lens))
    pin = wl.make_prefill(w, q_lens, device="cuda")
    inp = pin.paged
    if pin.q.shape[0] == 0:
        return
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(pin.q)
    out32 = prefill_both(pkv, out, pin.q, inp.k_cache, inp.v_cache,
                         torch.from_numpy(inp.block_tables).cuda(),
                         torch.from_numpy(inp.lengths.astype(np.int32)).cuda(),
                         torch.from_numpy(pin.query_start).cuda(),
                         w.softmax_scale,
                         max_q_len=int(max(pin.q_lens.max(), 1)),
                         max_context_len=int(inp.lengths.max()), pv=pv,
                         dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oa.paged_prefill(to_np(pin.q), to_np(inp.k_cache),
                           to_np(inp.v_cache), inp.block_tables, inp.lengths,
                           pin.query_start, w.softmax_scale)
    what = (f"seed {seed}: {dtype} G{g} Hkv{hkv} D{d} bs{bs} pv {pv} "
            f"lens {lens.tolist()} q_lens {pin.q_lens.tolist()}")
    if pv == "single":
        # one rounding of P: held to its own bound (see the precision test)
        vmax = float(inp.v_cache.abs().amax())
        u = 2.0 ** -8 if dtype == "bfloat16" else 2.0 ** -11
        got = to_np(out32).astype(np.float64)
        assert np.isfinite(got).all(), what
        assert np.abs(got - ref).max() <= u * vmax + 1e-4, what
        assert torch.equal(out, out32.to(out.dtype)), what
    else:
        check_prefill(out, out32, ref, what)
