"""GPU: precision of P in the prefill's P . V, per pa_prefill_pv mode.

The tensor cores take 16-bit operands, so the softmax weights P are rounded
to the input dtype before P . V.  Each mode runs on the same inputs with a
float32 output (the kernel's value before the output rounding), against the
fp64 oracle ([vLLM PagedAttention FAQ] "Does PagedAttention change the
mathematical attention output?": the result is that of contiguous attention):

  auto    P's residual added only in the tiles where some row may end with a
          key of weight above 1/16: must meet the tolerance with no carve-out
          (every element within 2e-3, every |ref| >= 0.2 within 1e-2 rel);
  split   the residual in every tile: the same bound;
  single  one rounding of P: held to its own bound, u * max |v| + 1e-4 with
          u = 2^-8 (bf16) or 2^-11 (fp16), the most one relative rounding of
          every weight can move a weighted mean of the values.

Each case prints one "PRECISION" line (case, mode, max abs, max rel); run
with -s to collect the table.  Cases: short mixed contexts (a row's weight on
few keys), peaky attention (softmax scale 1, short contexts), and the bench's
full-size chunked prefill, whole prompts and 4-draft verification on sampled
rows.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import workloads as wl

from helpers import check_strict, to_np

pytestmark = pytest.mark.gpu

MODES = ("auto", "split", "single")
UNIT_ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def _seq_pool(inp, b, need):
    """Sequence b's first `need` blocks, copied to the host as a sub-pool
    (the oracle's result does not depend on block ids)."""
    ids = torch.from_numpy(inp.block_tables[b, :need].astype(np.int64))
    ids = ids.to(inp.k_cache.device)
    return (to_np(inp.k_cache.index_select(0, ids)),
            to_np(inp.v_cache.index_select(0, ids)))


def _rows_ref_decode(pin, picks):
    """Oracle rows for (sequence, local new-token indices) picks: row i of a
    sequence's n new tokens is a decode over its first L - n + i + 1
    tokens."""
    inp, w = pin.paged, pin.paged.workload
    rows, refs = [], []
    for b, local in picks:
        L, n = int(inp.lengths[b]), int(pin.q_lens[b])
        local = np.asarray(sorted(set(int(i) for i in local if 0 <= i < n)))
        pos = L - n + local
        need = int(pos.max()) // w.block_size + 1
        kc, vc = _seq_pool(inp, b, need)
        sub = np.repeat(np.arange(need, dtype=np.int32)[None, :], len(pos),
                        axis=0)
        r = pin.query_start[b] + local
        refs.append(oa.paged_decode(to_np(pin.q)[r], kc, vc, sub, pos + 1,
                                    w.softmax_scale))
        rows.append(r)
    return np.concatenate(rows), np.concatenate(refs)


def _mixed(dtype, scale=None):
    lens = (1, 3, 6, 17, 40, 130, 300, 520, 64, 700, 33, 257)
    qlens = (1, 3, 6, 17, 40, 130, 57, 1, 4, 200, 33, 40)
    w = wl.Workload("pv_mixed", 51, len(lens), 64, 8, 128, 16, dtype,
                    "fixed", fixed_lengths=lens, scale=scale)
    pin = wl.make_prefill(w, qlens, device="cuda")
    inp = pin.paged
    ref = oa.paged_prefill(to_np(pin.q), to_np(inp.k_cache),
                           to_np(inp.v_cache), inp.block_tables, inp.lengths,
                           pin.query_start, w.softmax_scale)
    return pin, np.arange(pin.q.shape[0]), ref


def _chunked():
    w = wl.WORKLOADS["chunked_prefill_gqa8"]
    pin = wl.make_prefill(w, np.full(w.num_seqs, 512), device="cuda")
    rng = np.random.default_rng(1)
    picks = [(b, [0, 1, 63, 64, 255, 511, *rng.integers(0, 512, 10)])
             for b in (0, 7, 15)]
    return (pin, *_rows_ref_decode(pin, picks))


def _prompts():
    w = wl.WORKLOADS["prompt_prefill_gqa8"]
    lens = wl.make_paged(w, values=False).lengths
    pin = wl.make_prefill(w, lens, device="cuda")
    rng = np.random.default_rng(2)
    picks = []
    for b in (0, int(np.argmax(lens)), w.num_seqs - 1):
        L = int(lens[b])
        picks.append((b, [*range(0, 40), 63, 64, 127, 128, 255, 256, 1000,
                          L - 1, *rng.integers(0, L, 12)]))
    return (pin, *_rows_ref_decode(pin, picks))


def _verify4():
    w = wl.WORKLOADS["llama3_70b_gqa8"]
    pin = wl.make_prefill(w, np.full(w.num_seqs, 4), device="cuda")
    lens = pin.paged.lengths
    seqs = (0, int(np.argmax(lens)), int(np.argmin(lens)), 100, 200, 255)
    return (pin, *_rows_ref_decode(pin, [(b, range(4)) for b in seqs]))


CASES = {
    "mixed_short_bf16": lambda: _mixed("bfloat16"),
    "mixed_short_f16": lambda: _mixed("float16"),
    "peaky_scale1_bf16": lambda: _mixed("bfloat16", scale=1.0),
    "peaky_scale1_f16": lambda: _mixed("float16", scale=1.0),
    "chunked_prefill_gqa8": _chunked,
    "prompt_prefill_gqa8": _prompts,
    "verify_4_drafts_llama3_70b_gqa8": _verify4,
}


@functools.lru_cache(maxsize=1)
def _case(name):
    # one case's inputs and oracle rows at a time (the full-size pools are
    # large); parametrisation order keeps a case's three modes together
    return CASES[name]()


# the top decorator varies fastest: a case's three modes run together
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(CASES))
def test_pv_precision(pkv, name, mode):
    pin, rows, ref = _case(name)
    inp = pin.paged
    out32 = torch.full(pin.q.shape, float("nan"), dtype=torch.float32,
                       device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_prefill(out32, pin.q, inp.k_cache, inp.v_cache,
                   torch.from_numpy(inp.block_tables).cuda(),
                   torch.from_numpy(inp.lengths.astype(np.int32)).cuda(),
                   torch.from_numpy(pin.query_start).cuda(),
                   inp.workload.softmax_scale,
                   max_q_len=int(max(pin.q_lens.max(), 1)),
                   max_context_len=int(inp.lengths.max()), pv=mode,
                   dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = to_np(out32)[rows].astype(np.float64)
    d = np.abs(got - ref)
    big = np.abs(ref) >= 0.2
    max_abs = float(d.max())
    max_rel = float((d[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    print(f"PRECISION {name} {mode} max_abs={max_abs:.3e} "
          f"max_rel={max_rel:.3e} rows={len(rows)}")
    if mode == "single":
        vmax = float(inp.v_cache.abs().amax())
        bound = UNIT_ROUNDOFF[pin.q.dtype] * vmax + 1e-4
        assert np.isfinite(got).all()
        assert max_abs <= bound, (name, max_abs, bound)
    else:
        check_strict(got, ref, f"{name} pv={mode}")
