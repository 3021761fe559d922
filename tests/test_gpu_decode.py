"""GPU parity of pa_decode against the fp64 oracle (through the C ABI).

* every workload shape at oracle-sized scale (several pages, partitions and
  ragged tails), both compute variants;
* every workload at its full size, in the launch configuration the bench
  times, checked on sampled sequences;
* invariances: partition size, identity vs shuffled block tables;
* edge cases: empty batch, empty and one-token sequences, full tables, group
  sizes 1..8, head_dim 64/128, both dtypes;
* NaN in slots no sequence wrote does not reach the output;
* device-side index checks set the error word instead of faulting.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import workloads as wl

from helpers import (check_decode, oracle_paged_sample, poison_unwritten,
                     sample_seqs, to_np)

pytestmark = pytest.mark.gpu


def _run(pkv, inp, kernel="auto", partition_size=None, tables=None,
         lens=None, dev_err=None, reduce="auto"):
    w = inp.workload
    dev = inp.q.device
    bt = torch.from_numpy(inp.block_tables if tables is None else tables)
    bt = bt.to(dev)
    cl = torch.from_numpy(
        (inp.lengths if lens is None else lens).astype(np.int32)).to(dev)
    out = torch.empty_like(inp.q)
    ps = w.partition_size if partition_size is None else partition_size
    pkv.pa_decode(out, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                  w.softmax_scale, partition_size=ps, kernel=kernel,
                  reduce=reduce,
                  max_context_len=int(inp.lengths.max()) if len(inp.lengths)
                  else 0, dev_err=dev_err)
    torch.cuda.synchronize()
    return out


def _check_all(inp, out, what):
    w = inp.workload
    ref = oa.paged_decode(to_np(inp.q), to_np(inp.k_cache),
                          to_np(inp.v_cache), inp.block_tables, inp.lengths,
                          w.softmax_scale)
    return check_decode(to_np(out), ref, inp.q.dtype, what)


SMALL = {
    "tiny_mha_d64": dict(),
    "llama3_8b_gqa4": dict(num_seqs=6, low=20, high=700),
    "llama3_70b_gqa8": dict(num_seqs=8, cap=1500),
    "llama3_70b_gqa8_bs32": dict(num_seqs=8, cap=1500),
    "long_context_split": dict(num_seqs=3, low=1500, high=4000),
}


@pytest.mark.parametrize("kernel", ["mma", "simt"])
@pytest.mark.parametrize("name", list(SMALL))
def test_small_workloads(pkv, name, kernel):
    w = wl.WORKLOADS[name].scaled(**SMALL[name])
    inp = wl.make_paged(w, device="cuda")
    out = _run(pkv, inp, kernel=kernel)
    _check_all(inp, out, f"{name}/{kernel}")


@pytest.mark.parametrize("name", ["tiny_mha_d64", "llama3_8b_gqa4",
                                  "llama3_70b_gqa8", "llama3_70b_gqa8_bs32",
                                  "long_context_split"])
def test_full_size_sampled(pkv, name):
    """Full-size inputs, same launch as the bench; oracle on sampled seqs."""
    w = wl.WORKLOADS[name]
    inp = wl.make_paged(w, device="cuda")
    out = _run(pkv, inp)
    seqs = sample_seqs(inp.lengths, k=3 if name == "long_context_split" else 6)
    ref = oracle_paged_sample(inp.q, inp.k_cache, inp.v_cache,
                              inp.block_tables, inp.lengths, w.softmax_scale,
                              seqs)
    for b in seqs:
        check_decode(to_np(out[b]), ref[b], inp.q.dtype, f"{name} seq {b}")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("reduce", ["auto", "kernel"])
def test_partition_size_invariance(pkv, reduce):
    # 16-token partitions give up to 125 partitions per sequence (separate
    # reduce kernel even in auto mode); 256 gives <= 8 (fused in auto mode).
    w = wl.WORKLOADS["llama3_70b_gqa8"].scaled(num_seqs=6, cap=2000)
    inp = wl.make_paged(w, device="cuda")
    outs = {ps: _run(pkv, inp, partition_size=ps, reduce=reduce)
            for ps in (16, 64, 256, 512, 0)}
    for ps, out in outs.items():
        _check_all(inp, out, f"partition {ps} / {reduce}")
    a, b = outs[16].float(), outs[512].float()
    assert (a - b).abs().max().item() <= 4e-3


def test_fused_and_kernel_reduce_agree(pkv):
    w = wl.WORKLOADS["long_context_split"].scaled(num_seqs=3, low=1500,
                                                  high=4000)
    inp = wl.make_paged(w, device="cuda")
    fused = _run(pkv, inp, partition_size=512, reduce="auto")   # <= 8 parts
    kern = _run(pkv, inp, partition_size=512, reduce="kernel")
    _check_all(inp, fused, "fused")
    _check_all(inp, kern, "kernel")
    assert (fused.float() - kern.float()).abs().max().item() <= 2e-3


UNIT_GRID = {
    "gqa4_bf16_bs16": wl.Workload("unit_gqa4", 77, 20, 32, 8, 128, 16,
                                  "bfloat16", "uniform", low=1, high=6000),
    "mha_d64_f16_bs32": wl.Workload("unit_mha", 78, 20, 8, 8, 64, 32,
                                    "float16", "uniform", low=1, high=6000),
}


@pytest.mark.parametrize("kernel", ["mma", "simt"])
@pytest.mark.parametrize("name", list(UNIT_GRID))
def test_unit_ordered_grid(pkv, name, kernel):
    """1024-token partitions in a grid of under four waves: the decode runs
    one CTA per (KV head, partition unit), units longest first; ragged
    lengths from one token to six partitions, empty units included."""
    inp = wl.make_paged(UNIT_GRID[name], device="cuda")
    out = _run(pkv, inp, kernel=kernel, partition_size=1024)
    _check_all(inp, out, f"unit grid {name}/{kernel}")


def test_identity_vs_shuffled_tables(pkv):
    w = wl.WORKLOADS["llama3_8b_gqa4"].scaled(num_seqs=5, low=100, high=900)
    inp = wl.make_paged(w, device="cuda")
    out_shuf = _run(pkv, inp)
    # Move every sequence's blocks to consecutive physical ids 0, 1, 2, ...
    nblk = wl.blocks_needed(inp.lengths, w.block_size)
    ident = np.full_like(inp.block_tables, -1)
    kc = inp.k_cache.clone()
    vc = inp.v_cache.clone()
    nxt = 0
    for b in range(w.num_seqs):
        src = torch.from_numpy(inp.block_tables[b, :nblk[b]].astype(np.int64))
        dst = torch.arange(nxt, nxt + nblk[b])
        kc[dst.cuda()] = inp.k_cache[src.cuda()]
        vc[dst.cuda()] = inp.v_cache[src.cuda()]
        ident[b, :nblk[b]] = dst.numpy()
        nxt += nblk[b]
    inp2 = wl.PagedInputs(w, inp.lengths, ident, inp.num_blocks, inp.q, kc, vc)
    out_id = _run(pkv, inp2)
    assert torch.equal(out_shuf, out_id)


@pytest.mark.parametrize("dtype", ["float16", "bfloat16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (12, 4), (16, 4),
                                    (32, 4)])
@pytest.mark.parametrize("bs", [16, 32])
def test_shapes(pkv, dtype, head_dim, hq, hkv, bs):
    w = wl.Workload("shape", 7, 5, hq, hkv, head_dim, bs, dtype, "fixed",
                    fixed_lengths=(1, bs, bs + 1, 3 * bs - 1, 200))
    inp = wl.make_paged(w, device="cuda")
    for kernel in ("mma", "simt"):
        out = _run(pkv, inp, kernel=kernel, partition_size=2 * bs)
        _check_all(inp, out, f"{dtype}/{head_dim}/{hq}:{hkv}/bs{bs}/{kernel}")


def test_edge_lengths(pkv):
    # zero-length sequence -> zeros; one token -> that token's V exactly;
    # a sequence filling its whole table.
    w = wl.Workload("edges", 9, 4, 8, 2, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(0, 1, 64, 17))
    inp = wl.make_paged(w, device="cuda")
    tables = inp.block_tables.copy()
    for kernel in ("mma", "simt"):
        for ps in (0, 16):
            out = _run(pkv, inp, kernel=kernel, partition_size=ps,
                       tables=tables)
            assert torch.count_nonzero(out[0]) == 0
            v0 = inp.v_cache[int(tables[1, 0]), :, 0, :]          # [Hkv, D]
            assert torch.equal(out[1], v0.repeat_interleave(4, dim=0))
            _check_all(inp, out, f"edges/{kernel}/{ps}")


def test_empty_batch_is_noop(pkv):
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(0, 2, dtype=torch.int32, device="cuda")
    cl = torch.zeros(0, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pkv.pa_decode(out, q, kc, kc, bt, cl, 0.1)


def test_device_checks_flag_bad_inputs(pkv):
    w = wl.Workload("bad", 3, 3, 8, 2, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(40, 40, 40))
    inp = wl.make_paged(w, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = inp.block_tables.copy()
    tables[1, 1] = inp.num_blocks + 5             # block outside the pool
    out = _run(pkv, inp, tables=tables, dev_err=err)
    assert err.item() == 5                        # PA_ERR_DEVICE_OOB
    ref = oa.paged_decode(to_np(inp.q), to_np(inp.k_cache),
                          to_np(inp.v_cache), inp.block_tables, inp.lengths,
                          w.softmax_scale)
    for b in (0, 2):                              # other sequences intact
        check_decode(to_np(out[b]), ref[b], inp.q.dtype, f"seq {b}")
    err.zero_()
    lens = inp.lengths.copy()
    lens[2] = 10_000                              # beyond the table
    _run(pkv, inp, lens=lens, dev_err=err)
    assert err.item() == 5
    for reduce in ("auto", "kernel"):   # split sequences, both combines
        err.zero_()
        tables = inp.block_tables.copy()
        tables[0, 0] = -3
        out = _run(pkv, inp, tables=tables, dev_err=err, partition_size=16,
                   reduce=reduce)
        assert err.item() == 5
        for b in (1, 2):
            check_decode(to_np(out[b]), ref[b], inp.q.dtype,
                         f"split seq {b} / {reduce}")


@pytest.mark.parametrize("kernel", ["mma", "simt"])
@pytest.mark.parametrize("bs", [16, 32])
def test_unwritten_slots_hold_nan(pkv, kernel, bs):
    w = wl.Workload("nan_tail", 21, 6, 32, 8, 128, bs, "bfloat16", "fixed",
                    fixed_lengths=(1, 15, 17, 100, 333, 1000))
    inp = wl.make_paged(w, device="cuda")
    ref = oa.paged_decode(to_np(inp.q), to_np(inp.k_cache),
                          to_np(inp.v_cache), inp.block_tables, inp.lengths,
                          w.softmax_scale)
    poison_unwritten(inp)
    for ps in (0, 64):
        out = _run(pkv, inp, kernel=kernel, partition_size=ps)
        check_decode(to_np(out), ref, inp.q.dtype, f"{kernel} ps={ps}")


@pytest.mark.parametrize("ps", [16, 32, 64])
def test_warp_partitions_ragged_groups(pkv, ps):
    # Reduce-kernel path with short partitions: a CTA serves four
    # partitions, one per consumer warp.  Lengths leave groups of 1-4
    # partitions, partial last pages and partitions, an empty sequence and
    # a one-token sequence.
    lens = (0, 1, 16, 17, 48, 63, 64, 65, 100, 129, 200, 255)
    w = wl.Workload("warp_parts", 41, len(lens), 32, 8, 128, 16, "bfloat16",
                    "fixed", fixed_lengths=lens)
    inp = wl.make_paged(w, device="cuda")
    out = _run(pkv, inp, partition_size=ps, reduce="kernel")
    assert torch.count_nonzero(out[0]) == 0
    v0 = inp.v_cache[int(inp.block_tables[1, 0]), :, 0, :]
    assert torch.equal(out[1], v0.repeat_interleave(4, dim=0))
    _check_all(inp, out, f"warp partitions ps={ps}")
    ref = _run(pkv, inp, partition_size=256, reduce="auto")
    assert (out.float() - ref.float()).abs().max().item() <= 4e-3

