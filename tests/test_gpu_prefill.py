"""GPU parity of pa_prefill (causal attention of new tokens over the paged
cache, tcgen05 tensor cores) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import workloads as wl

from helpers import (check_decode, check_prefill, poison_unwritten,
                     prefill_both, to_np)

pytestmark = pytest.mark.gpu


def _run(pkv, pin, tables=None, err=None, kernel="auto"):
    """pa_prefill into a dtype output and a float32 one (the value before
    the output rounding); returns (out, out32)."""
    inp = pin.paged
    w = inp.workload
    out = torch.full_like(pin.q, float("nan"))
    bt = torch.from_numpy(inp.block_tables if tables is None
                          else tables).cuda()
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).cuda()
    qs = torch.from_numpy(pin.query_start).cuda()
    out32 = prefill_both(pkv, out, pin.q, inp.k_cache, inp.v_cache, bt, cl,
                         qs, w.softmax_scale,
                         max_q_len=int(max(pin.q_lens.max(), 1)),
                         max_context_len=int(inp.lengths.max()), dev_err=err,
                         kernel=kernel)
    torch.cuda.synchronize()
    return out, out32


def _check(pin, outs, what, seqs=None):
    inp = pin.paged
    ref = oa.paged_prefill(to_np(pin.q), to_np(inp.k_cache),
                           to_np(inp.v_cache), inp.block_tables, inp.lengths,
                           pin.query_start, inp.workload.softmax_scale,
                           seqs=seqs)
    rows = np.concatenate([np.arange(pin.query_start[b],
                                     pin.query_start[b + 1])
                           for b in (seqs if seqs is not None
                                     else range(len(pin.q_lens)))])
    return check_prefill(*outs, ref[rows], what, rows=rows)


@pytest.mark.parametrize("dtype", ["bfloat16", "float16"])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8)])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_mixed_chunks(pkv, dtype, hq, hkv, bs, head_dim):
    # whole prompts, chunks, single tokens and a few speculative tokens
    lens = (1, 17, 130, 300, 520, 64, 700, 33)
    qlens = (1, 17, 130, 57, 1, 4, 200, 33)
    w = wl.Workload("prefill", 11, len(lens), hq, hkv, head_dim, bs, dtype,
                    "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, qlens, device="cuda")
    out = _run(pkv, pin)
    _check(pin, out, f"{dtype}/{hq}:{hkv}/bs{bs}/d{head_dim}")


def test_single_token_matches_decode(pkv):
    w = wl.WORKLOADS["llama3_70b_gqa8"].scaled(num_seqs=8, cap=2000)
    pin = wl.make_prefill(w, np.ones(8), device="cuda")
    out = _run(pkv, pin)
    inp = pin.paged
    dec = torch.empty_like(pin.q)
    pkv.pa_decode(dec, pin.q, inp.k_cache, inp.v_cache,
                  torch.from_numpy(inp.block_tables).cuda(),
                  torch.from_numpy(inp.lengths.astype(np.int32)).cuda(),
                  w.softmax_scale, max_context_len=int(inp.lengths.max()))
    torch.cuda.synchronize()
    _check(pin, out, "prefill q_len=1")
    assert (out[0].float() - dec.float()).abs().max().item() <= 4e-3


def test_sequences_without_new_tokens(pkv):
    w = wl.Workload("prefill0", 12, 3, 32, 8, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(100, 50, 80))
    pin = wl.make_prefill(w, (0, 50, 0), device="cuda")
    out = _run(pkv, pin)
    _check(pin, out, "middle sequence only")
    assert out[0].shape[0] == 50


def test_chunked_prefill_full_size_sampled(pkv):
    w = wl.WORKLOADS["chunked_prefill_gqa8"]
    pin = wl.make_prefill(w, np.full(w.num_seqs, 512), device="cuda")
    out = _run(pkv, pin)
    _check(pin, out, "chunked prefill", seqs=[0, 7, 15])
    assert torch.isfinite(out[0].float()).all()


def test_bad_block_id_is_flagged(pkv):
    w = wl.Workload("prefillbad", 13, 3, 16, 8, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(90, 90, 90))
    pin = wl.make_prefill(w, (30, 30, 30), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = pin.paged.block_tables.copy()
    tables[1, 2] = pin.paged.num_blocks + 3
    out = _run(pkv, pin, tables=tables, err=err)
    assert err.item() == 5
    _check(pin, out, "other sequences intact", seqs=[0, 2])


@pytest.mark.parametrize("q_lens", [(30, 30, 30), (2, 2, 2)])
def test_bad_context_length_is_skipped_and_flagged(pkv, q_lens):
    """A sequence whose context length runs past its block table is flagged
    (PA_ERR_DEVICE_OOB) and its work items are skipped by every warp of the
    persistent grid; the other sequences' rows are still exact (tile and
    few-row layouts)."""
    w = wl.Workload("prefillbadlen", 17, 3, 16, 8, 128, 16, "bfloat16",
                    "fixed", fixed_lengths=(90, 90, 90))
    pin = wl.make_prefill(w, q_lens, device="cuda")
    inp = pin.paged
    lens = inp.lengths.astype(np.int32).copy()
    lens[1] = inp.block_tables.shape[1] * w.block_size + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full_like(pin.q, float("nan"))
    out32 = prefill_both(pkv, out, pin.q, inp.k_cache, inp.v_cache,
                         torch.from_numpy(inp.block_tables).cuda(),
                         torch.from_numpy(lens).cuda(),
                         torch.from_numpy(pin.query_start).cuda(),
                         w.softmax_scale, max_q_len=max(q_lens),
                         max_context_len=int(lens.max()), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    _check(pin, (out, out32), "other sequences intact", seqs=[0, 2])


def test_overlapping_rows_overflow_the_tile_map_and_are_flagged(pkv):
    """Sequences 0 and 2 both given query rows [0, 64) (each range valid on
    its own; sequence 1's runs backwards, 64 -> 0, and is flagged) list 8
    tiles of 16 tokens where the map holds min(64 / 16 + 3, 3 * 4) = 7: the
    plan kernel cuts the map at its capacity and flags PA_ERR_DEVICE_OOB;
    the call writes only rows of out and ends without a timeout."""
    w = wl.Workload("overlap", 19, 3, 64, 8, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(200, 200, 200))
    pin = wl.make_prefill(w, (64, 0, 0), device="cuda")
    inp = pin.paged
    q = pin.q[:64].contiguous()
    qs = torch.tensor([0, 64, 0, 64], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    pkv.pa_prefill(out, q, inp.k_cache, inp.v_cache,
                   torch.from_numpy(inp.block_tables).cuda(),
                   torch.from_numpy(inp.lengths.astype(np.int32)).cuda(), qs,
                   w.softmax_scale, max_q_len=64, max_context_len=200,
                   dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("q_lens,max_q", [((40, 10, 90), 40), ((3, 8, 2), 4)])
def test_sequence_above_max_q_len_is_flagged(pkv, q_lens, max_q):
    """A sequence with more new tokens than max_q_len gets no query tiles
    and sets PA_ERR_DEVICE_OOB; the other sequences' rows are still computed
    (the tile layout, and with max_q_len 4 the few-row layout)."""
    w = wl.Workload("over_max_q", 91, 3, 16, 4, 128, 16, "bfloat16", "fixed",
                    fixed_lengths=(300, 200, 90))
    pin = wl.make_prefill(w, q_lens, device="cuda")
    inp = pin.paged
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full_like(pin.q, float("nan"))
    out32 = prefill_both(pkv, out, pin.q, inp.k_cache, inp.v_cache,
                         torch.from_numpy(inp.block_tables).cuda(),
                         torch.from_numpy(inp.lengths.astype(np.int32)).cuda(),
                         torch.from_numpy(pin.query_start).cuda(),
                         w.softmax_scale, max_q_len=max_q,
                         max_context_len=int(inp.lengths.max()), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    ok = [b for b in range(3) if pin.q_lens[b] <= max_q]
    _check(pin, (out, out32), "sequences within max_q_len", seqs=ok)


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_unwritten_slots_hold_nan(pkv, bs, head_dim):
    lens = (1, 15, 17, 100, 333, 1000)
    w = wl.Workload("prefill_nan", 14, len(lens), 32, 8, head_dim, bs,
                    "bfloat16", "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, (1, 15, 5, 100, 40, 300), device="cuda")
    _check(pin, _run(pkv, pin), "clean pool")
    poison_unwritten(pin.paged)
    _check(pin, _run(pkv, pin), "poisoned pool")


def _contiguous_pool(K_seqs, V_seqs, bs):
    """Host pool holding each sequence's K/V in consecutive blocks, and the
    identity tables that reach them (built from inputs only)."""
    nblk = [(len(k) + bs - 1) // bs for k in K_seqs]
    hkv, d = K_seqs[0].shape[1:]
    kp = np.zeros((sum(nblk), hkv, bs, d))
    vp = np.zeros_like(kp)
    tables = np.full((len(K_seqs), max(nblk)), -1, dtype=np.int32)
    base = 0
    for b, (k, v) in enumerate(zip(K_seqs, V_seqs)):
        for t in range(len(k)):
            kp[base + t // bs, :, t % bs] = k[t]
            vp[base + t // bs, :, t % bs] = v[t]
        tables[b, :nblk[b]] = np.arange(base, base + nblk[b])
        base += nblk[b]
    return kp, vp, tables


def test_speculative_verify_and_rollback(pkv):
    """Prompt prefill -> 4 draft tokens verified in one pass -> rejected
    drafts rolled back with truncate -> next token written over the freed
    slots and decoded; every step against the oracle on input K/V."""
    from paged_kv_cache_383_b200 import flow
    hq, hkv, d, bs, draft = 32, 8, 128, 16, 4
    prompts, accept = [37, 64, 100, 5], [0, 1, 3, 4]
    B = len(prompts)
    g = torch.Generator(device="cuda")
    g.manual_seed(383007)
    rnd = lambda *s: torch.randn(*s, generator=g, device="cuda").to(
        torch.bfloat16)
    kc, vc = rnd(64, hkv, bs, d), rnd(64, hkv, bs, d)
    bm = pkv.BlockManager(64, bs)
    ids = list(range(B))
    for s in ids:
        bm.add_seq(s)
    K = [np.zeros((0, hkv, d)) for _ in ids]
    V = [np.zeros((0, hkv, d)) for _ in ids]
    scale = d ** -0.5

    def step(n_new):
        """Write n_new[b] tokens, attend their queries causally, check."""
        kn, vn = rnd(sum(n_new), hkv, d), rnd(sum(n_new), hkv, d)
        q = rnd(sum(n_new), hq, d)
        flow.write_tokens(bm, kc, vc, ids, n_new, kn, vn)
        qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
        for b in ids:
            K[b] = np.concatenate([K[b], to_np(kn[qs[b]:qs[b + 1]])])
            V[b] = np.concatenate([V[b], to_np(vn[qs[b]:qs[b + 1]])])
        bt, cl, lens = flow.tables_on_device(bm, ids, 16, "cuda")
        assert list(lens) == [len(k) for k in K]
        out = torch.empty_like(q)
        out32 = prefill_both(pkv, out, q, kc, vc, bt, cl,
                             torch.from_numpy(qs).cuda(), scale,
                             max_q_len=max(n_new),
                             max_context_len=int(lens.max()))
        kp, vp, tables = _contiguous_pool(K, V, bs)
        ref = oa.paged_prefill(to_np(q), kp, vp, tables, lens, qs, scale)
        torch.cuda.synchronize()
        check_prefill(out, out32, ref, f"step {n_new}")
        return q, bt, cl, lens, out

    step(prompts)                      # whole prompts
    step([draft] * B)                  # verify the drafts in one pass
    for b in ids:                      # keep the accepted drafts only
        keep = prompts[b] + accept[b]
        bm.truncate(b, keep)
        K[b], V[b] = K[b][:keep], V[b][:keep]
    q, bt, cl, lens, out = step([1] * B)   # next token over freed slots
    dec = torch.empty_like(q)
    pkv.pa_decode(dec, q, kc, vc, bt, cl, scale,
                  max_context_len=int(lens.max()))
    torch.cuda.synchronize()
    kp, vp, tables = _contiguous_pool(K, V, bs)
    check_decode(to_np(dec), oa.paged_decode(to_np(q), kp, vp, tables, lens,
                                             scale), q.dtype, "decode")


def test_prompt_prefill_full_size_sampled(pkv):
    """Whole prompts at the bench's full size (8 sequences, 1k-8k tokens,
    every token new).  Row p of a prompt attends to positions 0..p, i.e. a
    decode over the first p + 1 tokens, which the oracle computes for
    sampled rows: first and last tokens, tile boundaries, random ones."""
    w = wl.WORKLOADS["prompt_prefill_gqa8"]
    lens = wl.make_paged(w, values=False).lengths
    pin = wl.make_prefill(w, lens, device="cuda")
    out = _run(pkv, pin)
    inp = pin.paged
    rng = np.random.default_rng(7)
    kc, vc = to_np(inp.k_cache), to_np(inp.v_cache)
    for b in (0, int(np.argmax(lens)), w.num_seqs - 1):
        L = int(lens[b])
        pos = sorted({0, 1, 15, 16, 63, 64, 127, 128, L - 2, L - 1,
                      *rng.integers(0, L, size=6).tolist()})
        rows = pin.query_start[b] + np.array(pos)
        q = to_np(pin.q)[rows]
        tables = np.repeat(inp.block_tables[b:b + 1], len(pos), axis=0)
        ref = oa.paged_decode(q, kc, vc, tables, np.array(pos) + 1,
                              w.softmax_scale)
        check_prefill(*out, ref, f"prompt seq {b}", rows=rows)


def test_long_context_chunk_sampled(pkv):
    """Chunks at the end of 90k- and 70k-token contexts (block 16): the
    producer reads block ids from global memory, so shared memory does not
    grow with the context.  Sampled rows against the oracle (row i of a
    chunk of n is a decode over the first L - n + i + 1 tokens)."""
    w = wl.Workload("long_prefill", 15, 2, 32, 8, 128, 16, "bfloat16",
                    "fixed", fixed_lengths=(90_000, 70_001))
    pin = wl.make_prefill(w, (256, 200), device="cuda")
    out = _run(pkv, pin)
    inp = pin.paged
    bs = w.block_size
    for b in (0, 1):
        L, n = int(inp.lengths[b]), int(pin.q_lens[b])
        local = np.array([0, 1, 63, 64, 127, n - 1])
        rows = pin.query_start[b] + local
        pos = L - n + local
        # the sequence's own blocks, copied to the host as a sub-pool
        need = int(pos.max()) // bs + 1
        ids = torch.from_numpy(
            inp.block_tables[b, :need].astype(np.int64)).cuda()
        kc = to_np(inp.k_cache.index_select(0, ids))
        vc = to_np(inp.v_cache.index_select(0, ids))
        sub = np.repeat(np.arange(need, dtype=np.int32)[None, :], len(pos),
                        axis=0)
        ref = oa.paged_decode(to_np(pin.q)[rows], kc, vc, sub, pos + 1,
                              w.softmax_scale)
        check_prefill(*out, ref, f"long seq {b}", rows=rows)


def test_more_sequences_than_order_threads(pkv):
    """1300 sequences (more than the one-CTA longest-first sort has threads),
    uniform 1..200-token contexts, 0..5 new tokens each: the grid rows follow
    the sort's order, so every sequence must still land in its own rows.
    Sampled sequences against the oracle, and no row left unwritten."""
    w = wl.Workload("many_seqs", 31, 1300, 16, 2, 64, 16, "bfloat16",
                    "uniform", low=1, high=200)
    lens = wl.make_paged(w, values=False).lengths
    q_lens = np.minimum(lens, np.random.default_rng(3).integers(0, 6, 1300))
    pin = wl.make_prefill(w, q_lens, device="cuda")
    out = _run(pkv, pin)
    assert not torch.isnan(out[0]).any()
    rng = np.random.default_rng(4)
    seqs = sorted({0, 1, 1023, 1024, 1299, int(np.argmax(lens)),
                   int(np.argmin(lens)), *rng.integers(0, 1300, 25).tolist()})
    seqs = [b for b in seqs if q_lens[b] > 0]
    _check(pin, out, "1300 sequences", seqs=seqs)


@pytest.mark.parametrize("dtype", ["bfloat16", "float16"])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8)])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_few_rows_up_to_32(pkv, dtype, hq, hkv, bs, head_dim):
    """At most 32 query rows per KV head (0 .. 32/G new tokens: the tile
    kernel's 8-rows-per-warp layout), contexts around the 64-key tile and
    128-key edges."""
    qmax = 32 // (hq // hkv)
    lens = (1, 17, 130, 300, 520, 64, 700, 33, 129, 128, 255, 256)
    want = (1, qmax, 2, qmax, 1, 3, qmax, 0, qmax, 1, 2, qmax)
    qlens = tuple(min(L, q) for L, q in zip(lens, want))
    w = wl.Workload("prefill_rows32", 21, len(lens), hq, hkv, head_dim, bs,
                    dtype, "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, qlens, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(pkv, pin, err=err)
    assert err.item() == 0
    _check(pin, out, f"rows<=32 {dtype}/{hq}:{hkv}/bs{bs}/d{head_dim}")


@pytest.mark.parametrize("bs", [16, 32])
def test_few_rows_unwritten_slots_hold_nan(pkv, bs):
    lens = (1, 15, 17, 100, 333, 1000, 128, 129)
    w = wl.Workload("rows32_nan", 22, len(lens), 32, 8, 128, bs, "bfloat16",
                    "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, (1, 8, 5, 8, 3, 8, 8, 2), device="cuda")
    _check(pin, _run(pkv, pin), "clean pool")
    poison_unwritten(pin.paged)
    _check(pin, _run(pkv, pin), "poisoned pool")


def test_few_rows_many_sequences(pkv):
    """1300 sequences x 2 KV heads, 0 .. 4 new tokens each (G = 8: up to 32
    rows per KV head)."""
    w = wl.Workload("many_rows32", 33, 1300, 16, 2, 128, 16, "bfloat16",
                    "uniform", low=1, high=400)
    lens = wl.make_paged(w, values=False).lengths
    q_lens = np.minimum(lens, np.random.default_rng(5).integers(0, 5, 1300))
    pin = wl.make_prefill(w, q_lens, device="cuda")
    out = _run(pkv, pin)
    assert not torch.isnan(out[0]).any()
    rng = np.random.default_rng(6)
    seqs = sorted({0, 1, 147, 148, 1299, int(np.argmax(lens)),
                   *rng.integers(0, 1300, 30).tolist()})
    _check(pin, out, "rows<=32, 1300 sequences",
           seqs=[b for b in seqs if q_lens[b] > 0])


def test_speculative_verify_full_size_sampled(pkv):
    """4 draft tokens for each of the 256 sequences of the batch-256 decode
    mix (the bench's verification workload); sampled sequences against the
    oracle, over each sequence's own blocks."""
    w = wl.WORKLOADS["llama3_70b_gqa8"]
    pin = wl.make_prefill(w, np.full(w.num_seqs, 4), device="cuda")
    out = _run(pkv, pin)
    inp = pin.paged
    lens = inp.lengths
    for b in (0, int(np.argmax(lens)), int(np.argmin(lens)), 100, 255):
        L = int(lens[b])
        need = (L + w.block_size - 1) // w.block_size
        ids = torch.from_numpy(
            inp.block_tables[b, :need].astype(np.int64)).cuda()
        kc = to_np(inp.k_cache.index_select(0, ids))
        vc = to_np(inp.v_cache.index_select(0, ids))
        rows = np.arange(pin.query_start[b], pin.query_start[b + 1])
        sub = np.arange(need, dtype=np.int32)[None, :]
        ref = oa.paged_prefill(to_np(pin.q)[rows], kc, vc, sub,
                               np.array([L]), np.array([0, len(rows)],
                                                       dtype=np.int32),
                               w.softmax_scale)
        check_prefill(*out, ref, f"verify seq {b}", rows=rows)


@pytest.mark.parametrize("dtype", ["bfloat16", "float16"])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8)])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_few_rows_33_to_64(pkv, dtype, hq, hkv, bs, head_dim):
    """33 .. 64 query rows per KV head (the tile kernel's 16-rows-per-warp
    layout: two rows per thread), contexts around the tile edges."""
    G = hq // hkv
    qmax = 64 // G
    lens = (1, 17, 130, 300, 520, 64, 700, 33, 129, 128, 255, 256)
    want = (1, qmax, qmax - 1, 32 // G + 1, 2, qmax, qmax, 0, qmax, 1, 5,
            qmax)
    qlens = tuple(min(L, q) for L, q in zip(lens, want))
    assert 32 < max(qlens) * G <= 64
    w = wl.Workload("prefill_rows64", 24, len(lens), hq, hkv, head_dim, bs,
                    dtype, "fixed", fixed_lengths=lens)
    pin = wl.make_prefill(w, qlens, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(pkv, pin, err=err)
    assert err.item() == 0
    _check(pin, out, f"rows<=64 {dtype}/{hq}:{hkv}/bs{bs}/d{head_dim}")
