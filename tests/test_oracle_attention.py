"""Pins of the fp64 attention oracle to things other than itself.

* a library routine: torch's float64 scaled-dot-product attention on the
  contiguous K/V the paged cache was built from (the pages: paged attention is
  mathematically identical to contiguous multi-head attention);
* brute force at 60 significant digits with Python's ``decimal`` module on
  tiny inputs;
* closed forms: one token, equal keys, zero query, two tokens;
* invariance of the output under any relabelling of physical blocks;
* a GQA mapping probe where each KV head carries a distinct constant value.

The last tests plant mistakes in copies of the oracle (on the CPU) and check
that at least one pin fails for each.
"""
import decimal
import math

import numpy as np
import pytest
import torch

from oracle import attention as oa


def _scatter_to_pool(rng, K_seqs, V_seqs, block_size, num_blocks):
    """Test-side paging: put each sequence's contiguous K/V into randomly
    chosen physical blocks of a pool that is pre-filled with noise."""
    Hkv, D = K_seqs[0].shape[1], K_seqs[0].shape[2]
    kc = rng.standard_normal((num_blocks, Hkv, block_size, D)) * 7.0
    vc = rng.standard_normal((num_blocks, Hkv, block_size, D)) * 7.0
    order = rng.permutation(num_blocks)
    need = [-(-K.shape[0] // block_size) for K in K_seqs]
    max_blocks = max(need + [1])
    tables = -np.ones((len(K_seqs), max_blocks), dtype=np.int64)
    nxt = 0
    for b, (K, V) in enumerate(zip(K_seqs, V_seqs)):
        for i in range(need[b]):
            phys = order[nxt]
            nxt += 1
            tables[b, i] = phys
            rows = slice(i * block_size, min((i + 1) * block_size, K.shape[0]))
            n = rows.stop - rows.start
            kc[phys, :, :n, :] = K[rows].transpose(1, 0, 2)
            vc[phys, :, :n, :] = V[rows].transpose(1, 0, 2)
    return kc, vc, tables


def _case(seed, lens, Hq, Hkv, D, bs, extra_blocks=5):
    rng = np.random.default_rng(seed)
    K_seqs = [rng.standard_normal((L, Hkv, D)) for L in lens]
    V_seqs = [rng.standard_normal((L, Hkv, D)) for L in lens]
    q = rng.standard_normal((len(lens), Hq, D))
    nb = sum(-(-L // bs) for L in lens) + extra_blocks
    kc, vc, tables = _scatter_to_pool(rng, K_seqs, V_seqs, bs, nb)
    return q, K_seqs, V_seqs, kc, vc, tables, np.array(lens)


def _sdpa(q, K_seqs, V_seqs, scale):
    """torch float64 SDPA over contiguous K/V, GQA by consecutive groups."""
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        Hkv = K_seqs[b].shape[1]
        G = Hq // Hkv
        k = torch.from_numpy(K_seqs[b]).permute(1, 0, 2)       # [Hkv, L, D]
        v = torch.from_numpy(V_seqs[b]).permute(1, 0, 2)
        k = k.repeat_interleave(G, dim=0)                       # [Hq, L, D]
        v = v.repeat_interleave(G, dim=0)
        qq = torch.from_numpy(q[b]).unsqueeze(1)                # [Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(
            qq, k, v, scale=scale)
        out[b] = o[:, 0, :].numpy()
    return out


@pytest.mark.parametrize("lens,Hq,Hkv,D,bs", [
    ([47, 61, 13, 19], 8, 8, 16, 16),     # MHA, ragged tails
    ([33, 16, 1, 50], 8, 2, 8, 16),       # GQA 4
    ([70, 5, 32], 16, 2, 8, 32),          # GQA 8, block 32
])
def test_matches_torch_sdpa_on_contiguous(lens, Hq, Hkv, D, bs):
    q, Ks, Vs, kc, vc, bt, cl = _case(11, lens, Hq, Hkv, D, bs)
    scale = 1.0 / math.sqrt(D)
    got = oa.paged_decode(q, kc, vc, bt, cl, scale)
    want = _sdpa(q, Ks, Vs, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    got_c = oa.contiguous_decode(q, Ks, Vs, scale)
    np.testing.assert_allclose(got_c, want, rtol=0, atol=1e-12)


def _decimal_attention(q, K, V, scale):
    """Brute force at 60 digits: weights one by one, then the weighted sum."""
    ctx = decimal.Context(prec=60)
    Dm = decimal.Decimal
    scores = []
    for t in range(K.shape[0]):
        acc = Dm(0)
        for d in range(K.shape[1]):
            acc = ctx.add(acc, ctx.multiply(Dm(float(q[d])), Dm(float(K[t, d]))))
        scores.append(ctx.multiply(acc, Dm(scale)))
    exps = [ctx.exp(s) for s in scores]
    total = sum(exps, Dm(0))
    out = []
    for d in range(V.shape[1]):
        num = sum((ctx.multiply(e, Dm(float(V[t, d])))
                   for t, e in enumerate(exps)), Dm(0))
        out.append(float(ctx.divide(num, total)))
    return np.array(out)


def test_matches_brute_force_decimal():
    q, Ks, Vs, kc, vc, bt, cl = _case(5, [7, 3, 17], 4, 2, 6, 4)
    scale = 0.37
    got = oa.paged_decode(q, kc, vc, bt, cl, scale)
    for b in range(3):
        for h in range(4):
            kvh = h // 2
            want = _decimal_attention(q[b, h], Ks[b][:, kvh], Vs[b][:, kvh],
                                      scale)
            np.testing.assert_allclose(got[b, h], want, rtol=0, atol=1e-13)


def test_single_token_returns_its_value():
    q, Ks, Vs, kc, vc, bt, cl = _case(3, [1, 1], 4, 4, 8, 16)
    got = oa.paged_decode(q, kc, vc, bt, cl, 0.5)
    for b in range(2):
        for h in range(4):
            assert np.array_equal(got[b, h], Vs[b][0, h])


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(8)
    L, D = 29, 8
    K = np.tile(rng.standard_normal(D), (L, 1))
    V = rng.standard_normal((L, D))
    got = oa.attend(rng.standard_normal(D), K, V, 0.9)
    np.testing.assert_allclose(got, V.mean(axis=0), rtol=0, atol=1e-14)


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(9)
    K = rng.standard_normal((40, 8))
    V = rng.standard_normal((40, 8))
    np.testing.assert_allclose(oa.attend(np.zeros(8), K, V, 1.0),
                               V.mean(axis=0), rtol=0, atol=1e-14)


def test_two_tokens_closed_form():
    rng = np.random.default_rng(10)
    q, K, V = rng.standard_normal(8), rng.standard_normal((2, 8)), \
        rng.standard_normal((2, 8))
    scale = 0.3
    s0, s1 = scale * K[0] @ q, scale * K[1] @ q
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(oa.attend(q, K, V, scale),
                               w0 * V[0] + (1 - w0) * V[1], rtol=0, atol=1e-14)


def test_empty_sequence_gives_zeros():
    rng = np.random.default_rng(1)
    out = oa.attend(rng.standard_normal(8), np.zeros((0, 8)),
                    np.zeros((0, 8)), 1.0)
    assert np.array_equal(out, np.zeros(8))


def test_invariant_under_block_relabelling():
    q, Ks, Vs, kc, vc, bt, cl = _case(21, [47, 100, 9], 8, 4, 8, 16,
                                      extra_blocks=30)
    base = oa.paged_decode(q, kc, vc, bt, cl, 0.25)
    rng = np.random.default_rng(99)
    for _ in range(3):
        perm = rng.permutation(kc.shape[0])      # new id of old block i
        kc2 = np.empty_like(kc)
        vc2 = np.empty_like(vc)
        kc2[perm] = kc
        vc2[perm] = vc
        bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
        got = oa.paged_decode(q, kc2, vc2, bt2, cl, 0.25)
        assert np.array_equal(got, base)


def test_gqa_head_mapping_probe():
    # KV head j carries V == j everywhere; query head h must return h // G.
    B, Hq, Hkv, D, bs, L = 2, 8, 2, 4, 16, 37
    rng = np.random.default_rng(4)
    Ks = [rng.standard_normal((L, Hkv, D)) for _ in range(B)]
    Vs = [np.broadcast_to(np.arange(Hkv, dtype=float)[None, :, None],
                          (L, Hkv, D)).copy() for _ in range(B)]
    q = rng.standard_normal((B, Hq, D))
    kc, vc, bt = _scatter_to_pool(rng, Ks, Vs, bs, 10)
    got = oa.paged_decode(q, kc, vc, bt, np.array([L, L]), 0.5)
    for h in range(Hq):
        np.testing.assert_allclose(got[:, h], h // (Hq // Hkv), atol=1e-14)


def test_depage_rejects_bad_block_id():
    kc = np.zeros((4, 1, 16, 2))
    with pytest.raises(IndexError):
        oa.depage(kc, np.array([0, 9]), 20, 0, 16)


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin.

def _pins_pass(paged_decode):
    try:
        for lens, Hq, Hkv, D, bs in [([47, 61, 13, 19], 8, 8, 16, 16),
                                     ([33, 16, 1, 50], 8, 2, 8, 16)]:
            q, Ks, Vs, kc, vc, bt, cl = _case(11, lens, Hq, Hkv, D, bs)
            scale = 1.0 / math.sqrt(D)
            got = paged_decode(q, kc, vc, bt, cl, scale)
            want = _sdpa(q, Ks, Vs, scale)
            if not np.allclose(got, want, rtol=0, atol=1e-12):
                return False
        return True
    except (IndexError, ValueError):
        return False


def _mutant(monkeypatch, name, fn):
    monkeypatch.setattr(oa, name, fn)
    return oa.paged_decode


def test_unmutated_oracle_passes_pins():
    assert _pins_pass(oa.paged_decode)


@pytest.mark.parametrize("mutation", [
    "offset_from_quotient", "dropped_scale", "keys_for_values",
    "no_max_subtraction_wrong_sign", "kv_head_modulo", "off_by_one_block"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    real_depage, real_attend = oa.depage, oa.attend

    if mutation == "offset_from_quotient":
        def depage(cache, row, L, kvh, bs):
            t = np.arange(L)
            return np.asarray(cache[np.asarray(row)[t // bs], kvh,
                                    (t // bs) % bs], dtype=float)
        pd = _mutant(monkeypatch, "depage", depage)
    elif mutation == "dropped_scale":
        pd = _mutant(monkeypatch, "attend",
                     lambda q, K, V, s: real_attend(q, K, V, 1.0))
    elif mutation == "keys_for_values":
        pd = _mutant(monkeypatch, "attend",
                     lambda q, K, V, s: real_attend(q, K, K, s))
    elif mutation == "no_max_subtraction_wrong_sign":
        def attend(q, K, V, s):
            w = np.exp(-s * (K @ q))
            return (w / w.sum()) @ V
        pd = _mutant(monkeypatch, "attend", attend)
    elif mutation == "kv_head_modulo":
        pd = _mutant(monkeypatch, "kv_head_of",
                     lambda h, hq, hkv: h % hkv)
    elif mutation == "off_by_one_block":
        def depage(cache, row, L, kvh, bs):
            t = np.arange(L)
            blk = np.asarray(row)[np.minimum(t // bs + 1, len(row) - 1)]
            return np.asarray(cache[blk, kvh, t % bs], dtype=float)
        pd = _mutant(monkeypatch, "depage", depage)
    assert not _pins_pass(pd), mutation
    monkeypatch.setattr(oa, "depage", real_depage)
    monkeypatch.setattr(oa, "attend", real_attend)
