"""Pins of the causal (prefill / multi-query) oracle.

* torch's float64 SDPA with is_causal=True on contiguous K/V, for a whole
  prompt (q_len = L);
* torch's float64 SDPA with an explicit boolean mask for chunks (q_len < L):
  new token i sees the L - q_len + i + 1 oldest tokens;
* q_len = 1 equals the decode oracle (itself pinned to SDPA);
* closed form: the first token of a fresh prompt attends only to itself, so
  its output is its own value row.
"""
import math

import numpy as np
import torch

from oracle import attention as oa

from test_oracle_attention import _scatter_to_pool


def _case(seed, lens, qlens, Hq, Hkv, D, bs):
    rng = np.random.default_rng(seed)
    Ks = [rng.standard_normal((L, Hkv, D)) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)) for L in lens]
    qs = np.concatenate([rng.standard_normal((n, Hq, D)) for n in qlens])
    start = np.concatenate([[0], np.cumsum(qlens)])
    nb = sum(-(-L // bs) for L in lens) + 4
    kc, vc, bt = _scatter_to_pool(rng, Ks, Vs, bs, nb)
    return qs, Ks, Vs, kc, vc, bt, np.array(lens), start


def _sdpa_chunk(q, K, V, L, scale):
    """q [n, Hq, D], K/V [L, Hkv, D]; boolean mask for the chunk."""
    n, Hq, D = q.shape
    G = Hq // K.shape[1]
    k = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)
    v = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)
    qq = torch.from_numpy(q).permute(1, 0, 2)                    # [Hq, n, D]
    pos = torch.arange(L - n, L)[:, None]
    mask = torch.arange(L)[None, :] <= pos                       # [n, L]
    o = torch.nn.functional.scaled_dot_product_attention(
        qq, k, v, attn_mask=mask, scale=scale)
    return o.permute(1, 0, 2).numpy()


def test_whole_prompt_matches_sdpa_causal():
    q, Ks, Vs, kc, vc, bt, lens, start = _case(1, [37, 16, 50], [37, 16, 50],
                                              8, 2, 8, 16)
    scale = 1 / math.sqrt(8)
    got = oa.paged_prefill(q, kc, vc, bt, lens, start, scale)
    for b in range(3):
        G = 4
        k = torch.from_numpy(Ks[b]).permute(1, 0, 2).repeat_interleave(G, 0)
        v = torch.from_numpy(Vs[b]).permute(1, 0, 2).repeat_interleave(G, 0)
        qq = torch.from_numpy(q[start[b]:start[b + 1]]).permute(1, 0, 2)
        want = torch.nn.functional.scaled_dot_product_attention(
            qq, k, v, is_causal=True, scale=scale).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[start[b]:start[b + 1]], want,
                                   rtol=0, atol=1e-12)


def test_chunks_match_sdpa_with_mask():
    q, Ks, Vs, kc, vc, bt, lens, start = _case(2, [70, 33, 20], [5, 33, 1],
                                              16, 2, 8, 16)
    scale = 0.3
    got = oa.paged_prefill(q, kc, vc, bt, lens, start, scale)
    for b in range(3):
        want = _sdpa_chunk(q[start[b]:start[b + 1]], Ks[b], Vs[b], lens[b],
                           scale)
        np.testing.assert_allclose(got[start[b]:start[b + 1]], want,
                                   rtol=0, atol=1e-12)


def test_single_new_token_equals_decode():
    q, Ks, Vs, kc, vc, bt, lens, start = _case(3, [40, 9], [1, 1], 8, 8, 4, 16)
    got = oa.paged_prefill(q, kc, vc, bt, lens, start, 0.5)
    want = oa.paged_decode(q, kc, vc, bt, lens, 0.5)
    np.testing.assert_array_equal(got, want)


def test_first_prompt_token_returns_its_value():
    q, Ks, Vs, kc, vc, bt, lens, start = _case(4, [12], [12], 4, 2, 8, 16)
    got = oa.paged_prefill(q, kc, vc, bt, lens, start, 0.7)
    for h in range(4):
        assert np.array_equal(got[0, h], Vs[0][0, h // 2])
