"""GPU flow of the prefix cache: requests sharing a system prompt reference
its cached K/V blocks and prefill only their own tokens ([KV-cache chapter]
"RadixAttention: caching, not just packing, the prefix"); the result equals
the oracle's causal attention over the full contiguous K/V."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import flow

from helpers import check_prefill, prefill_both, to_np

pytestmark = pytest.mark.gpu


def _pool(K_seqs, V_seqs, bs):
    nblk = [(len(k) + bs - 1) // bs for k in K_seqs]
    hkv, d = K_seqs[0].shape[1:]
    kp = np.zeros((sum(nblk), hkv, bs, d))
    vp = np.zeros_like(kp)
    tables = np.full((len(K_seqs), max(nblk)), -1, dtype=np.int32)
    base = 0
    for b, (k, v) in enumerate(zip(K_seqs, V_seqs)):
        t = np.arange(len(k))
        kp[base + t // bs, :, t % bs] = k
        vp[base + t // bs, :, t % bs] = v
        tables[b, :nblk[b]] = np.arange(base, base + nblk[b])
        base += nblk[b]
    return kp, vp, tables


@pytest.mark.parametrize("bs", [16, 32])
def test_shared_prompt_prefills_only_the_suffix(pkv, bs):
    hq, hkv, d = 32, 8, 128
    prompt_len, questions = 200, [37, 64, 5, 120]
    g = torch.Generator(device="cuda")
    g.manual_seed(383008 + bs)
    rnd = lambda *s: torch.randn(*s, generator=g, device="cuda").to(
        torch.bfloat16)
    nb = 128
    kc, vc = rnd(nb, hkv, bs, d), rnd(nb, hkv, bs, d)
    bm = pkv.BlockManager(nb, bs)
    prompt = list(range(1000, 1000 + prompt_len))
    pk, pv = rnd(prompt_len, hkv, d), rnd(prompt_len, hkv, d)
    scale = d ** -0.5
    K, V, hits = [], [], []
    for r, qlen in enumerate(questions):
        toks = prompt + [50_000 + 1000 * r + i for i in range(qlen)]
        qk, qv = rnd(qlen, hkv, d), rnd(qlen, hkv, d)
        bm.add_seq(r)
        hit = bm.match_prefix(r, toks)
        hits.append(hit)
        # K/V of the tokens past the cached prefix: the rest of the prompt
        # (only the first request computes all of it), then the question
        new_k = torch.cat([pk[hit:], qk]) if hit < prompt_len else qk
        new_v = torch.cat([pv[hit:], qv]) if hit < prompt_len else qv
        flow.write_tokens(bm, kc, vc, [r], [len(toks) - hit], new_k, new_v)
        n_new = len(toks) - hit
        q = rnd(n_new, hq, d)
        bt, cl, lens = flow.tables_on_device(bm, [r], 32, "cuda")
        qs = torch.tensor([0, n_new], dtype=torch.int32, device="cuda")
        out = torch.empty_like(q)
        out32 = prefill_both(pkv, out, q, kc, vc, bt, cl, qs, scale,
                             max_q_len=n_new, max_context_len=int(lens[0]))
        bm.cache_insert(r, toks)
        Kr = np.concatenate([to_np(pk), to_np(qk)])
        Vr = np.concatenate([to_np(pv), to_np(qv)])
        kp, vp, tables = _pool([Kr], [Vr], bs)
        ref = oa.paged_prefill(to_np(q), kp, vp, tables, lens,
                               np.array([0, n_new]), scale)
        torch.cuda.synchronize()
        check_prefill(out, out32, ref, f"request {r}")
        K.append(Kr)
        V.append(Vr)
    shared = bs * (prompt_len // bs)
    assert hits == [0] + [shared] * (len(questions) - 1)
    # the prompt's full blocks are stored once
    table, _ = bm.block_table(list(range(len(questions))), 32)
    assert len({tuple(row[:prompt_len // bs]) for row in table}) == 1
