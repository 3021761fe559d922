"""All rows together on one pool, the way a serving loop drives them:

1. request A prefills a 200-token prompt and caches its full blocks;
2. request B arrives with the same prompt plus a question: it matches the
   cached prefix, prefills only its own tokens;
3. decode steps for A and B (one new token each, cache write then decode);
4. B verifies 4 draft tokens in one pass and keeps 2 (rollback);
5. A is preempted: swapped out to a pinned host pool, and request C takes
   the device blocks A freed;
6. A is swapped back in and a decode step runs for A, B and C.

Every attention output is checked against the oracle over each sequence's
logical K/V, tracked on the host from the inputs alone."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from paged_kv_cache_383_b200 import flow

from helpers import check_decode, check_prefill, prefill_both, to_np

pytestmark = pytest.mark.gpu

HQ, HKV, D, BS = 32, 8, 128, 16
SCALE = D ** -0.5


def _pool(K, V, bs):
    """Host pool holding each sequence's K/V in consecutive blocks, and the
    identity tables that reach them."""
    nblk = [(len(k) + bs - 1) // bs for k in K]
    kp = np.zeros((sum(nblk), HKV, bs, D))
    vp = np.zeros_like(kp)
    tables = np.full((len(K), max(nblk)), -1, dtype=np.int32)
    base = 0
    for b, (k, v) in enumerate(zip(K, V)):
        t = np.arange(len(k))
        kp[base + t // bs, :, t % bs] = k
        vp[base + t // bs, :, t % bs] = v
        tables[b, :nblk[b]] = np.arange(base, base + nblk[b])
        base += nblk[b]
    return kp, vp, tables


class Flow:
    def __init__(self, pkv, num_blocks=64, host_blocks=40):
        self.pkv = pkv
        self.g = torch.Generator(device="cuda")
        self.g.manual_seed(383011)
        self.kc = self.rnd(num_blocks, HKV, BS, D)
        self.vc = self.rnd(num_blocks, HKV, BS, D)
        self.bm = pkv.BlockManager(num_blocks, BS)
        self.bm.set_host_blocks(host_blocks)
        self.hk = torch.empty((host_blocks, HKV, BS, D),
                              dtype=torch.bfloat16, pin_memory=True)
        self.hv = torch.empty_like(self.hk, pin_memory=True)
        self.K, self.V, self.tok = {}, {}, {}
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def rnd(self, *shape):
        return torch.randn(*shape, generator=self.g,
                           device="cuda").to(torch.bfloat16)

    def write(self, s, k, v, toks):
        """Append and write tokens of sequence s (K/V given), track them."""
        flow.write_tokens(self.bm, self.kc, self.vc, [s], [len(toks)], k, v,
                          dev_err=self.err)
        self.K[s] = np.concatenate([self.K[s], to_np(k)])
        self.V[s] = np.concatenate([self.V[s], to_np(v)])
        self.tok[s] = self.tok[s] + list(toks)

    def new_seq(self, s, prompt_toks, prompt_k, prompt_v):
        """Match the cached prefix, then write the rest; returns the match."""
        self.bm.add_seq(s)
        hit = self.bm.match_prefix(s, prompt_toks)
        self.K[s] = to_np(prompt_k[:hit])
        self.V[s] = to_np(prompt_v[:hit])
        self.tok[s] = list(prompt_toks[:hit])
        self.write(s, prompt_k[hit:], prompt_v[hit:], prompt_toks[hit:])
        return hit

    def attend(self, seqs, q_lens, what):
        """Causal attention of each sequence's newest q_len tokens, through
        pa_prefill (q_len > 1) or pa_decode (all q_len == 1)."""
        bt, cl, lens = flow.tables_on_device(self.bm, seqs, 64, "cuda")
        qs = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        q = self.rnd(int(qs[-1]), HQ, D)
        out, out32 = torch.empty_like(q), None
        if max(q_lens) == 1:
            self.pkv.pa_decode(out, q, self.kc, self.vc, bt, cl, SCALE,
                               max_context_len=int(lens.max()),
                               dev_err=self.err)
        else:
            out32 = prefill_both(self.pkv, out, q, self.kc, self.vc, bt, cl,
                                 torch.from_numpy(qs).cuda(), SCALE,
                                 max_q_len=max(q_lens),
                                 max_context_len=int(lens.max()),
                                 dev_err=self.err)
        kp, vp, tables = _pool([self.K[s] for s in seqs],
                               [self.V[s] for s in seqs], BS)
        assert list(lens) == [len(self.K[s]) for s in seqs]
        ref = oa.paged_prefill(to_np(q), kp, vp, tables, lens, qs, SCALE)
        torch.cuda.synchronize()
        assert self.err.item() == 0, what
        if out32 is None:
            check_decode(to_np(out), ref, q.dtype, what)
        else:
            check_prefill(out, out32, ref, what)

    def swap(self, seqs, out):
        if out:
            pairs = self.bm.swap_out(seqs)
            dst = (self.hk, self.hv, self.kc, self.vc)
        else:
            pairs = self.bm.swap_in(seqs)
            dst = (self.kc, self.vc, self.hk, self.hv)
        self.pkv.pa_swap_blocks(*dst, torch.from_numpy(
            np.ascontiguousarray(pairs)).cuda(), dev_err=self.err)
        return pairs


def test_prefix_prefill_decode_verify_preempt_resume(pkv):
    f = Flow(pkv)
    A, B, C = 0, 1, 2
    prompt = list(range(5000, 5200))
    pk, pv = f.rnd(200, HKV, D), f.rnd(200, HKV, D)

    # 1. A prefills its whole prompt and caches it
    assert f.new_seq(A, prompt, pk, pv) == 0
    f.attend([A], [200], "A prompt")
    f.bm.cache_insert(A, f.tok[A])

    # 2. B: same prompt + 50-token question; only its own tokens prefilled
    question = list(range(9000, 9050))
    qk, qv = f.rnd(50, HKV, D), f.rnd(50, HKV, D)
    hit = f.new_seq(B, prompt + question, torch.cat([pk, qk]),
                    torch.cat([pv, qv]))
    assert hit == 192                       # 12 full cached blocks
    f.attend([B], [250 - hit], "B suffix over the cached prompt")
    f.bm.cache_insert(B, f.tok[B])
    shared = f.bm.block_table([A, B], 32)[0][:, :12]
    assert (shared[0] == shared[1]).all()

    # 3. three decode steps for A and B
    for step in range(3):
        for s in (A, B):
            f.write(s, f.rnd(1, HKV, D), f.rnd(1, HKV, D), [7000 + step])
        f.attend([A, B], [1, 1], f"decode step {step}")

    # 4. B verifies 4 drafts in one pass, keeps 2
    f.write(B, f.rnd(4, HKV, D), f.rnd(4, HKV, D), [1, 2, 3, 4])
    f.attend([B], [4], "B verifies drafts")
    keep = len(f.K[B]) - 2
    f.bm.truncate(B, keep)
    f.K[B], f.V[B], f.tok[B] = f.K[B][:keep], f.V[B][:keep], f.tok[B][:keep]

    # 5. A is preempted; C takes every block but what A needs to come back
    #    and one for C's next token
    need_back = f.bm.num_seq_blocks(A)
    f.swap([A], out=True)
    assert f.bm.is_swapped(A)
    c_tokens = (f.bm.num_free() - need_back - 1) * BS
    assert c_tokens > 0
    f.new_seq(C, list(range(20000, 20000 + c_tokens)),
              f.rnd(c_tokens, HKV, D), f.rnd(c_tokens, HKV, D))
    f.attend([B, C], [1, 1], "B and C while A is out")

    # 6. A comes back (its private copies; cache leaves evicted if needed)
    f.swap([A], out=False)
    for s in (A, B, C):
        f.write(s, f.rnd(1, HKV, D), f.rnd(1, HKV, D), [8000])
    f.attend([A, B, C], [1, 1, 1], "decode after resume")
    assert f.bm.num_used() + f.bm.num_free() == 64
