"""GPU: pa_cache_write and pa_copy_blocks are byte-exact.

The expected cache is built on the host by plain indexing of the same bytes
(the operations are permutations of bytes, so their result is fixed exactly).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _pool(nb, hkv, bs, d, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    k = torch.randn(nb, hkv, bs, d, generator=g, device="cuda").to(dtype)
    v = torch.randn(nb, hkv, bs, d, generator=g, device="cuda").to(dtype)
    return k, v


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("hkv,bs,d", [(8, 16, 128), (2, 32, 64), (1, 16, 8)])
def test_cache_write_exact(pkv, dtype, hkv, bs, d):
    nb, T = 50, 300
    kc, vc = _pool(nb, hkv, bs, d, dtype, 1)
    rng = np.random.default_rng(2)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[::7] = -1                                   # padding tokens
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    k = torch.randn(T, hkv, d, generator=g, device="cuda").to(dtype)
    v = torch.randn(T, hkv, d, generator=g, device="cuda").to(dtype)
    want_k, want_v = kc.cpu().clone(), vc.cpu().clone()
    for t, s in enumerate(slots):
        if s >= 0:
            want_k[s // bs, :, s % bs, :] = k[t].cpu()
            want_v[s // bs, :, s % bs, :] = v[t].cpu()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_cache_write(kc, vc, k, v, torch.from_numpy(slots).cuda(),
                       dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(kc.cpu().view(torch.int16), want_k.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), want_v.view(torch.int16))


def test_cache_write_out_of_range_slot_is_flagged(pkv):
    kc, vc = _pool(4, 2, 16, 64, torch.bfloat16, 4)
    before_k = kc.clone()
    k = torch.ones(2, 2, 64, dtype=torch.bfloat16, device="cuda")
    slots = torch.tensor([4 * 16, 5], dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_cache_write(kc, vc, k, k, slots, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    want = before_k.clone()
    want[0, :, 5, :] = 1
    assert torch.equal(kc, want)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_copy_blocks_exact(pkv, dtype):
    nb = 64
    kc, vc = _pool(nb, 8, 16, 128, dtype, 5)
    rng = np.random.default_rng(6)
    ids = rng.permutation(nb)
    pairs = np.stack([ids[:20], ids[20:40]], axis=1).astype(np.int32)
    want_k, want_v = kc.cpu().clone(), vc.cpu().clone()
    for s, d in pairs:
        want_k[d] = want_k[s]
        want_v[d] = want_v[s]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(kc.cpu().view(torch.int16), want_k.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), want_v.view(torch.int16))


def test_copy_blocks_bad_id_is_flagged(pkv):
    kc, vc = _pool(8, 2, 16, 64, torch.float16, 7)
    before = kc.clone()
    pairs = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pa_copy_blocks(kc, vc, pairs, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 5
    want = before.clone()
    want[2] = before[1]
    assert torch.equal(kc, want)
